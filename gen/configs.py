"""The five workload shapes of the routed-expert layer.

Shapes follow the Edge0 pages: the 35B-A3B tier has 40 layers, 256 routed
experts, top-4 routing and hidden size 2048 (autoark.ai blog, tier table;
2kiu.com article, "model structure" paragraph); the 8B-A1B tier has 24 layers,
128 routed experts and top-8 (same table).  Expert intermediate size, shared
expert size, LoRA rank and Prerouter width are synthetic choices stated with
each workload.

This module holds plain data only: no arithmetic of the method.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class MoEConfig:
    cfg_id: int
    name: str
    T: int            # tokens per step
    layers: int
    H: int            # hidden size
    E: int            # routed experts
    K: int            # experts per token
    I: int            # routed expert intermediate size
    I_s: int          # shared expert intermediate size
    r: int            # LoRA rank
    P: int            # Prerouter hidden width
    lora_shared: bool = True        # LoRA on every shared-expert projection
    lora_routed_down: bool = False  # LoRA on every routed expert's down projection
    lora_routed_gate_up: bool = False  # LoRA on every routed expert's gate and up projections
    zipf_s: float = 0.0             # per-expert router logit offset exponent (0 = none)
    predicted_routing: bool = False  # layers >= 1 route by the previous head's prediction

    @property
    def G(self) -> int:
        return self.H // 64

    @property
    def E_next(self) -> int:
        # every head predicts a layer of the same stack
        return self.E


CONFIGS = [
    MoEConfig(0, "tiny layer", T=4, layers=1, H=256, E=16, K=2, I=128, I_s=128, r=8, P=64),
    MoEConfig(1, "35B-shaped decode", T=1, layers=40, H=2048, E=256, K=4, I=512, I_s=512, r=16, P=256),
    MoEConfig(2, "8B-shaped decode", T=1, layers=24, H=2048, E=128, K=8, I=512, I_s=512, r=16, P=256),
    MoEConfig(3, "35B-shaped prefill", T=3328, layers=40, H=2048, E=256, K=4, I=512, I_s=512, r=16, P=256,
              zipf_s=1.1),
    MoEConfig(4, "35B-shaped batched decode", T=64, layers=40, H=2048, E=256, K=4, I=512, I_s=512, r=16, P=256,
              lora_routed_down=True, predicted_routing=True),
]


def get(cfg_id: int) -> MoEConfig:
    return CONFIGS[cfg_id]
