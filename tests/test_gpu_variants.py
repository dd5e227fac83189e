"""GPU parity of the layer variants: several LoRA adapters over one read-only base, and the 8B shape at many
tokens (tensor-core router, grouped GEMMs at top-8, tensor-core Prerouter first layer)."""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

from gen import CONFIGS, inputs
from gen.inputs import NO_EXPERT, TID
from oracle import moe_oracle as O
from parity import assert_close_inf, check_topk, prerouter_tau, router_tau_tc
from test_gpu_layer import Layer, M, expert_forward, oracle_out, prerouter, route, u_vals

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _adapter(cfg, layer_idx, seed):
    """Another set of LoRA tensors for the same layer: the shared expert's three projections and every routed
    expert's down projection, drawn with another seed."""
    sh = {f"lora_{p}": inputs.lora(cfg, layer_idx, NO_EXPERT, TID[f"sh_A_{p}"], TID[f"sh_B_{p}"],
                                   cfg.H if p == "down" else cfg.I_s, cfg.I_s if p == "down" else cfg.H, seed)
          for p in ("gate", "up", "down")}
    ex = {e: inputs.lora(cfg, layer_idx, e, TID["ex_A_down"], TID["ex_B_down"], cfg.H, cfg.I, seed)
          for e in range(cfg.E)}
    return sh, ex


class AdapterView:
    """A layer struct over the same read-only base (router, shared expert, expert pool) with other LoRA tensors."""

    def __init__(self, layer: Layer, sh: dict, ex: dict):
        from int4_expert_ffn_top_b200 import _lib
        s = _lib.moe_layer()
        ctypes.memmove(ctypes.byref(s), ctypes.byref(layer.dev.struct), ctypes.sizeof(s))
        self.keep = []
        for i, p in enumerate(("gate", "up", "down")):
            A = torch.from_numpy(sh[f"lora_{p}"]["A"]).to(DEV)
            B = torch.from_numpy(sh[f"lora_{p}"]["B"]).to(DEV)
            self.keep += [A, B]
            s.sh_lora_A[i], s.sh_lora_B[i] = A.data_ptr(), B.data_ptr()
        exA = torch.from_numpy(np.stack([ex[e]["A"] for e in range(len(ex))])).to(DEV)
        exB = torch.from_numpy(np.stack([ex[e]["B"] for e in range(len(ex))])).to(DEV)
        self.keep += [exA, exB]
        s.ex_lora_A, s.ex_lora_B = exA.data_ptr(), exB.data_ptr()
        self.struct = s


@pytest.mark.parametrize("T", [4, 64])  # GEMV path and grouped-GEMM path
def test_two_adapters_over_one_read_only_base(cuda_ok, T):
    cfg = dataclasses.replace(CONFIGS[0], lora_routed_down=True)
    lay = Layer(cfg, 0)
    sh2, ex2 = _adapter(cfg, 0, seed=1)
    view = AdapterView(lay, sh2, ex2)
    host2 = dict(lay.host, shared=dict(lay.host["shared"], **sh2),
                 experts={e: dict(x, down_lora=ex2[e]) for e, x in lay.host["experts"].items()})
    m = M()
    base_bytes = lay.dev.pool.clone()
    ub = inputs.activations(cfg, step=60 + T, T=T)
    u = u_vals(ub)
    _, idx, w = route(lay, ub, cfg.K)
    out1, _ = expert_forward(lay, ub, cfg.K, idx, w)
    out2 = torch.full((T, cfg.H), float("nan"), device=DEV)
    m.moe_expert_forward(view, torch.from_numpy(ub.view(np.int16)).to(DEV), cfg.K,
                         torch.from_numpy(idx.astype(np.int32)).to(DEV), torch.from_numpy(w.astype(np.float32)).to(DEV),
                         out2, 0, m.workspace(m.moe_workspace_size(view, T, cfg.K)))
    torch.cuda.synchronize()
    out2 = out2.cpu().numpy().astype(np.float64)
    ref1 = oracle_out(lay, u, idx, w)
    y2 = O.routed_outputs(u, host2["experts"], idx)
    ref2 = O.combine(w, y2, O.shared_gate(u, host2["shared"]), O.shared_expert(u, host2["shared"]))
    assert_close_inf(out1, ref1, what="adapter 1")
    assert_close_inf(out2, ref2, what="adapter 2")
    # the adapters matter (the test is not vacuous) and the base is untouched
    assert np.max(np.abs(ref1 - ref2)) > 5 * 2e-3 * np.max(np.abs(ref1))  # about 12x the tolerance here
    assert torch.equal(lay.dev.pool, base_bytes)


def test_8b_shape_prefill_layer(cuda_ok):
    """The 8B shape (128 experts, top-8) at 512 tokens: tensor-core router, grouped GEMMs, tensor-core Prerouter
    first layer; outputs checked on every 8th token."""
    cfg = CONFIGS[2]
    T = 512
    lay = Layer(cfg, 3)
    ub = inputs.activations(cfg, step=8, T=T)
    u = u_vals(ub)
    logits, idx, w = route(lay, ub, cfg.K)
    ref_logits = O.router_logits(u, lay.host["router"])
    tau = router_tau_tc(u, lay.host["router"])
    assert np.all(np.abs(logits - ref_logits) <= tau)
    check_topk(idx, ref_logits, tau, cfg.K)
    out, _ = expert_forward(lay, ub, cfg.K, idx, w)
    toks = np.arange(0, T, 8)
    assert_close_inf(out[toks], oracle_out(lay, u[toks], idx[toks], w[toks]))
    pred, scores = prerouter(lay, ub, idx, cfg.K)
    head = lay.host["prerouter"]
    ref_p = O.prerouter_scores(u[toks], idx[toks], head, cfg.E)
    tau_p = prerouter_tau(u[toks], idx[toks], head, cfg.E, tc=True)
    assert np.all(np.abs(scores[toks] - ref_p) <= tau_p)
    check_topk(pred[toks], ref_p, tau_p, cfg.K)


@pytest.mark.parametrize("T", [1, 4, 64])  # one token, below the 48-slot switch, above it: tensor cores throughout
def test_lora_on_every_routed_projection(cuda_ok, T):
    """LoRA on the gate, up and down projections of every routed expert (and of the shared expert)."""
    cfg = dataclasses.replace(CONFIGS[0], lora_routed_down=True, lora_routed_gate_up=True)
    lay = Layer(cfg, 0)
    ub = inputs.activations(cfg, step=70 + T, T=T)
    u = u_vals(ub)
    _, idx, w = route(lay, ub, cfg.K)
    out, _ = expert_forward(lay, ub, cfg.K, idx, w)
    ref = oracle_out(lay, u, idx, w)
    assert_close_inf(out, ref)
    # the gate/up adapters matter: without them the oracle's output moves by several times the tolerance
    bare = {e: {k: v for k, v in ex.items() if k not in ("gate_lora", "up_lora")} for e, ex in lay.host["experts"].items()}
    ref_bare = O.combine(w, O.routed_outputs(u, bare, idx), O.shared_gate(u, lay.host["shared"]),
                         O.shared_expert(u, lay.host["shared"]))
    assert np.max(np.abs(ref - ref_bare)) > 3 * 2e-3 * np.max(np.abs(ref))


def test_stack_with_lora_on_every_routed_projection(cuda_ok):
    """moe_stack_decode over layers whose routed experts carry gate/up/down adapters (the per-layer path)."""
    from test_gpu_layer import _check_stack, run_stack
    cfg = dataclasses.replace(CONFIGS[0], layers=3, lora_routed_down=True, lora_routed_gate_up=True)
    layer_fn = lambda l: inputs.layer(cfg, l)  # noqa: E731
    stack = M().DeviceStack(cfg, layer_fn)
    T = 1
    x0 = inputs.bf16_bits_to_f32(inputs.activations(cfg, step=19, T=T)) * 3.0
    res = run_stack(stack, cfg, T, x0, False)
    _check_stack(cfg, layer_fn, T, res, x0, range(cfg.layers))


@pytest.mark.parametrize("T", [4, 64])  # GEMV path and grouped-GEMM path
def test_shared_adapter_on_some_projections_only(cuda_ok, T):
    """A shared-expert adapter on the up and down projections but not the gate: each projection is taken on its
    own, and the gate's zero LoRA-A rows leave its products untouched."""
    cfg = CONFIGS[0]
    lay = Layer(cfg, 0)
    from int4_expert_ffn_top_b200 import _lib
    s = _lib.moe_layer()
    ctypes.memmove(ctypes.byref(s), ctypes.byref(lay.dev.struct), ctypes.sizeof(s))
    s.sh_lora_A[0] = s.sh_lora_B[0] = None

    class View:
        struct = s

    sh = {k: v for k, v in lay.host["shared"].items() if k != "lora_gate"}
    assert "lora_up" in sh and "lora_down" in sh
    ub = inputs.activations(cfg, step=80 + T, T=T)
    u = u_vals(ub)
    _, idx, w = route(lay, ub, cfg.K)
    m = M()
    out = torch.full((T, cfg.H), float("nan"), device=DEV)
    m.moe_expert_forward(View, torch.from_numpy(ub.view(np.int16)).to(DEV), cfg.K,
                         torch.from_numpy(idx.astype(np.int32)).to(DEV), torch.from_numpy(w.astype(np.float32)).to(DEV),
                         out, 0, m.workspace(m.moe_workspace_size(View, T, cfg.K)))
    torch.cuda.synchronize()
    ref = O.combine(w, O.routed_outputs(u, lay.host["experts"], idx), O.shared_gate(u, sh), O.shared_expert(u, sh))
    assert_close_inf(out.cpu().numpy().astype(np.float64), ref)
    full = oracle_out(lay, u, idx, w)  # the gate's adapter matters here
    assert np.max(np.abs(full - ref)) > 3 * 2e-3 * np.max(np.abs(ref))
