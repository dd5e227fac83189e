"""Seeded synthetic inputs for the routed-expert layer.

Every tensor is drawn from its own counter-addressed stream,
``Philox(SeedSequence([seed, cfg_id, layer, expert, tensor_id]))``, so any single
expert of any layer can be regenerated on the host by itself.  Both the CPU
oracle (through the tests) and the CUDA path (through the binding) consume these
arrays; this module holds none of the method's arithmetic, only the draws and
the storage formats:

* int4 matrix ``[out, in]``: ``q[out][in/8]`` uint32 with nibble ``k`` of a row
  at bits ``4*(k%8)`` of word ``k//8`` (low nibble first), codes uniform 0..15
  (a uniform 32-bit word carries eight uniform nibbles); ``scale[out][in/64]``
  fp16 ~ U(0.005, 0.02); ``bias = -8*scale`` (exact in fp16).  This is the
  4-bit affine, group-64 format of the Edge0 checkpoint config
  (2kiu.com article, "SSD expert offload" bullet).
* 8-bit matrix (router and shared-expert gate, which the checkpoint keeps at
  8 bits: 2kiu.com article, closing paragraph on config.json):
  ``q[out][in/4]`` uint32, low byte first, codes uniform 0..255,
  ``scale`` ~ U(0.005, 0.02)/16, ``bias = -128*scale``.
* LoRA ``A[r][in]``, ``B[out][r]`` fp16 ~ N(0, 0.02).
* Prerouter ``W1[P][H+E]`` ~ N(0, 1/sqrt(H+E)), ``W2[E][P]`` ~ N(0, 1/sqrt(P)),
  biases ~ N(0, 0.1), all fp16.
* Activations ~ N(0, 1) rounded to bf16 (round to nearest even), returned as
  uint16 bit patterns.
* Prefill router offset (Zipf reading): ``beta[e] = -s*ln(rank[e])`` with
  ``rank`` a seeded permutation of 1..E, fp32; zero when ``s == 0``.
"""
from __future__ import annotations

from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

from .configs import MoEConfig

NO_EXPERT = 65535

# tensor ids of the per-tensor streams
TID = dict(
    router_q=0, router_s=1, router_beta=2,
    sgate_q=3, sgate_s=4,
    sh_gu_q=5, sh_gu_s=6, sh_dn_q=7, sh_dn_s=8,
    sh_A_gate=9, sh_B_gate=10, sh_A_up=11, sh_B_up=12, sh_A_down=13, sh_B_down=14,
    ex_gu_q=20, ex_gu_s=21, ex_dn_q=22, ex_dn_s=23, ex_A_down=24, ex_B_down=25,
    ex_A_gate=26, ex_B_gate=27, ex_A_up=28, ex_B_up=29,
    pre_W1=30, pre_b1=31, pre_W2=32, pre_b2=33,
    act=40,
)


def rng(cfg_id: int, layer: int, expert: int, tid: int, seed: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, cfg_id, layer, expert, tid])))


def _words(g: np.random.Generator, n_words: int) -> np.ndarray:
    raw = g.bit_generator.random_raw((n_words + 1) // 2)
    return raw.view(np.uint32)[:n_words]


def _uniform_f16(g: np.random.Generator, shape, lo: float, hi: float) -> np.ndarray:
    return g.uniform(lo, hi, size=shape).astype(np.float16)


def _normal_f16(g: np.random.Generator, shape, std: float) -> np.ndarray:
    return (g.standard_normal(size=shape) * std).astype(np.float16)


def f32_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even) and return the bit patterns."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def int4_matrix(cfg: MoEConfig, layer: int, expert: int, tid_q: int, tid_s: int, out_dim: int, in_dim: int,
                seed: int = 0) -> dict:
    assert in_dim % 64 == 0
    q = _words(rng(cfg.cfg_id, layer, expert, tid_q, seed), out_dim * in_dim // 8).reshape(out_dim, in_dim // 8)
    s = _uniform_f16(rng(cfg.cfg_id, layer, expert, tid_s, seed), (out_dim, in_dim // 64), 0.005, 0.02)
    b = (np.float16(-8.0) * s).astype(np.float16)
    return dict(q=q, s=s, b=b, bits=4)


def int8_matrix(cfg: MoEConfig, layer: int, tid_q: int, tid_s: int, out_dim: int, in_dim: int,
                seed: int = 0) -> dict:
    assert in_dim % 64 == 0
    q = _words(rng(cfg.cfg_id, layer, NO_EXPERT, tid_q, seed), out_dim * in_dim // 4).reshape(out_dim, in_dim // 4)
    s = (_uniform_f16(rng(cfg.cfg_id, layer, NO_EXPERT, tid_s, seed), (out_dim, in_dim // 64), 0.005, 0.02)
         / np.float16(16.0)).astype(np.float16)
    b = (np.float16(-128.0) * s).astype(np.float16)
    return dict(q=q, s=s, b=b, bits=8)


def lora(cfg: MoEConfig, layer: int, expert: int, tid_a: int, tid_b: int, out_dim: int, in_dim: int,
         seed: int = 0) -> dict:
    A = _normal_f16(rng(cfg.cfg_id, layer, expert, tid_a, seed), (cfg.r, in_dim), 0.02)
    B = _normal_f16(rng(cfg.cfg_id, layer, expert, tid_b, seed), (out_dim, cfg.r), 0.02)
    return dict(A=A, B=B, scale=1.0)


def expert(cfg: MoEConfig, layer: int, e: int, seed: int = 0) -> dict:
    """One routed expert: gate/up stacked as ``[2I, H]`` (gate rows first), down ``[H, I]``."""
    d = dict(
        gate_up=int4_matrix(cfg, layer, e, TID["ex_gu_q"], TID["ex_gu_s"], 2 * cfg.I, cfg.H, seed),
        down=int4_matrix(cfg, layer, e, TID["ex_dn_q"], TID["ex_dn_s"], cfg.H, cfg.I, seed),
    )
    if cfg.lora_routed_down:
        d["down_lora"] = lora(cfg, layer, e, TID["ex_A_down"], TID["ex_B_down"], cfg.H, cfg.I, seed)
    if cfg.lora_routed_gate_up:
        d["gate_lora"] = lora(cfg, layer, e, TID["ex_A_gate"], TID["ex_B_gate"], cfg.I, cfg.H, seed)
        d["up_lora"] = lora(cfg, layer, e, TID["ex_A_up"], TID["ex_B_up"], cfg.I, cfg.H, seed)
    return d


def shared(cfg: MoEConfig, layer: int, seed: int = 0) -> dict:
    """Shared expert (gate/up ``[2I_s, H]``, down ``[H, I_s]``), its LoRA and its 8-bit sigmoid gate ``[1, H]``."""
    d = dict(
        gate_up=int4_matrix(cfg, layer, NO_EXPERT, TID["sh_gu_q"], TID["sh_gu_s"], 2 * cfg.I_s, cfg.H, seed),
        down=int4_matrix(cfg, layer, NO_EXPERT, TID["sh_dn_q"], TID["sh_dn_s"], cfg.H, cfg.I_s, seed),
        gate=int8_matrix(cfg, layer, TID["sgate_q"], TID["sgate_s"], 1, cfg.H, seed),
    )
    if cfg.lora_shared:
        d["lora_gate"] = lora(cfg, layer, NO_EXPERT, TID["sh_A_gate"], TID["sh_B_gate"], cfg.I_s, cfg.H, seed)
        d["lora_up"] = lora(cfg, layer, NO_EXPERT, TID["sh_A_up"], TID["sh_B_up"], cfg.I_s, cfg.H, seed)
        d["lora_down"] = lora(cfg, layer, NO_EXPERT, TID["sh_A_down"], TID["sh_B_down"], cfg.H, cfg.I_s, seed)
    return d


def router(cfg: MoEConfig, layer: int, seed: int = 0) -> dict:
    d = int8_matrix(cfg, layer, TID["router_q"], TID["router_s"], cfg.E, cfg.H, seed)
    if cfg.zipf_s > 0:
        rank = rng(cfg.cfg_id, layer, NO_EXPERT, TID["router_beta"], seed).permutation(cfg.E) + 1
        d["beta"] = (-cfg.zipf_s * np.log(rank.astype(np.float64))).astype(np.float32)
    else:
        d["beta"] = np.zeros(cfg.E, dtype=np.float32)
    return d


def prerouter(cfg: MoEConfig, layer: int, seed: int = 0) -> dict:
    """Prerouter head of ``layer``: ``Linear(H+E, P) -> SiLU -> Linear(P, E_next)``."""
    fan1 = cfg.H + cfg.E
    return dict(
        W1=_normal_f16(rng(cfg.cfg_id, layer, NO_EXPERT, TID["pre_W1"], seed), (cfg.P, fan1), 1.0 / np.sqrt(fan1)),
        b1=_normal_f16(rng(cfg.cfg_id, layer, NO_EXPERT, TID["pre_b1"], seed), (cfg.P,), 0.1),
        W2=_normal_f16(rng(cfg.cfg_id, layer, NO_EXPERT, TID["pre_W2"], seed), (cfg.E_next, cfg.P),
                       1.0 / np.sqrt(cfg.P)),
        b2=_normal_f16(rng(cfg.cfg_id, layer, NO_EXPERT, TID["pre_b2"], seed), (cfg.E_next,), 0.1),
    )


def activations(cfg: MoEConfig, step: int = 0, T: int | None = None, seed: int = 0) -> np.ndarray:
    """bf16 bit patterns ``[T, H]`` of N(0,1) activations for one step."""
    T = cfg.T if T is None else T
    g = rng(cfg.cfg_id, NO_EXPERT, step, TID["act"], seed)
    return f32_to_bf16_bits(g.standard_normal(size=(T, cfg.H), dtype=np.float32))


def layer(cfg: MoEConfig, layer_idx: int, experts=None, seed: int = 0, threads: int | None = None) -> dict:
    """All tensors of one layer; ``experts`` limits which routed experts are drawn (default: all)."""
    experts = range(cfg.E) if experts is None else experts
    threads = threads or min(16, os.cpu_count() or 1)
    with ThreadPoolExecutor(threads) as ex:
        ex_list = list(ex.map(lambda e: expert(cfg, layer_idx, e, seed), experts))
    return dict(
        router=router(cfg, layer_idx, seed),
        shared=shared(cfg, layer_idx, seed),
        experts=dict(zip(experts, ex_list)),
        prerouter=prerouter(cfg, layer_idx, seed),
    )
