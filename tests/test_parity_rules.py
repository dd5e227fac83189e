"""CPU checks of the comparison rules the GPU parity tests apply (``tests/parity.py``).

* ``router_tau`` bounds the error of an fp32 evaluation of the logits in the
  router kernel's order (16-element chunks of fp16 activation x code products,
  the split ``s (q - 128)`` / ``(b + 128 s) sum(u)`` dot per chunk, a
  butterfly reduction over the lanes of a row, the bias add), emulated here
  with one float32 rounding per operation -- including activations so small
  that their fp16 copies round.
* ``router_tau_tc`` bounds the tensor-core router's error under a pessimistic
  model of the MMA (each 16-product block added to the accumulator with every
  addend truncated at the largest one's last place, the result truncated to
  fp32), followed by the kernel's fp32 group sums and fused multiply-adds.
* ``check_topk`` accepts the exact top-K and certified near-ties and refuses
  wrong sets, duplicates, out-of-range indices and wrong order.
* ``check_bf16_rounding`` accepts round-to-nearest-even and, only next to a
  rounding midpoint, the other neighbour.
"""
import dataclasses

import numpy as np
import pytest

from gen import CONFIGS, inputs
from oracle import moe_oracle as O
from parity import (EPS32, check_bf16_rounding, check_topk, fp16_input_error, qmat_abs_terms, router_tau,
                    router_tau_tc)

f32 = np.float32


def emulate_router_fp32(u: np.ndarray, router: dict) -> np.ndarray:
    """Router logits [T, E] evaluated in float32 in the router kernel's order."""
    T, H = u.shape
    NCH = H // 16
    SEG = min(NCH, 32)
    CPL = NCH // SEG
    qm = O.unpack_codes(router["q"], 8).astype(np.float64) - 128.0  # [E, H], exact small integers
    E = qm.shape[0]
    s = router["s"].astype(np.float32)  # [E, H/64]
    bprime = (router["b"].astype(np.float32) + f32(128.0) * s).astype(np.float32)
    u16 = u.astype(np.float16).astype(np.float64)
    chunks = u.reshape(T, NCH, 16)
    sum16 = np.zeros((T, NCH), np.float32)
    for i in range(16):
        sum16 = (sum16.astype(np.float64) + chunks[:, :, i]).astype(np.float32)
    acc = np.zeros((T, E, SEG), np.float32)
    lanes = np.arange(SEG)
    for c in range(CPL):
        ch = lanes + c * SEG  # chunk of each lane
        g = ch >> 2
        d = np.zeros((T, E, SEG), np.float32)
        for i in range(16):
            k = 16 * ch + i
            prod = u16[:, None, k] * qm[None, :, k]  # exact in float64 (11-bit x 8-bit significands)
            d = (d.astype(np.float64) + prod).astype(np.float32)
        inner = (bprime[None, :, g].astype(np.float64) * sum16[:, None, ch] + acc).astype(np.float32)
        acc = (s[None, :, g].astype(np.float64) * d + inner).astype(np.float32)
    o = SEG // 2
    while o:
        acc = (acc.astype(np.float64) + acc[:, :, lanes ^ o]).astype(np.float32)
        o //= 2
    beta = np.asarray(router["beta"], np.float32)
    return (acc[:, :, 0].astype(np.float64) + beta).astype(np.float32).astype(np.float64)


def _bf16(v):
    return inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(np.asarray(v, np.float32))).astype(np.float64)


@pytest.mark.parametrize("cfg_id,H,zipf", [(0, 256, 0.0), (0, 256, 1.1), (1, 2048, 0.0)])
@pytest.mark.parametrize("scale", [1.0, 3e-6])
def test_router_tau_bounds_an_fp32_evaluation_in_kernel_order(cfg_id, H, zipf, scale):
    cfg = dataclasses.replace(CONFIGS[cfg_id], E=16, H=H, zipf_s=zipf)
    router = inputs.router(cfg, 0)
    rng = np.random.default_rng(int(scale * 1e6) + H)
    u = _bf16(rng.standard_normal((3, H)) * scale)
    exact = O.router_logits(u, router)
    err = np.abs(emulate_router_fp32(u, router) - exact)
    tau = router_tau(u, router)
    assert np.all(err <= tau), float(np.max(err / tau))
    if scale < 1e-5:  # below 2^-17 the fp16 copies of u round: the rounding-count term alone is not a bound
        assert np.any(fp16_input_error(u) > 0)
        beta = np.abs(np.asarray(router["beta"], np.float64))
        rounding_only = 64 * EPS32 * (np.abs(u) @ qmat_abs_terms(router).T) + 4 * EPS32 * beta
        assert np.any(err > rounding_only)
    else:
        assert np.all(fp16_input_error(u) == 0)


def _f32_toward_zero(x):
    m, e = np.frexp(np.asarray(x, np.float64))
    return np.ldexp(np.trunc(m * 2.0 ** 24) / 2.0 ** 24, e)


def _truncating_block(acc, prods):
    """acc + sum(prods) with every addend truncated at the last place of the largest, then to fp32."""
    add = np.concatenate([acc[..., None], prods], axis=-1)
    mx = np.max(np.abs(add), axis=-1, keepdims=True)
    quantum = np.where(mx > 0, np.ldexp(1.0, (np.frexp(np.where(mx > 0, mx, 1.0))[1] - 1) - 23), 1.0)
    return _f32_toward_zero(np.sum(np.trunc(add / quantum) * quantum, axis=-1))


def emulate_router_tc(u: np.ndarray, router: dict) -> np.ndarray:
    """Tensor-core router logits [T, E]: per group four truncating 16-product blocks of (q - 128) u, the fp32
    group sum of u (four 16-element runs, then pairwise), b + 128 s in fp32, two fp32 fused multiply-adds."""
    T, H = u.shape
    qm = O.unpack_codes(router["q"], 8).astype(np.float64) - 128.0
    E = qm.shape[0]
    s = router["s"].astype(np.float64)
    bprime = (router["b"].astype(np.float32) + f32(128.0) * router["s"].astype(np.float32)).astype(np.float64)
    acc = np.zeros((T, E), np.float64)
    for g in range(H // 64):
        D = np.zeros((T, E))
        for blk in range(4):
            k = slice(64 * g + 16 * blk, 64 * g + 16 * blk + 16)
            D = _truncating_block(D, u[:, None, k] * qm[None, :, k])
        quarters = []
        for qq in range(4):
            run = u[:, 64 * g + 16 * qq: 64 * g + 16 * qq + 16].astype(np.float32)
            acc_q = np.zeros(T, np.float32)
            for i in range(16):
                acc_q = (acc_q + run[:, i]).astype(np.float32)
            quarters.append(acc_q)
        U = ((quarters[0] + quarters[1]).astype(np.float32) + (quarters[2] + quarters[3]).astype(np.float32))
        U = U.astype(np.float32).astype(np.float64)
        acc = (s[None, :, g] * D + acc).astype(np.float32).astype(np.float64)
        acc = (bprime[None, :, g] * U[:, None] + acc).astype(np.float32).astype(np.float64)
    beta = np.asarray(router["beta"], np.float32)
    return (acc + beta).astype(np.float32).astype(np.float64)


@pytest.mark.parametrize("H,zipf", [(256, 0.0), (2048, 1.1)])
@pytest.mark.parametrize("scale", [1.0, 3e-6])
def test_router_tau_tc_bounds_a_truncating_tensor_core_model(H, zipf, scale):
    cfg = dataclasses.replace(CONFIGS[0], E=16, H=H, zipf_s=zipf)
    router = inputs.router(cfg, 0)
    rng = np.random.default_rng(int(scale * 1e6) + H + 7)
    u = _bf16(rng.standard_normal((3, H)) * scale)
    exact = O.router_logits(u, router)
    err = np.abs(emulate_router_tc(u, router) - exact)
    tau = router_tau_tc(u, router)
    assert np.all(err <= tau), float(np.max(err / tau))
    # the model is not trivially exact: truncation leaves a visible error
    assert np.max(err) > 0


# ----------------------------------------------------------------------------- check_topk
REF = np.array([[5.0, 4.0, 3.0 + 1e-7, 3.0, 1.0, 0.0]])


def test_check_topk_accepts_the_exact_answer_and_certified_near_ties():
    assert check_topk([[0, 1, 2]], REF, 1e-9, 3) == 0
    assert check_topk([[0, 1, 3]], REF, 1e-6, 3) == 1  # 3rd/4th gap 1e-7 is inside the margin 2e-6
    assert check_topk([[0, 1, 2]], REF, 1e-6, 3) == 1


@pytest.mark.parametrize("gpu,tau", [([[0, 1, 3]], 1e-9),   # gap 1e-7 above the margin: the set is wrong
                                     ([[0, 1, 4]], 1e-6),   # 1.0 is far below the 3rd value
                                     ([[0, 0, 2]], 1e-9),   # duplicate
                                     ([[0, 1, 6]], 1e-9),   # out of range
                                     ([[1, 0, 2]], 1e-9)])  # wrong order with well-separated values
def test_check_topk_refuses(gpu, tau):
    with pytest.raises(AssertionError):
        check_topk(gpu, REF, tau, 3)


# ----------------------------------------------------------------------------- check_bf16_rounding
def test_check_bf16_rounding_rules():
    ref = np.array([1.1, -3.7, 1.0 + 2.0 ** -8, 2.5e-3])  # the third is a rounding midpoint (ties to 1.0)
    want = O.round_bf16(ref)
    bits = inputs.f32_to_bf16_bits(want.astype(np.float32))
    assert check_bf16_rounding(bits, ref, 1e-6) == 0
    other = bits.copy()
    other[2] += 1  # the neighbour above the midpoint: allowed within the fp32 error
    assert check_bf16_rounding(other, ref, 1e-6) == 1
    bad = bits.copy()
    bad[0] += 1  # 1.1 is far from a midpoint: one bf16 ulp off is an error
    with pytest.raises(AssertionError):
        check_bf16_rounding(bad, ref, 1e-6)
