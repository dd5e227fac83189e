"""CPU checks of the comparison rules the GPU parity tests apply (``tests/parity.py``).

* ``router_tau`` bounds the error of an fp32 evaluation of the logits in the
  router kernel's order (16-element chunks of fp16 activation x code products,
  the split ``s (q - 128)`` / ``(b + 128 s) sum(u)`` dot per chunk, a
  butterfly reduction over the lanes of a row, the bias add), emulated here
  with one float32 rounding per operation -- including activations so small
  that their fp16 copies round.
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
from parity import EPS32, check_bf16_rounding, check_topk, fp16_input_error, qmat_abs_terms, router_tau

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
