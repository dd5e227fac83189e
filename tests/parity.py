"""Comparison rules between the CUDA path and the float64 oracle.

* Floating-point outputs: ``max|gpu - ref| <= 2e-3 * max|ref|`` (bf16 activations,
  fp32 accumulation).
* Top-K indices: exact wherever the oracle's gap between the K-th and (K+1)-th
  score exceeds twice a certified bound on the GPU's fp32 score error; inside
  that margin ("certified near-ties") the GPU set must be one the margin admits.
* bf16-rounded values (the RMSNorm glue): exact unless the float64 value lies
  within the fp32 computation's relative error of a rounding midpoint.
"""
from __future__ import annotations

import numpy as np

from gen import inputs
from oracle import moe_oracle as O

EPS32 = 2.0 ** -24
OUT_RTOL = 2e-3


def assert_close_inf(gpu, ref, rtol=OUT_RTOL, what="output"):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = max(float(np.max(np.abs(ref))), 1e-30)
    err = float(np.max(np.abs(gpu - ref))) if ref.size else 0.0
    assert err <= rtol * scale, f"{what}: max|err| {err:.3e} > {rtol:g} * {scale:.3e}"
    return err / scale


def qmat_abs_terms(m: dict) -> np.ndarray:
    """Per-element magnitudes |s (q - mid)| + |b + mid*s| of the GPU's split dequantisation."""
    mid = 8 if m["bits"] == 4 else 128
    q = O.unpack_codes(m["q"], m["bits"]).astype(np.float64)
    s = np.repeat(m["s"].astype(np.float64), 64, 1)
    b = np.repeat(m["b"].astype(np.float64), 64, 1)
    return np.abs(q - mid) * s + np.abs(b + mid * s)


def fp16_input_error(u: np.ndarray) -> np.ndarray:
    """|u - fp16(u)|: the GEMV kernels multiply weights by the activations rounded to fp16.

    bf16 values convert to fp16 exactly down to 2^-17 in magnitude; below that
    (fp16 subnormals) the conversion rounds, which this term accounts for.
    """
    u = np.asarray(u, np.float64)
    return np.abs(u - u.astype(np.float16).astype(np.float64))


def router_tau(u: np.ndarray, router: dict, n_round: int = 64) -> np.ndarray:
    """Bound [T, E] on |fp32 GPU logit - exact logit| for inputs u (bf16 values).

    ``n_round`` fp32 roundings on the path of any product term (the router
    kernel takes at most 38 at H = 4096: 16 within a 16-element chunk, 2 per
    chunk of a lane, a 5-level lane reduction, the bias add), plus the exact
    effect of rounding u to fp16 in the ``s (q - mid)`` part of the split dot.
    """
    beta = np.abs(np.asarray(router["beta"], np.float64))
    mid = 8 if router["bits"] == 4 else 128
    q = O.unpack_codes(router["q"], router["bits"]).astype(np.float64)
    s = np.repeat(router["s"].astype(np.float64), 64, 1)
    return (n_round * EPS32 * (np.abs(u) @ qmat_abs_terms(router).T) + 4 * EPS32 * beta
            + fp16_input_error(u) @ (np.abs(q - mid) * s).T)


def tc_chain_rounds(blocks: int) -> int:
    """fp32 rounding units charged to a chain of ``blocks`` tensor-core MMA blocks.

    One tcgen05 kind::f16 block adds 16 exact products to the fp32 accumulator.
    The bound assumes nothing finer than this: every one of the 17 addends is
    aligned to the largest and truncated to within one unit in the last place
    (2 EPS32 of the largest magnitude, hence of the sum of magnitudes).
    """
    return 34 * blocks


def router_tau_tc(u: np.ndarray, router: dict) -> np.ndarray:
    """Bound [T, E] on |GPU logit - exact logit| for the tensor-core router (many-token path).

    Per group: the four 16-wide MMA blocks of sum_k (q-128) u (exact products),
    the group sum of u (16-term sums, two pairwise adds) and b + 128 s (one
    rounding); then two fused multiply-adds per group into the fp32 logit and
    the bias add.  u enters unrounded (bf16 operands).
    """
    G = u.shape[1] // 64
    beta = np.abs(np.asarray(router["beta"], np.float64))
    n = tc_chain_rounds(4) + 2 * G + 4
    return n * EPS32 * (np.abs(u) @ qmat_abs_terms(router).T) + 4 * EPS32 * beta


def prerouter_tau(u, sel, head, E, n_round=128, tc=False):
    """Bound [T, E_next] on |fp32 GPU scores - exact| (first order through SiLU, |silu'| <= 1.1).

    ``tc``: the first layer ran on the tensor cores: W1 split exactly into two
    bf16 parts, u unrounded, four accumulation chains of 2 (H + E) / 64 MMA
    blocks each, then three chain adds and the bias add.  Otherwise the GEMV:
    ``n_round`` roundings per product term and u rounded to fp16.  The second
    layer takes at most 33 + ceil(P / 32) roundings per product (32-term chunk
    sums added up, then the bias) on the many-token path and 8 ceil(P / 256) + 6
    in the decode kernels; ``n_round`` must cover both.
    """
    P = head["W2"].shape[1]
    assert n_round >= max(33 + -(-P // 32), 8 * -(-P // 256) + 6)
    W1 = np.abs(head["W1"].astype(np.float64))
    W2 = np.abs(head["W2"].astype(np.float64))
    xin = np.concatenate([np.abs(u), O.multi_hot(sel, E)], axis=1)
    if tc:
        n1 = tc_chain_rounds(2 * (u.shape[1] + E) // 64) + 8
        a_err = n1 * EPS32 * (xin @ W1.T + np.abs(head["b1"].astype(np.float64)))
    else:
        a_err = n_round * EPS32 * (xin @ W1.T + np.abs(head["b1"].astype(np.float64)))
        a_err = a_err + fp16_input_error(u) @ W1[:, :u.shape[1]].T  # u enters W1 rounded to fp16
    z = np.abs(O.silu(np.concatenate([u, O.multi_hot(sel, E)], 1) @ head["W1"].astype(np.float64).T
                      + head["b1"].astype(np.float64)))
    return (1.1 * a_err + 8 * EPS32 * z) @ W2.T + n_round * EPS32 * (z @ W2.T + np.abs(head["b2"].astype(np.float64)))


def check_topk(gpu_idx, ref, tau_row, K: int, exact_order: bool = True) -> int:
    """Check GPU top-K indices against float64 scores ``ref`` [T, E]; returns #certified near-tie rows."""
    gpu_idx = np.asarray(gpu_idx)
    T, E = ref.shape
    near = 0
    for t in range(T):
        m = 2.0 * float(np.max(tau_row[t]) if np.ndim(tau_row) else tau_row)
        order = np.lexsort((np.arange(E), -ref[t]))
        kth = ref[t, order[K - 1]]
        nxt = ref[t, order[K]] if K < E else -np.inf
        g = [int(i) for i in gpu_idx[t]]
        assert len(set(g)) == K and all(0 <= i < E for i in g), (t, g)
        if kth - nxt > m:
            assert set(g) == set(order[:K].tolist()), (t, g, order[:K])
        else:
            near += 1
            chosen = np.zeros(E, bool)
            chosen[g] = True
            assert np.all(ref[t, chosen] >= kth - m) and np.all(ref[t, ~chosen] <= kth + m), (t, g)
        vals = ref[t, g]
        assert np.all(vals[:-1] >= vals[1:] - m), (t, g, vals)
        if exact_order:
            gaps = np.diff(np.sort(ref[t, order[:K + (1 if K < E else 0)]]))
            if np.all(np.abs(gaps) > m):
                assert g == order[:K].tolist(), (t, g, order[:K])
    return near


def check_bf16_rounding(gpu_bits, ref64, rel_err: float):
    """GPU bf16 values equal round_bf16(ref) except where ref is within rel_err of a rounding midpoint."""
    gpu = inputs.bf16_bits_to_f32(np.asarray(gpu_bits).view(np.uint16)).astype(np.float64)
    want = O.round_bf16(ref64)
    lo = O.round_bf16(ref64 * (1 - rel_err))
    hi = O.round_bf16(ref64 * (1 + rel_err))
    ok = (gpu == want) | ((lo != hi) & ((gpu == lo) | (gpu == hi)))
    assert np.all(ok), f"{int((~ok).sum())} bf16 values off the certified rounding"
    return int((gpu != want).sum())
