"""GPU parity of the tensor-core many-token router and Prerouter first layer against the float64 oracle.

From 256 tokens on, moe_route_topk (E a multiple of 128) and prerouter_predict (P a multiple of 128, E of 64)
multiply on the tensor cores with bf16 operands: the router's codes minus 128 against u with per-group
accumulators, and the Prerouter's W1 split exactly into two bf16 parts against [u ; multi-hot].  Logits and
scores are held to ``router_tau_tc`` / ``prerouter_tau(tc=True)``; indices to the certified near-tie rule.
Token counts cover whole 64-token tiles, a ragged last tile and several tiles per CTA.
"""
import dataclasses

import numpy as np
import pytest
import torch

from gen import CONFIGS, inputs
from oracle import moe_oracle as O
from parity import check_topk, prerouter_tau, router_tau_tc
from test_gpu_layer import Layer, M, dev_bits, prerouter, route, u_vals

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check_route(lay, T, step, K):
    ub = inputs.activations(lay.cfg, step=step, T=T)
    u = u_vals(ub)
    logits, idx, w = route(lay, ub, K)
    ref = O.router_logits(u, lay.host["router"])
    tau = router_tau_tc(u, lay.host["router"])
    err = np.abs(logits - ref)
    assert np.all(err <= tau), float(np.max(err / tau))
    near = check_topk(idx, ref, tau, K)
    assert np.allclose(w, O.gating(ref, idx), atol=1e-6 + 4 * float(tau.max()), rtol=0)
    assert np.allclose(w.sum(1), 1.0, atol=1e-6)
    return near, float(np.max(err / tau))


@pytest.mark.parametrize("T", [256, 300, 1000])
def test_route_topk_tensor_core_prefill_shape(cuda_ok, T):
    """35B-shaped prefill router (H 2048, E 256, Zipf-offset logits) on the tensor-core path."""
    cfg = CONFIGS[3]
    lay = Layer(cfg, 0, experts=[])
    near, _ = _check_route(lay, T, 11 + T, cfg.K)
    assert near <= max(2, T // 20)


@pytest.mark.parametrize("H,E,K", [(256, 128, 2), (4096, 256, 8), (2048, 128, 8)])
def test_route_topk_tensor_core_shapes(cuda_ok, H, E, K):
    """Smallest and largest H (4 and 64 groups), E of one and two 128-row tiles, K up to 8."""
    cfg = dataclasses.replace(CONFIGS[0], H=H, E=E, K=K, I=128, I_s=128)
    lay = Layer(cfg, 0, experts=[])
    _check_route(lay, 333, 5 + H, K)


def test_route_topk_paths_agree_at_the_switch(cuda_ok):
    """255 tokens (CUDA-core GEMV) and the same tokens plus one (tensor cores) give logits within the sum of the
    two paths' bounds of each other, and the same indices outside certified near-ties."""
    cfg = CONFIGS[3]
    lay = Layer(cfg, 0, experts=[])
    ub = inputs.activations(cfg, step=77, T=256)
    u = u_vals(ub)
    lg_small, idx_small, _ = route(lay, ub[:255], cfg.K)
    lg_big, idx_big, _ = route(lay, ub, cfg.K)
    ref = O.router_logits(u, lay.host["router"])
    tau = router_tau_tc(u, lay.host["router"])
    from parity import router_tau
    tau_g = router_tau(u[:255], lay.host["router"])
    assert np.all(np.abs(lg_small - lg_big[:255]) <= tau[:255] + tau_g)
    check_topk(idx_small, ref[:255], tau_g, cfg.K)
    check_topk(idx_big, ref, tau, cfg.K)


def _distinct_sel(rng, T, E, K):
    return np.argsort(rng.random((T, E)), axis=1)[:, :K].astype(np.int32)


@pytest.mark.parametrize("cfg_over,T", [({}, 300), ({}, 1000),
                                         (dict(H=256, E=64, K=2, P=128), 257),
                                         (dict(H=4096, E=128, K=8, P=256), 320)])
def test_prerouter_tensor_core(cuda_ok, cfg_over, T):
    """Prerouter on the tensor-core first layer: 35B prefill shape, the smallest H with a multi-hot of one K
    step (E 64, router on the GEMV), and the largest H with K 8."""
    base = CONFIGS[3]
    cfg = dataclasses.replace(base, **cfg_over) if cfg_over else base
    if cfg_over:
        cfg = dataclasses.replace(cfg, I=128, I_s=128)
    lay = Layer(cfg, 1, experts=[])
    ub = inputs.activations(cfg, step=3 + T, T=T)
    u = u_vals(ub)
    sel = _distinct_sel(np.random.default_rng(T), T, cfg.E, cfg.K)
    pred, scores = prerouter(lay, ub, sel, cfg.K)
    head = lay.host["prerouter"]
    ref = O.prerouter_scores(u, sel, head, cfg.E)
    tau = prerouter_tau(u, sel, head, cfg.E, tc=True)
    err = np.abs(scores - ref)
    assert np.all(err <= tau), float(np.max(err / tau))
    check_topk(pred, ref, tau, cfg.K)


def test_prerouter_paths_agree_at_the_switch(cuda_ok):
    """The multi-hot term on the tensor cores equals the GEMV's column sums: 255 vs 256 tokens."""
    cfg = CONFIGS[3]
    lay = Layer(cfg, 2, experts=[])
    ub = inputs.activations(cfg, step=91, T=256)
    u = u_vals(ub)
    sel = _distinct_sel(np.random.default_rng(5), 256, cfg.E, cfg.K)
    p_small, s_small = prerouter(lay, ub[:255], sel[:255], cfg.K)
    p_big, s_big = prerouter(lay, ub, sel, cfg.K)
    head = lay.host["prerouter"]
    tau_t = prerouter_tau(u, sel, head, cfg.E, tc=True)
    tau_g = prerouter_tau(u[:255], sel[:255], head, cfg.E)
    assert np.all(np.abs(s_small - s_big[:255]) <= tau_t[:255] + tau_g)
