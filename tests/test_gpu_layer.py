"""GPU parity of the per-layer entry points against the float64 oracle.

Every case feeds the same seeded inputs to both sides; expert-forward cases
give both the same routing so that routing and expert math are checked
separately; routing is checked with the certified near-tie rule.
"""
import dataclasses

import numpy as np
import pytest
import torch

from gen import CONFIGS, inputs
from oracle import moe_oracle as O
from parity import (EPS32, assert_close_inf, check_bf16_rounding, check_topk, prerouter_tau, router_tau,
                    router_tau_tc)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def M():
    import int4_expert_ffn_top_b200 as mod
    return mod


def dev_bits(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV)


def u_vals(bits: np.ndarray) -> np.ndarray:
    return inputs.bf16_bits_to_f32(bits).astype(np.float64)


class Layer:
    def __init__(self, cfg, l=0, experts=None):
        self.cfg = cfg
        self.host = inputs.layer(cfg, l, experts)
        self.dev = M().DeviceLayer(cfg, self.host)
        self.head = M().DeviceHead(cfg, self.host["prerouter"])


def route(layer: Layer, u_bits: np.ndarray, K: int):
    T, E = u_bits.shape[0], layer.cfg.E
    logits = torch.full((T, E), float("nan"), device=DEV)
    idx = torch.full((T, K), -1, dtype=torch.int32, device=DEV)
    w = torch.full((T, K), float("nan"), device=DEV)
    M().moe_route_topk(layer.dev, dev_bits(u_bits), K, logits, idx, w)
    torch.cuda.synchronize()
    return logits.cpu().numpy().astype(np.float64), idx.cpu().numpy(), w.cpu().numpy().astype(np.float64)


def expert_forward(layer: Layer, u_bits, K, idx, w, mode=0, x0=None, perm=False, offset=0):
    """offset > 0 places out that many elements into a larger buffer (an output not 16-byte aligned)."""
    m = M()
    T, H = u_bits.shape[0], layer.cfg.H
    if mode == 1:
        out = torch.zeros(T * H + offset, dtype=torch.int16, device=DEV)[offset:].view(T, H)
    elif mode == 2:
        out = torch.empty(T * H + offset, device=DEV)[offset:].view(T, H)
        out.copy_(torch.from_numpy(x0.astype(np.float32)))
    else:
        out = torch.full((T * H + offset,), float("nan"), device=DEV)[offset:].view(T, H)
    ws = m.workspace(m.moe_workspace_size(layer.dev, T, K))
    ws.fill_(0xA5)  # contents on entry must not matter
    perm_out = torch.full((T * K,), -1, dtype=torch.int32, device=DEV) if perm else None
    m.moe_expert_forward(layer.dev, dev_bits(u_bits), K, torch.from_numpy(idx.astype(np.int32)).to(DEV),
                         torch.from_numpy(w.astype(np.float32)).to(DEV), out, mode, ws, perm_out=perm_out)
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    if mode == 1:
        o = inputs.bf16_bits_to_f32(o.view(np.uint16))
    return (o.astype(np.float64), perm_out.cpu().numpy() if perm else None)


def oracle_out(layer: Layer, u, idx, w):
    L = layer.host
    y = O.routed_outputs(u, L["experts"], idx)
    return O.combine(w, y, O.shared_gate(u, L["shared"]), O.shared_expert(u, L["shared"]))


def prerouter(layer: Layer, u_bits, sel, K_next):
    m = M()
    T = u_bits.shape[0]
    pred = torch.full((T, K_next), -1, dtype=torch.int32, device=DEV)
    scores = torch.full((T, layer.cfg.E_next), float("nan"), device=DEV)
    ws = m.workspace(m.prerouter_workspace_size(layer.head, T))
    m.prerouter_predict(layer.head, dev_bits(u_bits), torch.from_numpy(sel.astype(np.int32)).to(DEV), K_next, pred,
                        scores, ws)
    torch.cuda.synchronize()
    return pred.cpu().numpy(), scores.cpu().numpy().astype(np.float64)


@pytest.fixture(scope="module")
def c0(cuda_ok):
    return Layer(CONFIGS[0])


# ----------------------------------------------------------------------------- glue
@pytest.mark.parametrize("T,H", [(1, 256), (5, 2048), (3, 4096)])
def test_rmsnorm_bf16_certified_rounding(cuda_ok, T, H):
    m = M()
    rng = np.random.default_rng(T * H)
    x = (rng.standard_normal((T, H)) * rng.uniform(0.1, 50.0, size=(T, 1))).astype(np.float32)
    u = torch.zeros((T, H), dtype=torch.int16, device=DEV)
    m.moe_rmsnorm_bf16(torch.from_numpy(x).to(DEV), 1e-6, u)
    torch.cuda.synchronize()
    ref = O.rmsnorm(x.astype(np.float64), 1e-6)
    check_bf16_rounding(u.cpu().numpy(), ref, rel_err=(H / 256 + 24) * EPS32)


# ----------------------------------------------------------------------------- routing
@pytest.mark.parametrize("T", [1, 4, 13])
def test_route_topk_c0(c0, T):
    cfg = c0.cfg
    ub = inputs.activations(cfg, step=T, T=T)
    u = u_vals(ub)
    logits, idx, w = route(c0, ub, cfg.K)
    ref = O.router_logits(u, c0.host["router"])
    tau = router_tau(u, c0.host["router"])
    assert np.all(np.abs(logits - ref) <= tau), float(np.max(np.abs(logits - ref) / tau))
    check_topk(idx, ref, tau, cfg.K)
    assert np.allclose(w, O.gating(ref, idx), atol=1e-6 + 4 * float(tau.max()), rtol=0)
    assert np.allclose(w.sum(1), 1.0, atol=1e-6)


@pytest.mark.parametrize("K", [1, 8])
def test_route_topk_extreme_k(c0, K):
    ub = inputs.activations(c0.cfg, step=100 + K, T=6)
    u = u_vals(ub)
    logits, idx, w = route(c0, ub, K)
    ref = O.router_logits(u, c0.host["router"])
    check_topk(idx, ref, router_tau(u, c0.host["router"]), K)
    if K == 1:
        assert np.all(w == 1.0)


def test_route_topk_prefill_router_with_zipf_offsets(cuda_ok):
    cfg = CONFIGS[3]
    lay = Layer(cfg, 0, experts=[])
    ub = inputs.activations(cfg, step=0, T=200)
    u = u_vals(ub)
    logits, idx, w = route(lay, ub, cfg.K)
    ref = O.router_logits(u, lay.host["router"])
    tau = router_tau(u, lay.host["router"])
    assert np.all(np.abs(logits - ref) <= tau)
    near = check_topk(idx, ref, tau, cfg.K)
    assert near <= 10
    # the offsets skew the load: the most popular expert gets far more than the mean share
    counts = np.bincount(idx.reshape(-1), minlength=cfg.E)
    assert counts.max() > 8 * idx.size / cfg.E


# ----------------------------------------------------------------------------- experts + combine
@pytest.mark.parametrize("T", [1, 4, 13])
@pytest.mark.parametrize("mode", [0, 1, 2])
def test_expert_forward_c0(c0, T, mode):
    cfg = c0.cfg
    ub = inputs.activations(cfg, step=7 + T, T=T)
    u = u_vals(ub)
    ref_logits = O.router_logits(u, c0.host["router"])
    idx = O.topk(ref_logits, cfg.K)
    w = O.gating(ref_logits, idx)
    x0 = np.random.default_rng(T).standard_normal((T, cfg.H)) * 4 if mode == 2 else None
    out, _ = expert_forward(c0, ub, cfg.K, idx, w, mode=mode, x0=x0)
    ref = oracle_out(c0, u, idx, w)
    if mode == 2:
        out = out - x0.astype(np.float32)
    if mode == 1:
        half_ulp = np.abs(O.round_bf16(ref) - ref)
        assert np.all(np.abs(out - ref) <= 2e-3 * np.abs(ref).max() + half_ulp + 1e-30)
    else:
        assert_close_inf(out, ref)


@pytest.mark.parametrize("offset", [0, 1])
@pytest.mark.parametrize("mode", [0, 1, 2])
def test_expert_forward_gemm_output_modes(c0, mode, offset):
    """The three output modes on the grouped-GEMM path (80 slots), with out aligned and not 16-byte aligned."""
    cfg = c0.cfg
    T = 40
    ub = inputs.activations(cfg, step=90 + mode, T=T)
    u = u_vals(ub)
    ref_logits = O.router_logits(u, c0.host["router"])
    idx = O.topk(ref_logits, cfg.K)
    w = O.gating(ref_logits, idx)
    x0 = np.random.default_rng(mode).standard_normal((T, cfg.H)) * 4 if mode == 2 else None
    out, _ = expert_forward(c0, ub, cfg.K, idx, w, mode=mode, x0=x0, offset=offset)
    ref = oracle_out(c0, u, idx, w)
    if mode == 2:
        out = out - x0.astype(np.float32)
    if mode == 1:
        half_ulp = np.abs(O.round_bf16(ref) - ref)
        assert np.all(np.abs(out - ref) <= 2e-3 * np.abs(ref).max() + half_ulp + 1e-30)
    else:
        assert_close_inf(out, ref)


def test_expert_forward_duplicate_and_skewed_routing(c0):
    cfg = c0.cfg
    T = 11
    ub = inputs.activations(cfg, step=3, T=T)
    u = u_vals(ub)
    idx = np.tile(np.array([[3, 5]]), (T, 1))
    idx[2] = [7, 7]          # the same expert twice in one token
    idx[9] = [15, 0]         # first and last experts
    w = np.random.default_rng(0).dirichlet([1, 1], size=T)
    out, perm = expert_forward(c0, ub, cfg.K, idx, w, perm=True)
    assert_close_inf(out, oracle_out(c0, u, idx, w))
    assert np.array_equal(perm, O.buckets(idx, cfg.E)["perm"])


@pytest.mark.parametrize("T,K", [(13, 2), (64, 8), (1, 1)])
def test_bucket_permutation_bit_exact(c0, T, K):
    cfg = c0.cfg
    rng = np.random.default_rng(T * 10 + K)
    idx = np.stack([rng.choice(cfg.E, size=K, replace=False) for _ in range(T)])
    ub = inputs.activations(cfg, step=50, T=T)
    w = rng.dirichlet(np.ones(K), size=T)
    out, perm = expert_forward(c0, ub, K, idx, w, perm=True)
    assert np.array_equal(perm, O.buckets(idx, cfg.E)["perm"])
    assert_close_inf(out, oracle_out(c0, u_vals(ub), idx, w))


def test_zero_tokens_is_a_no_op(c0):
    m = M()
    out = torch.full((1, c0.cfg.H), 7.0, device=DEV)
    ws = m.workspace(256)
    empty = torch.zeros((0, c0.cfg.H), dtype=torch.int16, device=DEV)
    m.moe_expert_forward(c0.dev, empty, 2, torch.zeros((0, 2), dtype=torch.int32, device=DEV),
                         torch.zeros((0, 2), device=DEV), out, 0, ws)
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


def test_workspace_too_small_is_rejected(c0):
    m = M()
    ub = dev_bits(inputs.activations(c0.cfg, T=4))
    need = m.moe_workspace_size(c0.dev, 4, 2)
    with pytest.raises(m.MoEError) as e:
        m.moe_expert_forward(c0.dev, ub, 2, torch.zeros((4, 2), dtype=torch.int32, device=DEV),
                             torch.zeros((4, 2), device=DEV), torch.zeros((4, c0.cfg.H), device=DEV), 0,
                             m.workspace(need - 256))
    assert e.value.code == 3


# ----------------------------------------------------------------------------- Prerouter
@pytest.mark.parametrize("T", [1, 4, 13])
def test_prerouter_c0(c0, T):
    cfg = c0.cfg
    ub = inputs.activations(cfg, step=20 + T, T=T)
    u = u_vals(ub)
    sel = O.topk(O.router_logits(u, c0.host["router"]), cfg.K)
    pred, scores = prerouter(c0, ub, sel, cfg.K)
    ref = O.prerouter_scores(u, sel, c0.host["prerouter"], cfg.E)
    tau = prerouter_tau(u, sel, c0.host["prerouter"], cfg.E)
    assert np.all(np.abs(scores - ref) <= tau), float(np.max(np.abs(scores - ref) / tau))
    check_topk(pred, ref, tau, cfg.K)


# ----------------------------------------------------------------------------- full-size layers
@pytest.mark.parametrize("cfg_id,l,T", [(1, 0, 1), (1, 39, 1), (2, 5, 1), (1, 3, 3)])
def test_full_size_layer(cuda_ok, cfg_id, l, T):
    cfg = CONFIGS[cfg_id]
    lay = Layer(cfg, l)
    ub = inputs.activations(cfg, step=1000 + l, T=T)
    u = u_vals(ub)
    logits, idx, w = route(lay, ub, cfg.K)
    ref_logits = O.router_logits(u, lay.host["router"])
    tau = router_tau(u, lay.host["router"])
    assert np.all(np.abs(logits - ref_logits) <= tau)
    check_topk(idx, ref_logits, tau, cfg.K)
    out, _ = expert_forward(lay, ub, cfg.K, idx, w.astype(np.float64))
    assert_close_inf(out, oracle_out(lay, u, idx, w))
    pred, scores = prerouter(lay, ub, idx, cfg.K)
    ref_p = O.prerouter_scores(u, idx, lay.host["prerouter"], cfg.E)
    tau_p = prerouter_tau(u, idx, lay.host["prerouter"], cfg.E)
    assert np.all(np.abs(scores - ref_p) <= tau_p)
    check_topk(pred, ref_p, tau_p, cfg.K)


# ----------------------------------------------------------------------------- stacks
def _check_stack(cfg, stack_layers, T, res, x0, sample, tc=False):
    """Teacher-forced per-layer parity on the sampled layers of a stack run (``tc``: the run's router and
    Prerouter first layer took the tensor-core many-token path)."""
    xs = res["x_trace"]
    for l in sample:
        L = stack_layers(l)
        ub = res["u_trace"][l]
        u = u_vals(ub)
        if l == 0:
            check_bf16_rounding(ub, O.rmsnorm(x0.astype(np.float64), 1e-6), rel_err=(cfg.H / 256 + 24) * EPS32)
        ref_logits = O.router_logits(u, L["router"])
        tau = router_tau_tc(u, L["router"]) if tc else router_tau(u, L["router"])
        check_topk(res["true_idx"][l], ref_logits, tau, cfg.K)
        executed = res["idx"][l]
        if cfg.predicted_routing and l > 0:
            assert np.array_equal(executed, res["pred"][l - 1])
        else:
            assert np.array_equal(executed, res["true_idx"][l])
        w = O.gating(ref_logits, executed)
        y = O.routed_outputs(u, L["experts"], executed)
        ref_out = O.combine(w, y, O.shared_gate(u, L["shared"]), O.shared_expert(u, L["shared"]))
        x_next = xs[l + 1] if l + 1 < len(xs) else res["x"]
        assert_close_inf(x_next.astype(np.float64) - xs[l].astype(np.float64), ref_out, what=f"layer {l} output")
        ref_p = O.prerouter_scores(u, executed, L["prerouter"], cfg.E)
        check_topk(res["pred"][l], ref_p, prerouter_tau(u, executed, L["prerouter"], cfg.E, tc=tc), cfg.K)


def run_stack(stack, cfg, T, x0, predicted, opts=None):
    m = M()
    n = stack.n
    x = torch.from_numpy(x0.astype(np.float32)).to(DEV)
    err = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    tr = dict(x_trace=torch.zeros((n, T, cfg.H), device=DEV),
              u_trace=torch.zeros((n, T, cfg.H), dtype=torch.int16, device=DEV),
              idx_all=torch.full((n, T, cfg.K), -1, dtype=torch.int32, device=DEV),
              true_idx_all=torch.full((n, T, cfg.K), -1, dtype=torch.int32, device=DEV),
              pred_all=torch.full((n, T, cfg.K), -1, dtype=torch.int32, device=DEV))
    st = m.StackStructs(stack)
    ws = m.workspace(m.moe_stack_workspace_size(st, T, cfg.K, cfg.K))
    m.moe_stack_decode(st, x, cfg.K, cfg.K, 1e-6, ws, use_predicted_routing=predicted, err_word=err, opts=opts, **tr)
    torch.cuda.synchronize()
    return dict(err=int(err.item()), x=x.cpu().numpy(), x_trace=tr["x_trace"].cpu().numpy(),
                u_trace=tr["u_trace"].cpu().numpy().view(np.uint16), idx=tr["idx_all"].cpu().numpy(),
                true_idx=tr["true_idx_all"].cpu().numpy(), pred=tr["pred_all"].cpu().numpy())


@pytest.mark.parametrize("predicted", [False, True])
def test_small_stack(cuda_ok, predicted):
    cfg = dataclasses.replace(CONFIGS[0], layers=4, lora_routed_down=predicted, predicted_routing=predicted)
    layer_fn = lambda l: inputs.layer(cfg, l)  # noqa: E731
    stack = M().DeviceStack(cfg, layer_fn)
    T = 5
    x0 = inputs.bf16_bits_to_f32(inputs.activations(cfg, step=9, T=T)) * 3.0
    res = run_stack(stack, cfg, T, x0, predicted)
    _check_stack(cfg, layer_fn, T, res, x0, range(cfg.layers))


SMALL_SINGLE = [dict(H=1024, E=32, K=4, P=128), dict(H=1024, E=64, K=8, P=64), dict(H=2048, E=16, K=2, P=256)]


@pytest.mark.parametrize("shape", SMALL_SINGLE)
def test_single_launch_stack(cuda_ok, shape):
    """The one-launch stack kernel on small stacks, against the oracle and the per-layer path."""
    m = M()
    cfg = dataclasses.replace(CONFIGS[1], layers=5, I=512, I_s=512, r=16, **shape)
    layer_fn = lambda l: inputs.layer(cfg, l)  # noqa: E731
    stack = m.DeviceStack(cfg, layer_fn)
    x0 = inputs.bf16_bits_to_f32(inputs.activations(cfg, step=11, T=1))
    res = run_stack(stack, cfg, 1, x0, False, opts=m.stack_opts(path=m.PATH_SINGLE))
    assert res["err"] == 0
    _check_stack(cfg, layer_fn, 1, res, x0, range(cfg.layers))
    ref = run_stack(stack, cfg, 1, x0, False, opts=m.stack_opts(path=m.PATH_LAYERS))
    assert ref["err"] == 0
    # both paths agree wherever routing agrees (it does unless a certified near-tie flips)
    if all(np.array_equal(a, b) for a, b in zip(res["idx"], ref["idx"])):
        assert_close_inf(res["x"], ref["x"], what="single launch vs per-layer launches")


def test_single_launch_bounded_wait_reports_timeout(cuda_ok):
    """A residual publication that never arrives: the waits give up and the status says so."""
    m = M()
    cfg = dataclasses.replace(CONFIGS[1], layers=3, H=1024, E=32, K=4, P=128)
    stack = m.DeviceStack(cfg, lambda l: inputs.layer(cfg, l))
    x0 = inputs.bf16_bits_to_f32(inputs.activations(cfg, step=12, T=1))
    res = run_stack(stack, cfg, 1, x0, False,
                    opts=m.stack_opts(path=m.PATH_SINGLE, timeout_ns=20_000_000, drop_layer=1, drop_cta=3))
    assert res["err"] == 5
    # the context stays usable: the next call succeeds
    res2 = run_stack(stack, cfg, 1, x0, False, opts=m.stack_opts(path=m.PATH_SINGLE))
    assert res2["err"] == 0 and np.all(np.isfinite(res2["x"]))


def test_single_launch_rejects_ineligible_shapes(cuda_ok, c0):
    m = M()
    st = m.StackStructs([c0.dev], [c0.head])
    ws = m.workspace(m.moe_stack_workspace_size(st, 1, 2, 2))
    x = torch.zeros((1, c0.cfg.H), device=DEV)
    with pytest.raises(m.MoEError) as e:
        m.moe_stack_decode(st, x, 2, 2, 1e-6, ws, opts=m.stack_opts(path=m.PATH_SINGLE))
    assert e.value.code == 2


@pytest.mark.slow
@pytest.mark.parametrize("cfg_id", [1, 2])
def test_full_size_stack_sampled_layers(cuda_ok, cfg_id):
    """The whole 35B-/8B-shaped stack at batch 1, checked on sampled layers."""
    cfg = CONFIGS[cfg_id]
    stack = M().DeviceStack(cfg, lambda l: inputs.layer(cfg, l))
    T = 1
    x0 = inputs.bf16_bits_to_f32(inputs.activations(cfg, step=77, T=T))
    res = run_stack(stack, cfg, T, x0, False)
    assert res["err"] == 0
    del stack
    torch.cuda.empty_cache()
    sample = [0, 1, cfg.layers // 2, cfg.layers - 1]
    needed = {l: sorted(set(res["idx"][l].reshape(-1).tolist())) for l in sample}
    _check_stack(cfg, lambda l: inputs.layer(cfg, l, experts=needed[l]), T, res, x0, sample)


@pytest.mark.slow
def test_batched_decode_stack_with_predicted_routing(cuda_ok):
    """35B-shaped stack at 64 tokens per step: layers >= 1 execute the previous head's prediction, every
    routed expert carries a down-projection LoRA; the experts take the grouped-GEMM path (64*4 slots)."""
    cfg = CONFIGS[4]
    stack = M().DeviceStack(cfg, lambda l: inputs.layer(cfg, l))
    T = cfg.T
    x0 = inputs.bf16_bits_to_f32(inputs.activations(cfg, step=123, T=T))
    res = run_stack(stack, cfg, T, x0, True)
    assert res["err"] == 0
    del stack
    torch.cuda.empty_cache()
    sample = [0, 1, cfg.layers // 2, cfg.layers - 1]
    needed = {l: sorted(set(res["idx"][l].reshape(-1).tolist())) for l in sample}
    _check_stack(cfg, lambda l: inputs.layer(cfg, l, experts=needed[l]), T, res, x0, sample)


@pytest.mark.slow
def test_prefill_stack_full_size_sampled(cuda_ok):
    """35B-shaped prefill exactly as the benchmark runs it: 3,328 tokens through all 40 layers (per-layer
    launches, grouped-GEMM experts), checked on sampled layers for every 52nd token."""
    cfg = CONFIGS[3]
    stack = M().DeviceStack(cfg, lambda l: inputs.layer(cfg, l))
    T = cfg.T
    x0 = inputs.bf16_bits_to_f32(inputs.activations(cfg, step=1, T=T))
    res = run_stack(stack, cfg, T, x0, False, opts=M().stack_opts(path=M().PATH_LAYERS))
    assert res["err"] == 0
    del stack
    torch.cuda.empty_cache()
    toks = np.arange(0, T, 52)
    sub = {k: (v[:, toks] if k in ("x_trace", "u_trace", "idx", "true_idx", "pred") else v[toks]) for k, v in res.items()
           if k != "err"}
    sample = [0, 1, cfg.layers // 2, cfg.layers - 1]
    needed = {l: sorted(set(sub["idx"][l].reshape(-1).tolist())) for l in sample}
    _check_stack(cfg, lambda l: inputs.layer(cfg, l, experts=needed[l]), len(toks), sub, x0[toks], sample, tc=True)


# Largest supported shapes (H 4096, I 2048) on both expert paths: 4 tokens (GEMV), 64 tokens (grouped GEMM).
@pytest.mark.parametrize("T", [4, 64])
def test_expert_forward_max_shapes(cuda_ok, T):
    cfg = dataclasses.replace(CONFIGS[0], H=4096, I=2048, I_s=2048, r=32, lora_routed_down=True)
    lay = Layer(cfg, 0)
    ub = inputs.activations(cfg, step=31 + T, T=T)
    u = u_vals(ub)
    logits = O.router_logits(u, lay.host["router"])
    idx = O.topk(logits, cfg.K)
    w = O.gating(logits, idx)
    out, perm = expert_forward(lay, ub, cfg.K, idx, w, perm=True)
    assert np.array_equal(perm, O.buckets(idx, cfg.E)["perm"])
    assert_close_inf(out, oracle_out(lay, u, idx, w))


# ----------------------------------------------------------------------------- many-token (tensor-core) path
@pytest.mark.parametrize("T", [64, 200])
@pytest.mark.parametrize("routed_lora", [False, True])
def test_expert_forward_grouped_gemm_small(cuda_ok, T, routed_lora):
    """T*K >= 48 slots take the tcgen05 grouped-GEMM path; same definition as the decode path."""
    _grouped_gemm_case(dataclasses.replace(CONFIGS[0], lora_routed_down=routed_lora), T)


@pytest.mark.parametrize("T", [23, 24])  # 46 slots (GEMVs) and 48 slots (grouped GEMMs) at top-2
def test_expert_forward_at_the_path_switch(cuda_ok, T):
    """Both sides of the GEMV / grouped-GEMM switch give the oracle's output, bucket permutation included."""
    _grouped_gemm_case(dataclasses.replace(CONFIGS[0], lora_routed_down=True), T)


# (H, I): gate/up and down with different m-tile counts; K/64 above the pipeline depth of 4
@pytest.mark.parametrize("H,I", [(256, 256), (512, 128), (1024, 512)])
def test_expert_forward_grouped_gemm_shapes(cuda_ok, H, I):
    _grouped_gemm_case(dataclasses.replace(CONFIGS[0], H=H, I=I, I_s=I, lora_routed_down=True), 96)


def _grouped_gemm_case(cfg, T):
    lay = Layer(cfg, 0)
    ub = inputs.activations(cfg, step=500 + T, T=T)
    u = u_vals(ub)
    logits = O.router_logits(u, lay.host["router"])
    idx = O.topk(logits, cfg.K)
    w = O.gating(logits, idx)
    out, perm = expert_forward(lay, ub, cfg.K, idx, w, perm=True)
    assert np.array_equal(perm, O.buckets(idx, cfg.E)["perm"])
    assert_close_inf(out, oracle_out(lay, u, idx, w))
    x0 = np.random.default_rng(T).standard_normal((T, cfg.H))
    out2, _ = expert_forward(lay, ub, cfg.K, idx, w, mode=2, x0=x0)
    assert_close_inf(out2 - x0.astype(np.float32), oracle_out(lay, u, idx, w))


def test_expert_forward_grouped_gemm_skewed_buckets(cuda_ok):
    """One expert takes most slots (several 128-token tiles), others one or none."""
    cfg = CONFIGS[0]
    lay = Layer(cfg, 0)
    T = 300
    ub = inputs.activations(cfg, step=77, T=T)
    u = u_vals(ub)
    rng = np.random.default_rng(5)
    idx = np.stack([[3, int(rng.integers(4, 16))] if t % 7 else [int(rng.integers(0, 3)), 3] for t in range(T)])
    w = rng.dirichlet([1, 1], size=T)
    out, perm = expert_forward(lay, ub, cfg.K, idx, w, perm=True)
    assert np.array_equal(perm, O.buckets(idx, cfg.E)["perm"])
    assert_close_inf(out, oracle_out(lay, u, idx, w))


def test_expert_forward_grouped_gemm_full_size_layer(cuda_ok):
    """35B-shaped prefill layer (Zipf-offset router) on 512 tokens, sampled tokens checked."""
    cfg = CONFIGS[3]
    lay = Layer(cfg, 1)
    T = 512
    ub = inputs.activations(cfg, step=9, T=T)
    u = u_vals(ub)
    logits, idx, w = route(lay, ub, cfg.K)
    out, perm = expert_forward(lay, ub, cfg.K, idx, w, perm=True)
    assert np.array_equal(perm, O.buckets(idx, cfg.E)["perm"])
    sample = np.arange(0, T, 37)
    ref = oracle_out(lay, u[sample], idx[sample], w[sample])
    assert_close_inf(out[sample], ref)


# ----------------------------------------------------------------------------- device-side status (error word)
def _status_calls(layer: Layer, ub, K):
    """Run the three per-layer entry points on u with one error word each; returns their statuses."""
    m = M()
    T, cfg = ub.shape[0], layer.cfg
    errs = [torch.zeros((1,), dtype=torch.int32, device=DEV) for _ in range(3)]
    u = dev_bits(ub)
    logits = torch.empty((T, cfg.E), device=DEV)
    idx = torch.empty((T, K), dtype=torch.int32, device=DEV)
    w = torch.empty((T, K), device=DEV)
    m.moe_route_topk(layer.dev, u, K, logits, idx, w, err_word=errs[0])
    sel = torch.from_numpy(np.tile(np.arange(K, dtype=np.int32), (T, 1))).to(DEV)
    wfix = torch.full((T, K), 1.0 / K, device=DEV)
    out = torch.empty((T, cfg.H), device=DEV)
    ws = m.workspace(m.moe_workspace_size(layer.dev, T, K))
    m.moe_expert_forward(layer.dev, u, K, sel, wfix, out, 0, ws, err_word=errs[1])
    pred = torch.empty((T, K), dtype=torch.int32, device=DEV)
    scores = torch.empty((T, cfg.E_next), device=DEV)
    pws = m.workspace(m.prerouter_workspace_size(layer.head, T))
    m.prerouter_predict(layer.head, u, sel, K, pred, scores, pws, err_word=errs[2])
    torch.cuda.synchronize()
    return [int(e.item()) for e in errs], out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("T", [4, 64])  # GEMV path and grouped-GEMM path (64 x 2 slots)
def test_activation_beyond_fp16_range_is_reported(c0, T):
    """An activation fp16 cannot hold (|u| > 65504) sets MOE_ERR_RANGE in every entry point's error word."""
    ub = inputs.activations(c0.cfg, step=41, T=T)
    ok, _ = _status_calls(c0, ub, c0.cfg.K)
    assert ok == [0, 0, 0]
    bad = ub.copy()
    bad[T // 2, 17] = inputs.f32_to_bf16_bits(np.array([7.0e4], np.float32))[0]
    st, _ = _status_calls(c0, bad, c0.cfg.K)
    assert st == [6, 6, 6]


@pytest.mark.parametrize("T", [4, 64])
@pytest.mark.parametrize("scale", [2.0 ** -4, 8.0])
def test_expert_forward_parity_across_activation_scales(c0, T, scale):
    """Activations below and above unit scale whose SwiGLU outputs stay in fp16's normal range (the envelope the
    kernels compute in, see moe.h, Errors): parity with the oracle on both expert paths, and no status."""
    cfg = c0.cfg
    ub = inputs.f32_to_bf16_bits(inputs.bf16_bits_to_f32(inputs.activations(cfg, step=43, T=T)) * np.float32(scale))
    u = u_vals(ub)
    st, out = _status_calls(c0, ub, cfg.K)
    assert st == [0, 0, 0]
    idx = np.tile(np.arange(cfg.K), (T, 1))
    w = np.full((T, cfg.K), 1.0 / cfg.K)
    assert_close_inf(out, oracle_out(c0, u, idx, w), what=f"scale {scale}")


@pytest.mark.parametrize("T", [4, 64])
def test_swiglu_output_beyond_fp16_range_is_reported(c0, T):
    """At 1000x unit-scale activations the SwiGLU outputs exceed fp16's range (both paths keep h in fp16): the
    expert forward reports MOE_ERR_RANGE instead of returning silent infinities."""
    ub = inputs.f32_to_bf16_bits(inputs.bf16_bits_to_f32(inputs.activations(c0.cfg, step=44, T=T)) * np.float32(1e3))
    st, _ = _status_calls(c0, ub, c0.cfg.K)
    assert st[0] == 0 and st[1] == 6


def test_grouped_gemm_bounded_wait_reports_timeout(cuda_ok):
    """A grouped-GEMM CTA whose first operand stage is never marked full (test hook): its waits run out, the
    stack's error word says MOE_ERR_TIMEOUT, and the next call on the same context succeeds."""
    m = M()
    cfg = dataclasses.replace(CONFIGS[0], layers=2)
    stack = m.DeviceStack(cfg, lambda l: inputs.layer(cfg, l))
    T = 64  # 64 x 2 slots: the tensor-core path
    x0 = inputs.bf16_bits_to_f32(inputs.activations(cfg, step=45, T=T))
    res = run_stack(stack, cfg, T, x0, False,
                    opts=m.stack_opts(path=m.PATH_LAYERS, timeout_ns=20_000_000, drop_layer=1, drop_cta=0))
    assert res["err"] == 5
    res2 = run_stack(stack, cfg, T, x0, False, opts=m.stack_opts(path=m.PATH_LAYERS))
    assert res2["err"] == 0
    _check_stack(cfg, lambda l: inputs.layer(cfg, l), T, res2, x0, range(cfg.layers))
