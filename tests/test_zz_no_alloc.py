"""The allocation-free expert forward against the workspace entry point.

moe_expert_forward_noalloc serves callers that cannot allocate device memory
for a workspace (a host framework that owns every device allocation, or a
process whose allocator already holds nearly all of HBM).  It must give the
same results as moe_expert_forward, call after call, although every call
reuses the library's one fixed scratch array.
"""
import numpy as np
import pytest
import torch

from gen import CONFIGS, inputs
from oracle import moe_oracle as O
from parity import assert_close_inf

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _routing(host, ub, K):
    u = inputs.bf16_bits_to_f32(ub).astype(np.float64)
    logits = O.router_logits(u, host["router"])
    idx = O.topk(logits, K)
    return idx, O.gating(logits, idx)


def _both(M, layer, ub, K, idx, w, mode):
    T, H = ub.shape
    u = torch.from_numpy(ub.view(np.int16)).to(DEV)
    idx_d = torch.from_numpy(idx.astype(np.int32)).to(DEV)
    w_d = torch.from_numpy(w.astype(np.float32)).to(DEV)
    dtype = torch.int16 if mode == 1 else torch.float32
    base = torch.randn((T, H), device=DEV) if mode == 2 else None
    outs, perms = [], []
    for noalloc in (False, True):
        out = base.clone() if mode == 2 else torch.zeros((T, H), dtype=dtype, device=DEV)
        perm = torch.full((T * K,), -1, dtype=torch.int32, device=DEV)
        if noalloc:
            M.moe_expert_forward_noalloc(layer, u, K, idx_d, w_d, out, mode, perm_out=perm)
        else:
            ws = M.workspace(M.moe_workspace_size(layer, T, K))
            M.moe_expert_forward(layer, u, K, idx_d, w_d, out, mode, ws, perm_out=perm)
        torch.cuda.synchronize()
        o = out.cpu().numpy()
        if mode == 1:
            o = inputs.bf16_bits_to_f32(o.view(np.uint16))
        outs.append(o.astype(np.float64))
        perms.append(perm.cpu().numpy())
    return outs, perms


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row(cuda_ok):
    import int4_expert_ffn_top_b200 as M
    assert M.moe_noalloc_scratch_bytes() == 4 << 20
    for cfg_id, calls in ((0, [(13, 0), (4, 2)]), (1, [(1, 0), (3, 1)])):
        cfg = CONFIGS[cfg_id]
        host = inputs.layer(cfg, 2)
        layer = M.DeviceLayer(cfg, host)
        for call, (T, mode) in enumerate(calls):
            ub = inputs.activations(cfg, step=300 + 10 * call + cfg_id, T=T)
            idx, w = _routing(host, ub, cfg.K)
            (ref, got), (pref, pgot) = _both(M, layer, ub, cfg.K, idx, w, mode)
            assert np.all(np.isfinite(got))
            assert_close_inf(got, ref, what=f"cfg {cfg_id} call {call}")
            assert np.array_equal(pgot, pref)


def _oracle_out(host, ub, idx, w):
    u = inputs.bf16_bits_to_f32(ub).astype(np.float64)
    y = O.routed_outputs(u, host["experts"], idx)
    return O.combine(w, y, O.shared_gate(u, host["shared"]), O.shared_expert(u, host["shared"]))


def test_noalloc_tensor_core_path_on_two_calls_in_a_row(cuda_ok):
    """64 tokens x top-2 (128 slots) take the grouped-GEMM path, whose tensor maps, tile lists and bucket
    histograms then live in the shared scratch array: two calls in a row with different routing agree with the
    workspace entry point bit for bit and with the oracle."""
    import int4_expert_ffn_top_b200 as M
    cfg = CONFIGS[0]
    host = inputs.layer(cfg, 3)
    layer = M.DeviceLayer(cfg, host)
    T = 64
    assert M.moe_workspace_size(layer, T, cfg.K) <= M.moe_noalloc_scratch_bytes()
    for call in range(2):
        ub = inputs.activations(cfg, step=400 + call, T=T)
        idx, w = _routing(host, ub, cfg.K)
        if call:
            idx = (idx + 5) % cfg.E  # different buckets from the first call
        (ref, got), (pref, pgot) = _both(M, layer, ub, cfg.K, idx, w, 0)
        assert np.array_equal(got, ref) and np.array_equal(pgot, pref)
        assert_close_inf(got, _oracle_out(host, ub, idx, w), what=f"call {call}")


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_ok):
    import int4_expert_ffn_top_b200 as M
    cfg = CONFIGS[0]
    layer = M.DeviceLayer(cfg, inputs.layer(cfg, 0, experts=[]))
    T = 8000
    assert M.moe_workspace_size(layer, T, cfg.K) > M.moe_noalloc_scratch_bytes()
    out = torch.full((T, cfg.H), 5.0, device=DEV)
    with pytest.raises(M.MoEError) as e:
        M.moe_expert_forward_noalloc(layer, torch.zeros((T, cfg.H), dtype=torch.int16, device=DEV), cfg.K,
                                     torch.zeros((T, cfg.K), dtype=torch.int32, device=DEV),
                                     torch.zeros((T, cfg.K), device=DEV), out, 0)
    assert e.value.code == 3
    torch.cuda.synchronize()
    assert torch.all(out == 5.0)
