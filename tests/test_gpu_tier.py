"""GPU tests of the tiered expert pool: a layer's routed experts in pinned host memory behind an HBM cache.

The expert forward over the cache runs the same kernels over the same bytes as over a resident pool, so its
output must equal the resident pool's bit for bit, on both expert paths (GEMVs below 48 slots, grouped GEMMs
from 48); the cache's replacement choices are checked through the slot ids it hands out.
"""
import numpy as np
import pytest
import torch

from gen import CONFIGS, inputs
from oracle import moe_oracle as O
from parity import assert_close_inf
from test_gpu_layer import M, dev_bits, u_vals

pytestmark = pytest.mark.gpu
DEV = "cuda"


class Setup:
    def __init__(self, n_slots, cfg=CONFIGS[0]):
        m = M()
        self.cfg = cfg
        self.host = inputs.layer(cfg, 0)
        self.full = m.DeviceLayer(cfg, self.host)
        stride = m.block_stride(cfg.H, cfg.I)
        self.lean = m.DeviceLayer(cfg, dict(self.host, experts={}), pool=torch.zeros(stride, dtype=torch.uint8,
                                                                                       device=DEV))
        self.tier = m.TieredPool(self.lean, m.host_pool(cfg, self.host["experts"]), n_slots)


def _call(s, rng, T, experts_pool, step):
    """One forward over the cache and over the resident pool with tokens routed among experts_pool."""
    m, cfg, K = M(), s.cfg, s.cfg.K
    idx_h = np.stack([rng.choice(experts_pool, size=K, replace=False) for _ in range(T)]).astype(np.int32)
    w_h = rng.random((T, K)).astype(np.float32)
    w_h /= w_h.sum(1, keepdims=True)
    ub = inputs.activations(cfg, step=step, T=T)
    u, idx, w = dev_bits(ub), torch.from_numpy(idx_h).to(DEV), torch.from_numpy(w_h).to(DEV)
    idx_slot = torch.full_like(idx, -1)
    s.tier.acquire(idx_h, idx, idx_slot)
    out_t = torch.full((T, cfg.H), float("nan"), device=DEV)
    m.moe_expert_forward(s.tier, u, K, idx_slot, w, out_t, 0, m.workspace(m.moe_workspace_size(s.tier, T, K)))
    s.tier.release()
    out_f = torch.full((T, cfg.H), float("nan"), device=DEV)
    m.moe_expert_forward(s.full, u, K, idx, w, out_f, 0, m.workspace(m.moe_workspace_size(s.full, T, K)))
    torch.cuda.synchronize()
    return ub, idx_h, w_h, idx_slot.cpu().numpy(), out_t.cpu().numpy(), out_f.cpu().numpy()


@pytest.mark.parametrize("T", [13, 40])  # 26 slots (GEMVs) and 80 slots (grouped GEMMs) at top-2
def test_tiered_forward_equals_resident_pool(cuda_ok, T):
    s = Setup(n_slots=6)
    rng = np.random.default_rng(T)
    for step in range(6):  # six calls over different expert sets: the cache refills and evicts
        pool = rng.choice(s.cfg.E, size=6, replace=False)
        ub, idx_h, w_h, slots, out_t, out_f = _call(s, rng, T, pool, 100 + step)
        assert np.array_equal(out_t, out_f), f"call {step}"
        assert np.all((slots >= 0) & (slots < 6))
        if step == 0:  # and the oracle agrees with both
            L = s.host
            u = u_vals(ub)
            ref = O.combine(w_h, O.routed_outputs(u, L["experts"], idx_h), O.shared_gate(u, L["shared"]),
                            O.shared_expert(u, L["shared"]))
            assert_close_inf(out_t, ref)
    st = s.tier.stats()
    assert st["acquires"] == 6 and st["hits"] + st["misses"] == st["requested"]
    assert st["bytes_acquired"] == st["misses"] * M().block_bytes(s.cfg.H, s.cfg.I)


def _acquire(s, experts):
    idx = torch.tensor([experts], dtype=torch.int32, device=DEV)
    out = torch.full_like(idx, -1)
    s.tier.acquire(np.array(experts, np.int32), idx, out)
    s.tier.release()
    torch.cuda.synchronize()
    return out.cpu().numpy()[0].tolist()


def test_tiered_replacement_is_least_recently_used(cuda_ok):
    s = Setup(n_slots=3)
    assert _acquire(s, [0, 1]) == [0, 1]          # two misses into free slots
    assert _acquire(s, [2, 3]) == [2, 0]          # free slot 2, then the least recently used: expert 0's
    assert _acquire(s, [1, 2]) == [1, 2]          # hits
    assert _acquire(s, [0, 3]) == [1, 0]          # 3 hits in slot 0; 0 takes slot 1 (1 and 2 tie; lower slot)
    st = s.tier.stats()
    assert (st["requested"], st["hits"], st["misses"]) == (8, 3, 5)


def test_tiered_prefetch_hits_and_spares_the_last_acquire(cuda_ok):
    s = Setup(n_slots=4)
    side = torch.cuda.Stream()
    assert _acquire(s, [0, 1]) == [0, 1]
    s.tier.prefetch([2, 3, 4], stream=side)  # two free slots; slots of 0 and 1 are the last acquire's
    st = s.tier.stats()
    assert st["prefetched"] == 2
    rng = np.random.default_rng(7)
    ub, idx_h, w_h, slots, out_t, out_f = _call(s, rng, 13, np.array([2, 3]), 300)
    assert np.array_equal(out_t, out_f)
    st = s.tier.stats()
    assert st["prefetch_hits"] == 2 and st["misses"] == 2  # only the first acquire's two misses
    assert sorted(set(slots.reshape(-1).tolist())) == [2, 3]


def test_tiered_refusals(cuda_ok):
    s = Setup(n_slots=4)
    with pytest.raises(M().MoEError) as e:
        _acquire(s, [0, 1, 2, 3, 4])  # five distinct experts, four slots
    assert e.value.code == 3
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    idx = torch.tensor([[0, 5]], dtype=torch.int32, device=DEV)  # 5 was not acquired
    out = torch.full_like(idx, -1)
    s.tier.acquire(np.array([0], np.int32), idx, out, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 1
