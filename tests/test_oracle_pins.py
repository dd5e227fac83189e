"""Pins of the CPU oracle against what the Edge0 pages and plain mathematics fix.

Each test checks the oracle against something other than itself: exact rational
arithmetic, hand-built bit patterns, closed forms on structured weights,
invariants, and brute force on tiny inputs.  ``test_planted_mistakes_are_caught``
plants plausible mistakes in the oracle and checks that a pin fails for each.
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from gen import CONFIGS, inputs
from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- helpers (test-side packing)
def pack(codes: np.ndarray, bits: int) -> np.ndarray:
    """Inverse of the storage format: element k of a row at bits ``bits*(k % per)`` of word ``k // per``."""
    per = 32 // bits
    R, C = codes.shape
    c = codes.reshape(R, C // per, per).astype(np.uint64)
    w = np.zeros((R, C // per), dtype=np.uint64)
    for j in range(per):
        w |= c[:, :, j] << np.uint64(bits * j)
    return w.astype(np.uint32)


def qmat(codes, scale, bias, bits):
    codes = np.asarray(codes)
    R, C = codes.shape
    s = np.broadcast_to(np.asarray(scale, np.float16), (R, C // 64)).copy()
    b = np.broadcast_to(np.asarray(bias, np.float16), (R, C // 64)).copy()
    return dict(q=pack(codes, bits), s=s, b=b, bits=bits)


def zero_qmat(R, C, s=0.01, bits=4):
    mid = 8 if bits == 4 else 128
    return qmat(np.full((R, C), mid), s, -mid * np.float16(s), bits)


# ----------------------------------------------------------------------------- golden constants
def test_configs_match_page_constants():
    g = json.load(open(os.path.join(GOLDEN, "tiers.json")))
    c35, c8 = CONFIGS[1], CONFIGS[2]
    assert (c35.layers, c35.E, c35.K, c35.H) == (g["edge0-35b"]["layers"], g["edge0-35b"]["routed_experts"],
                                                g["edge0-35b"]["top_k"], g["edge0-35b"]["hidden"])
    assert (c8.layers, c8.E, c8.K) == (g["edge0-8b"]["layers"], g["edge0-8b"]["routed_experts"],
                                       g["edge0-8b"]["top_k"])
    for c in (CONFIGS[3], CONFIGS[4]):
        assert (c.layers, c.E, c.K, c.H) == (c35.layers, c35.E, c35.K, c35.H)
    assert O.GROUP == g["quant"]["group_size"]
    cfg = CONFIGS[1]
    ex = inputs.expert(cfg, 0, 0)
    assert ex["gate_up"]["bits"] == g["quant"]["expert_bits"]
    assert inputs.router(cfg, 0)["bits"] == g["quant"]["router_gate_bits"]
    assert inputs.shared(cfg, 0)["gate"]["bits"] == g["quant"]["shared_expert_gate_bits"]


# ----------------------------------------------------------------------------- formats and dequant
def test_hand_built_words():
    assert list(O.unpack_codes(np.array([[0x76543210]], np.uint32), 4)[0]) == list(range(8))
    assert list(O.unpack_codes(np.array([[0xFEDCBA98]], np.uint32), 4)[0]) == list(range(8, 16))
    assert list(O.unpack_codes(np.array([[0x03020100]], np.uint32), 8)[0]) == [0, 1, 2, 3]
    assert list(O.unpack_codes(np.array([[0xFF7F8001]], np.uint32), 8)[0]) == [1, 128, 127, 255]
    # second word holds elements 8..15
    w = np.array([[0x00000000, 0x000000F0]], np.uint32)
    assert list(np.nonzero(O.unpack_codes(w, 4)[0])[0]) == [9]


@pytest.mark.parametrize("bits", [4, 8])
def test_dequant_exhaustive_codes_exact(bits):
    n = 1 << bits
    rng = np.random.default_rng(1)
    for trial in range(20):
        s = np.float16(rng.uniform(0.005, 0.02) / (16 if bits == 8 else 1))
        b = np.float16(rng.uniform(-0.2, 0.2))
        codes = np.tile(np.arange(n), 64 // n if n < 64 else 1)[None, :64]
        if n > 64:
            codes = np.arange(n).reshape(n // 64, 64)
        m = qmat(codes, s, b, bits)
        got = O.dequant(m)
        for r in range(codes.shape[0]):
            for k in range(64):
                exact = Fraction(int(codes[r, k])) * Fraction(float(s)) + Fraction(float(b))
                assert Fraction(got[r, k]) == exact


def test_dequant_group_boundaries():
    codes = np.full((2, 192), 3)
    s = np.array([[0.01, 0.02, 0.005], [0.0078125, 0.015625, 0.03125]], np.float16)
    b = np.array([[0.1, -0.1, 0.0], [0.0, 0.5, -0.25]], np.float16)
    m = dict(q=pack(codes, 4), s=s, b=b, bits=4)
    W = O.dequant(m)
    for r in range(2):
        for k in (0, 63, 64, 127, 128, 191):
            g = k // 64
            assert W[r, k] == 3 * float(s[r, g]) + float(b[r, g])


def test_generator_formats():
    cfg = CONFIGS[0]
    ex = inputs.expert(cfg, 0, 3)
    gu = ex["gate_up"]
    assert gu["q"].shape == (2 * cfg.I, cfg.H // 8) and gu["q"].dtype == np.uint32
    assert np.all(gu["b"] == (np.float16(-8) * gu["s"]))
    assert gu["s"].min() >= np.float16(0.005) and gu["s"].max() <= np.float16(0.02)
    codes = O.unpack_codes(gu["q"], 4)
    hist = np.bincount(codes.reshape(-1), minlength=16)
    assert hist.size == 16 and hist.min() > 0.8 * codes.size / 16
    r = inputs.router(cfg, 0)
    assert np.all(r["b"] == (np.float16(-128) * r["s"]))
    # same stream -> same tensor; different expert -> different tensor
    assert np.array_equal(inputs.expert(cfg, 0, 3)["down"]["q"], ex["down"]["q"])
    assert not np.array_equal(inputs.expert(cfg, 0, 4)["down"]["q"], ex["down"]["q"])


def test_zipf_offsets_are_log_ranks():
    cfg = CONFIGS[3]
    beta = inputs.router(cfg, 0)["beta"].astype(np.float64)
    want = -1.1 * np.log(np.arange(1, cfg.E + 1))
    assert np.allclose(np.sort(beta)[::-1], want, rtol=1e-6, atol=1e-6)
    assert np.all(inputs.router(CONFIGS[1], 0)["beta"] == 0)


# ----------------------------------------------------------------------------- bf16 rounding and the glue
def test_round_bf16_known_values():
    cases = {1.0: 1.0, 1 + 2 ** -8: 1.0, 1 + 3 * 2 ** -8: 1 + 2 ** -6, 3.14159265: 3.140625,
             -2.0 - 2 ** -7: -2.0, 1 + 2 ** -8 + 2 ** -20: 1 + 2 ** -7, 0.0: 0.0}
    for v, want in cases.items():
        assert O.round_bf16(np.array([v]))[0] == want, v


def test_round_bf16_agrees_with_bit_rounding_of_fp32():
    v = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 10
    a = O.round_bf16(v.astype(np.float64))
    b = inputs.bf16_bits_to_f32(inputs.f32_to_bf16_bits(v)).astype(np.float64)
    assert np.array_equal(a, b)


def test_rmsnorm_closed_forms():
    x = np.full((1, 64), 3.0)
    assert np.allclose(O.rmsnorm(x, 0.0), 1.0)
    x = np.random.default_rng(2).standard_normal((3, 256))
    r = O.rmsnorm(x, 0.0)
    assert np.allclose(np.mean(r * r, axis=1), 1.0)
    assert np.allclose(O.rmsnorm(7.5 * x, 0.0), r)
    assert np.allclose(O.rmsnorm(np.full((1, 4), 1e-3), 1e-6)[0], 1e-3 / np.sqrt(1e-6 + 1e-6))


def test_activation_closed_forms():
    a = np.linspace(-40, 40, 801)
    assert O.silu(np.array([0.0]))[0] == 0.0 and O.sigmoid(np.array([0.0]))[0] == 0.5
    assert np.allclose(O.silu(a) - O.silu(-a), a, atol=1e-12)
    assert np.allclose(O.sigmoid(a) + O.sigmoid(-a), 1.0, atol=1e-15)
    assert np.allclose(O.sigmoid(np.array([1.0])), 1 / (1 + np.e ** -1), rtol=1e-15)
    assert np.all(np.isfinite(O.silu(np.array([-1e4, 1e4]))))


# ----------------------------------------------------------------------------- routing
def _brute_topk(scores, K):
    E = len(scores)
    key = lambda i: (scores[i], -i)  # larger score first, then lower index
    for S in itertools.combinations(range(E), K):
        rest = [j for j in range(E) if j not in S]
        if all(key(i) > key(j) for i in S for j in rest):
            return sorted(S, key=key, reverse=True)
    raise AssertionError


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(3)
    for _ in range(300):
        E = int(rng.integers(2, 11))
        K = int(rng.integers(1, min(E, 4) + 1))
        s = rng.integers(-3, 4, size=E).astype(np.float64)  # many ties
        assert list(O.topk(s[None], K)[0]) == _brute_topk(list(s), K)


def test_topk_all_equal_gives_lowest_indices():
    assert list(O.topk(np.zeros((1, 16)), 4)[0]) == [0, 1, 2, 3]


def test_gating_closed_forms():
    l = np.array([[0.3, -1.2, 2.0, 0.0]])
    idx = np.array([[2, 0]])
    w = O.gating(l, idx)
    assert np.isclose(w[0, 0], 1 / (1 + np.exp(0.3 - 2.0)), rtol=1e-14)
    assert np.isclose(w.sum(), 1.0, rtol=1e-15)
    assert np.allclose(O.gating(np.zeros((1, 8)), np.array([[0, 1, 2, 3]])), 0.25)
    assert np.allclose(O.gating(l + 100.0, idx), w, rtol=1e-13)
    # softmax over K equals softmax over all E renormalised on the K
    full = np.exp(l - l.max()) / np.exp(l - l.max()).sum()
    sel = full[0, idx[0]] / full[0, idx[0]].sum()
    assert np.allclose(w[0], sel, rtol=1e-14)


def test_router_closed_form_on_one_hot_weights():
    H, E = 128, 8
    rng = np.random.default_rng(4)
    pi = rng.permutation(H)[:E]
    c = rng.integers(1, 100, size=E)
    codes = np.full((E, H), 128)
    for e in range(E):
        codes[e, pi[e]] = 128 + c[e]
    s = np.float16(0.0009765625)
    R = qmat(codes, s, -128 * s, 8)
    R["beta"] = rng.standard_normal(E).astype(np.float32)
    u = O.round_bf16(rng.standard_normal((3, H)))
    want = c[None, :] * float(s) * u[:, pi] + R["beta"].astype(np.float64)
    assert np.allclose(O.router_logits(u, R), want, rtol=1e-15, atol=0)


# ----------------------------------------------------------------------------- expert FFN, LoRA, shared gate
def _perm_expert(H, I, rng):
    """Expert whose gate/up/down are scaled selection matrices: closed form output."""
    pg, pu = rng.permutation(H)[:I], rng.permutation(H)[:I]
    sig = rng.integers(0, I, size=H)
    s, sd = np.float16(0.015625), np.float16(0.0078125)
    gu = np.full((2 * I, H), 8)
    for j in range(I):
        gu[j, pg[j]] = 9       # gate_j = s * u[pg[j]]
        gu[I + j, pu[j]] = 10  # up_j = 2 s * u[pu[j]]
    dn = np.full((H, I), 8)
    for o in range(H):
        dn[o, sig[o]] = 5      # y_o = -3 sd * h[sig[o]]
    ex = dict(gate_up=qmat(gu, s, -8 * s, 4), down=qmat(dn, sd, -8 * sd, 4))
    return ex, pg, pu, sig, float(s), float(sd)


def test_expert_ffn_closed_form_on_selection_weights():
    rng = np.random.default_rng(5)
    H, I = 128, 64
    ex, pg, pu, sig, s, sd = _perm_expert(H, I, rng)
    u = O.round_bf16(rng.standard_normal((4, H)))
    g = s * u[:, pg]
    up = 2 * s * u[:, pu]
    h = g / (1 + np.exp(-g)) * up
    want = -3 * sd * h[:, sig]
    assert np.allclose(O.expert_ffn(u, ex), want, rtol=1e-13, atol=1e-15)
    assert np.allclose(O.expert_hidden(u, ex), h, rtol=1e-13, atol=1e-15)


def test_zero_expert_gives_zero():
    H, I = 128, 64
    ex = dict(gate_up=zero_qmat(2 * I, H), down=zero_qmat(H, I))
    u = np.random.default_rng(6).standard_normal((2, H))
    assert np.all(O.expert_ffn(u, ex) == 0.0)


def test_lora_unmerged_equals_merged_and_one_hot():
    rng = np.random.default_rng(7)
    H, I, r = 128, 64, 8
    cfg = CONFIGS[0]
    ex = inputs.expert(cfg, 0, 1)
    lo = dict(A=(rng.standard_normal((r, H)) * 0.02).astype(np.float16),
              B=(rng.standard_normal((I, r)) * 0.02).astype(np.float16), scale=1.0)
    u = rng.standard_normal((5, cfg.H))
    # unmerged delta on the gate equals merging B A into the dequantised gate rows
    ex2 = dict(gate_up=ex["gate_up"], down=ex["down"])
    Wgu = O.dequant(ex["gate_up"])
    I2 = Wgu.shape[0] // 2
    lo2 = dict(A=(rng.standard_normal((r, cfg.H)) * 0.02).astype(np.float16),
               B=(rng.standard_normal((I2, r)) * 0.02).astype(np.float16), scale=1.0)
    merged_gate = Wgu[:I2] + lo2["B"].astype(np.float64) @ lo2["A"].astype(np.float64)
    a = u @ merged_gate.T
    b = u @ Wgu[I2:].T
    want = (a / (1 + np.exp(-a)) * b) @ O.dequant(ex["down"]).T
    assert np.allclose(O.expert_ffn(u, ex2, lora_gate=lo2), want, rtol=1e-11, atol=1e-11)
    # B = 0: no delta
    z = dict(A=lo["A"], B=np.zeros_like(lo["B"]), scale=1.0)
    x = rng.standard_normal((2, H))
    assert np.all(O.lora_delta(x, z) == 0)
    # rank-1 one-hot: delta[:, j] = x[:, i]
    A = np.zeros((1, H), np.float16); A[0, 17] = 1
    B = np.zeros((I, 1), np.float16); B[41, 0] = 1
    d = O.lora_delta(x, dict(A=A, B=B, scale=1.0))
    assert np.array_equal(d[:, 41], x[:, 17]) and np.count_nonzero(d) == np.count_nonzero(x[:, 17])


def _one_hot_lora(out_dim, in_dim, i, j, c, r=2):
    """Rank-r adapter whose only nonzero path maps input ``i`` to output ``j`` with gain ``c`` (through rank 1)."""
    A = np.zeros((r, in_dim), np.float16)
    A[1, i] = 1
    B = np.zeros((out_dim, r), np.float16)
    B[j, 1] = c
    return dict(A=A, B=B, scale=1.0)


def test_lora_on_every_projection_closed_form():
    """Selection-matrix expert with a one-hot adapter on each of gate, up and down (2kiu.com, "Recover-LoRA"
    bullet: the adapter stays unmerged on the frozen base).  Each adapter adds ``c * input[i]`` to one output of
    its own projection, before the activation, so the closed form says which projection carries which adapter;
    the shared expert must wire ``lora_gate`` / ``lora_up`` / ``lora_down`` to the same projections."""
    rng = np.random.default_rng(13)
    H, I = 128, 64
    ex, pg, pu, sig, s, sd = _perm_expert(H, I, rng)
    u = O.round_bf16(rng.standard_normal((4, H)))
    (ig, jg, cg), (iu, ju, cu), (ih, od, cd) = (5, 7, 0.5), (9, 11, -0.25), (13, 17, 0.75)
    lg, lu, ld = _one_hot_lora(I, H, ig, jg, cg), _one_hot_lora(I, H, iu, ju, cu), _one_hot_lora(H, I, ih, od, cd)
    g = s * u[:, pg]
    g[:, jg] += cg * u[:, ig]
    up = 2 * s * u[:, pu]
    up[:, ju] += cu * u[:, iu]
    h = g / (1 + np.exp(-g)) * up
    want = -3 * sd * h[:, sig]
    want[:, od] += cd * h[:, ih]
    assert np.allclose(O.expert_hidden(u, ex, lg, lu), h, rtol=1e-13, atol=1e-15)
    assert np.allclose(O.expert_ffn(u, ex, lg, lu, ld), want, rtol=1e-13, atol=1e-15)
    sh = dict(ex, lora_gate=lg, lora_up=lu, lora_down=ld)
    assert np.allclose(O.shared_expert(u, sh), want, rtol=1e-13, atol=1e-15)


def test_lora_unmerged_equals_merged_on_up_and_down():
    """``W + B A`` merged into the dequantised up and down matrices equals the unmerged deltas."""
    rng = np.random.default_rng(14)
    cfg = CONFIGS[0]
    ex = inputs.expert(cfg, 0, 2)
    H, I, r = cfg.H, cfg.I, 4
    lo = lambda o, i: dict(A=(rng.standard_normal((r, i)) * 0.05).astype(np.float16),
                           B=(rng.standard_normal((o, r)) * 0.05).astype(np.float16), scale=1.0)
    lu, ld = lo(I, H), lo(H, I)
    Wgu = O.dequant(ex["gate_up"])
    Wu = Wgu[I:] + lu["B"].astype(np.float64) @ lu["A"].astype(np.float64)
    Wd = O.dequant(ex["down"]) + ld["B"].astype(np.float64) @ ld["A"].astype(np.float64)
    u = rng.standard_normal((3, H))
    a = u @ Wgu[:I].T
    want = (a / (1 + np.exp(-a)) * (u @ Wu.T)) @ Wd.T
    assert np.allclose(O.expert_ffn(u, ex, lora_up=lu, lora_down=ld), want, rtol=1e-11, atol=1e-11)


def test_routed_down_lora_reaches_the_layer_output():
    """A one-hot down adapter on every routed expert (the batched-decode workload's LoRA) adds
    ``c * h_e[i]`` to output ``o`` of every slot; through the combine the layer output moves by
    ``sum_k w_k c h_{e_k}[i]`` at ``o`` and nowhere else."""
    cfg = CONFIGS[0]
    L = _tiny_layer(cfg)
    u = O.round_bf16(inputs.bf16_bits_to_f32(inputs.activations(cfg)).astype(np.float64))
    ih, od, cd = 3, 29, 0.625
    base = O.layer_forward(u, L, cfg.K)
    for e in L["experts"]:
        L["experts"][e]["down_lora"] = _one_hot_lora(cfg.H, cfg.I, ih, od, cd)
    r = O.layer_forward(u, L, cfg.K)
    assert np.array_equal(r["idx"], base["idx"])
    hk = np.stack([[O.expert_hidden(u[t:t + 1], L["experts"][int(e)])[0, ih] for e in base["idx"][t]]
                   for t in range(cfg.T)])
    dy = r["y"] - base["y"]
    assert np.allclose(dy[:, :, od], cd * hk, rtol=1e-12, atol=1e-15)
    assert np.count_nonzero(np.delete(dy, od, axis=2)) == 0
    dout = r["out"] - base["out"]
    assert np.allclose(dout[:, od], (base["w"] * cd * hk).sum(1), rtol=1e-11, atol=1e-15)
    assert np.count_nonzero(np.delete(dout, od, axis=1)) == 0


def test_routed_gate_up_lora_reaches_the_slot_outputs():
    """One-hot gate and up adapters on every routed expert: the gate adapter adds ``cg * u[ig]`` to gate output
    ``jg`` and the up adapter ``cu * u[iu]`` to up output ``ju`` of every slot, before the SiLU, so each slot's
    hidden values change at ``jg`` and ``ju`` only, by the closed form through ``silu(a) * b``."""
    cfg = CONFIGS[0]
    L = _tiny_layer(cfg)
    u = O.round_bf16(inputs.bf16_bits_to_f32(inputs.activations(cfg)).astype(np.float64))
    ig, jg, cg, iu, ju, cu = 5, 7, 0.75, 11, 19, -0.5
    base = O.layer_forward(u, L, cfg.K)
    for e in L["experts"]:
        L["experts"][e]["gate_lora"] = _one_hot_lora(cfg.I, cfg.H, ig, jg, cg)
        L["experts"][e]["up_lora"] = _one_hot_lora(cfg.I, cfg.H, iu, ju, cu)
    r = O.layer_forward(u, L, cfg.K)
    assert np.array_equal(r["idx"], base["idx"])
    for t in range(cfg.T):
        for k, e in enumerate(base["idx"][t]):
            ex = L["experts"][int(e)]
            Wgu = O.dequant(ex["gate_up"])
            I = Wgu.shape[0] // 2
            a = u[t] @ Wgu[:I].T
            b = u[t] @ Wgu[I:].T
            a2, b2 = a.copy(), b.copy()
            a2[jg] += cg * u[t, ig]
            b2[ju] += cu * u[t, iu]
            h2 = O.silu(a2) * b2
            assert np.allclose(r["y"][t, k], h2 @ O.dequant(ex["down"]).T, rtol=1e-11, atol=1e-12)
            dh = h2 - O.silu(a) * b
            assert np.count_nonzero(np.delete(dh, [jg, ju])) == 0 and dh[jg] != 0 and dh[ju] != 0


def test_shared_gate_half_on_zero_weights():
    H = 128
    sh = dict(gate=zero_qmat(1, H, s=0.01 / 16, bits=8))
    u = np.random.default_rng(8).standard_normal((3, H))
    assert np.all(O.shared_gate(u, sh) == 0.5)


# ----------------------------------------------------------------------------- layer-level invariants
def _tiny_layer(cfg, layer=0):
    return inputs.layer(cfg, layer, threads=2)


def test_layer_with_zero_routed_experts_is_half_shared():
    cfg = CONFIGS[0]
    L = _tiny_layer(cfg)
    for e in L["experts"]:
        L["experts"][e] = dict(gate_up=zero_qmat(2 * cfg.I, cfg.H), down=zero_qmat(cfg.H, cfg.I))
    L["shared"]["gate"] = zero_qmat(1, cfg.H, s=0.01 / 16, bits=8)
    u = O.round_bf16(inputs.bf16_bits_to_f32(inputs.activations(cfg)).astype(np.float64))
    r = O.layer_forward(u, L, cfg.K)
    assert np.allclose(r["out"], 0.5 * O.shared_expert(u, L["shared"]), rtol=1e-14, atol=0)


def test_layer_sparse_equals_dense_masked_mixture():
    cfg = CONFIGS[0]
    L = _tiny_layer(cfg)
    u = inputs.bf16_bits_to_f32(inputs.activations(cfg)).astype(np.float64)
    r = O.layer_forward(u, L, cfg.K)
    # dense: every expert on every token, weights zero outside the selection
    Y = np.stack([O.expert_ffn(u, L["experts"][e]) for e in range(cfg.E)], axis=1)  # [T,E,H]
    Wd = np.zeros((cfg.T, cfg.E))
    for t in range(cfg.T):
        Wd[t, r["idx"][t]] = r["w"][t]
    dense = np.einsum("te,teh->th", Wd, Y) + r["g"][:, None] * r["ys"]
    assert np.allclose(r["out"], dense, rtol=1e-12, atol=1e-12)
    # K = E reduces to the dense softmax mixture over all experts
    rE = O.layer_forward(u, L, cfg.E)
    pfull = np.exp(rE["logits"] - rE["logits"].max(1, keepdims=True))
    pfull /= pfull.sum(1, keepdims=True)
    assert np.allclose(np.einsum("te,teh->th", pfull, Y) + rE["g"][:, None] * rE["ys"], rE["out"],
                       rtol=1e-12, atol=1e-12)


def test_predicted_routing_overrides_indices_not_weights():
    cfg = CONFIGS[0]
    L = _tiny_layer(cfg)
    u = inputs.bf16_bits_to_f32(inputs.activations(cfg)).astype(np.float64)
    forced = np.array([[5, 3], [0, 1], [15, 2], [7, 8]])
    r = O.layer_forward(u, L, cfg.K, routing=forced)
    assert np.array_equal(r["idx"], forced)
    assert np.allclose(r["w"], O.gating(r["logits"], forced))


# ----------------------------------------------------------------------------- prerouter
def test_prerouter_closed_forms():
    H, E, P = 64, 16, 16
    rng = np.random.default_rng(9)
    u = rng.standard_normal((3, H))
    sel = np.array([[3, 9], [0, 15], [4, 5]])
    # zero weights: the prediction is the ranking of b2
    b2 = rng.permutation(E).astype(np.float16)
    head = dict(W1=np.zeros((P, H + E), np.float16), b1=np.zeros(P, np.float16),
                W2=np.zeros((E, P), np.float16), b2=b2)
    pred, p = O.prerouter_predict(u, sel, head, E, 2)
    assert all(list(pred[t]) == list(np.argsort(-b2.astype(float), kind="stable")[:2]) for t in range(3))
    # multi-hot path through a permutation: p[pi(e)] = silu(c) for selected e
    pi = rng.permutation(E)
    W1 = np.zeros((P, H + E), np.float16)
    W1[np.arange(E), H + np.arange(E)] = 2.0        # z_e = silu(2 * mh_e)
    W2 = np.zeros((E, P), np.float16)
    W2[pi, np.arange(E)] = 1.0                       # p[pi[e]] = z_e
    head = dict(W1=W1, b1=np.zeros(P, np.float16), W2=W2, b2=np.zeros(E, np.float16))
    pred, p = O.prerouter_predict(u, sel, head, E, 2)
    for t in range(3):
        assert sorted(pred[t]) == sorted(pi[sel[t]])
        assert list(pred[t]) == sorted(pi[sel[t]])  # equal scores: lower index first
        assert np.isclose(p[t, pi[sel[t][0]]], 2 / (1 + np.exp(-2.0)), rtol=1e-15)
    assert np.all(O.multi_hot(sel, E).sum(1) == 2)


def test_prerouter_reads_the_executed_experts_under_predicted_routing():
    """The head's multi-hot input is the set the layer executed, not the router's own top-K: with a head
    that maps the multi-hot through a permutation, the prediction is the permuted executed set."""
    cfg = CONFIGS[0]
    L = _tiny_layer(cfg)
    E, H, P = cfg.E, cfg.H, cfg.P
    rng = np.random.default_rng(12)
    pi = rng.permutation(E)
    W1 = np.zeros((P, H + E), np.float16)
    W1[np.arange(E), H + np.arange(E)] = 2.0  # z_e = silu(2 * multi_hot_e); the u columns are zero
    W2 = np.zeros((E, P), np.float16)
    W2[pi, np.arange(E)] = 1.0                 # p[pi[e]] = z_e
    L["prerouter"] = dict(W1=W1, b1=np.zeros(P, np.float16), W2=W2, b2=np.zeros(E, np.float16))
    u = inputs.bf16_bits_to_f32(inputs.activations(cfg)).astype(np.float64)
    true_idx = O.layer_forward(u, L, cfg.K)["true_idx"]
    forced = (true_idx + 5) % E  # never the router's own choice
    r = O.layer_forward(u, L, cfg.K, routing=forced)
    for t in range(cfg.T):
        assert sorted(r["pred"][t]) == sorted(pi[forced[t]])
        assert not set(r["pred"][t]) & set(pi[true_idx[t]])


# ----------------------------------------------------------------------------- buckets
def test_buckets_brute_force_and_invariants():
    rng = np.random.default_rng(10)
    for _ in range(50):
        E = int(rng.integers(1, 12))
        T, K = int(rng.integers(0, 9)), int(rng.integers(1, 4))
        idx = rng.integers(0, E, size=(T, K))
        b = O.buckets(idx, E)
        flat = idx.reshape(-1)
        brute = [s for e in range(E) for s in range(T * K) if flat[s] == e]
        assert list(b["perm"]) == brute
        assert list(b["count"]) == [int((flat == e).sum()) for e in range(E)]
        assert b["offset"][0] == 0 and b["offset"][-1] == T * K
        assert np.array_equal(np.diff(b["offset"]), b["count"])
        assert np.array_equal(b["perm"][b["inv"]], np.arange(T * K))


# ----------------------------------------------------------------------------- pin sensitivity
def _ffn_lora_after_silu(u, ex, lora_gate=None, lora_up=None, lora_down=None):
    """Planted mistake: the gate projection's LoRA delta added after SiLU instead of before."""
    Wgu = O.dequant(ex["gate_up"])
    I = Wgu.shape[0] // 2
    a = np.asarray(u, np.float64) @ Wgu[:I].T
    b = np.asarray(u, np.float64) @ Wgu[I:].T + O.lora_delta(u, lora_up)
    h = (O.silu(a) + O.lora_delta(u, lora_gate)) * b
    return h @ O.dequant(ex["down"]).T + O.lora_delta(h, lora_down)


def _prerouter_on_true_topk(monkeypatch):
    """Planted mistake: the head's multi-hot built from the router's own top-K instead of the executed set."""
    layer_forward = O.layer_forward

    def lf(u, L, K, routing=None, K_next=None):
        r = layer_forward(u, L, K, routing, K_next)
        if "prerouter" in L:
            r["pred"], r["p"] = O.prerouter_predict(u, r["true_idx"], L["prerouter"], r["logits"].shape[1],
                                                    K_next or K)
        return r

    monkeypatch.setattr(O, "layer_forward", lf)
    return O.prerouter_predict


def _reverse_within_buckets(b):
    perm = b["perm"].copy()
    for e in range(len(b["count"])):
        perm[b["offset"][e]:b["offset"][e + 1]] = perm[b["offset"][e]:b["offset"][e + 1]][::-1]
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    return dict(b, perm=perm, inv=inv)


def test_planted_mistakes_are_caught(monkeypatch):
    """Plant plausible mistakes in the oracle (on the CPU) and check a pin fails for each."""
    planted = {
        "dequant drops bias": lambda: monkeypatch.setattr(
            O, "dequant", lambda m, _d=O.dequant: _d(dict(m, b=np.zeros_like(m["b"])))),
        "nibbles high first": lambda: monkeypatch.setattr(
            O, "unpack_codes", lambda w, bits, _u=O.unpack_codes: _u(w, bits).reshape(
                w.shape[0], -1, 32 // bits)[:, :, ::-1].reshape(w.shape[0], -1)),
        "gate/up halves swapped": lambda: monkeypatch.setattr(
            O, "expert_ffn", lambda u, ex, *a, _f=O.expert_ffn, **k: _f(u, dict(ex, gate_up=dict(
                ex["gate_up"], q=np.roll(ex["gate_up"]["q"], ex["gate_up"]["q"].shape[0] // 2, 0),
                s=np.roll(ex["gate_up"]["s"], ex["gate_up"]["s"].shape[0] // 2, 0),
                b=np.roll(ex["gate_up"]["b"], ex["gate_up"]["b"].shape[0] // 2, 0))), *a, **k)),
        "top-k tie to higher index": lambda: monkeypatch.setattr(
            O, "topk", lambda s, K: np.stack([np.lexsort((-np.arange(s.shape[1]), -row))[:K] for row in s])),
        "silu sign flipped": lambda: monkeypatch.setattr(O, "sigmoid", lambda a: 0.5 * (1.0 - np.tanh(0.5 * a))),
        "predicted routing ignored": lambda: monkeypatch.setattr(
            O, "layer_forward", lambda u, L, K, routing=None, K_next=None, _f=O.layer_forward: _f(u, L, K, None, K_next)),
        "layer input not rounded to bf16": lambda: monkeypatch.setattr(
            O, "layer_input", lambda x, eps=1e-6: O.rmsnorm(x, eps)),
        "gating softmax over all E, not the K": lambda: monkeypatch.setattr(
            O, "gating", lambda l, idx: np.take_along_axis(
                np.exp(l - l.max(1, keepdims=True)) / np.exp(l - l.max(1, keepdims=True)).sum(1, keepdims=True),
                idx, axis=1)),
        "LoRA delta dropped": lambda: monkeypatch.setattr(O, "lora_delta", lambda x, lo: 0.0),
        "gate LoRA added after the activation": lambda: monkeypatch.setattr(O, "expert_ffn", _ffn_lora_after_silu),
        "shared gate ignored": lambda: monkeypatch.setattr(
            O, "shared_gate", lambda u, sh: np.ones(np.asarray(u).shape[0])),
        "combine drops the shared expert": lambda: monkeypatch.setattr(
            O, "combine", lambda w, y, g, ys: np.einsum("tk,tkh->th", w, y)),
        "Prerouter fed the router's own top-K": lambda: monkeypatch.setattr(
            O, "prerouter_predict", _prerouter_on_true_topk(monkeypatch)),
        "bucket order descending within an expert": lambda: monkeypatch.setattr(
            O, "buckets", lambda idx, E, _b=O.buckets: _reverse_within_buckets(_b(idx, E))),
        "router offset beta ignored": lambda: monkeypatch.setattr(
            O, "router_logits", lambda u, R, _r=O.router_logits: _r(u, dict(R, beta=np.zeros_like(R["beta"])))),
        "RMSNorm without eps": lambda: monkeypatch.setattr(
            O, "rmsnorm", lambda x, eps=1e-6, _n=O.rmsnorm: _n(x, 0.0)),
        "up LoRA dropped": lambda: monkeypatch.setattr(
            O, "expert_ffn", lambda u, ex, lora_gate=None, lora_up=None, lora_down=None, _f=O.expert_ffn:
            _f(u, ex, lora_gate, None, lora_down)),
        "down LoRA dropped": lambda: monkeypatch.setattr(
            O, "expert_ffn", lambda u, ex, lora_gate=None, lora_up=None, lora_down=None, _f=O.expert_ffn:
            _f(u, ex, lora_gate, lora_up, None)),
        "routed down LoRA dropped": lambda: monkeypatch.setattr(
            O, "routed_outputs", lambda u, experts, idx, _r=O.routed_outputs: _r(
                u, {e: {k: v for k, v in ex.items() if k != "down_lora"} for e, ex in experts.items()}, idx)),
        "routed gate/up adapters dropped": lambda: monkeypatch.setattr(
            O, "routed_outputs", lambda u, experts, idx, _r=O.routed_outputs: _r(
                u, {e: {k: v for k, v in ex.items() if k not in ("gate_lora", "up_lora")} for e, ex in experts.items()},
                idx)),
        "routed gate/up adapters swapped": lambda: monkeypatch.setattr(
            O, "routed_outputs", lambda u, experts, idx, _r=O.routed_outputs: _r(
                u, {e: dict(ex, **({"gate_lora": ex["up_lora"], "up_lora": ex["gate_lora"]} if "up_lora" in ex else {}))
                    for e, ex in experts.items()}, idx)),
        "shared gate/up adapters swapped": lambda: monkeypatch.setattr(
            O, "shared_expert", lambda u, sh, _f=O.expert_ffn: _f(u, sh, sh.get("lora_up"), sh.get("lora_gate"),
                                                                  sh.get("lora_down"))),
    }
    pins = [test_hand_built_words, lambda: test_dequant_exhaustive_codes_exact(4), test_dequant_group_boundaries,
            test_expert_ffn_closed_form_on_selection_weights, test_topk_brute_force_with_ties,
            test_topk_all_equal_gives_lowest_indices, test_activation_closed_forms,
            test_router_closed_form_on_one_hot_weights, test_stack_forward_with_zero_experts_keeps_the_residual,
            test_stack_forward_predicted_routing_executes_the_previous_prediction, test_rmsnorm_closed_forms,
            test_gating_closed_forms, test_lora_unmerged_equals_merged_and_one_hot, test_shared_gate_half_on_zero_weights,
            test_layer_with_zero_routed_experts_is_half_shared, test_layer_sparse_equals_dense_masked_mixture,
            test_prerouter_closed_forms, test_prerouter_reads_the_executed_experts_under_predicted_routing,
            test_buckets_brute_force_and_invariants, test_lora_on_every_projection_closed_form,
            test_lora_unmerged_equals_merged_on_up_and_down, test_routed_down_lora_reaches_the_layer_output,
            test_routed_gate_up_lora_reaches_the_slot_outputs]
    for name, plant in planted.items():
        plant()
        failed = False
        for pin in pins:
            try:
                pin()
            except AssertionError:
                failed = True
                break
        monkeypatch.undo()
        assert failed, f"no pin caught: {name}"


# ----------------------------------------------------------------------------- stack glue and predicted routing
def _zeroed_layer(cfg, l):
    """A c0-shaped layer whose routed experts, shared expert and LoRA deltas are all exactly zero."""
    L = inputs.layer(cfg, l)
    for m in [*(ex[k] for ex in L["experts"].values() for k in ("gate_up", "down")),
              L["shared"]["gate_up"], L["shared"]["down"]]:
        m["s"] = np.zeros_like(m["s"])
        m["b"] = np.zeros_like(m["b"])
    for k in ("lora_gate", "lora_up", "lora_down"):
        if L["shared"].get(k):
            L["shared"][k]["B"] = np.zeros_like(L["shared"][k]["B"])
    return L


def test_stack_forward_with_zero_experts_keeps_the_residual():
    """x_{l+1} = x_l + MoE_l(...) with every expert weight zero: x never changes, so every layer sees
    the same normed input bf16(rmsnorm(x0))."""
    cfg = CONFIGS[0]
    x0 = np.random.default_rng(3).standard_normal((cfg.T, cfg.H))
    res = O.stack_forward(x0, [_zeroed_layer(cfg, l) for l in range(3)], cfg.K)
    assert np.array_equal(res["x"], x0)
    u0 = O.round_bf16(O.rmsnorm(x0))
    for tr in res["trace"]:
        assert np.array_equal(tr["u"], u0)


def test_stack_forward_predicted_routing_executes_the_previous_prediction():
    """With zero Prerouter weights the prediction is the ranking of b2 (a permutation here); with
    predicted routing every layer after the first executes exactly that prediction, layer 0 its own top-K."""
    cfg = CONFIGS[0]
    rng = np.random.default_rng(11)
    b2 = rng.permutation(cfg.E).astype(np.float16)
    want = list(np.argsort(-b2.astype(float), kind="stable")[:cfg.K])
    layers = []
    for l in range(3):
        L = inputs.layer(cfg, l)
        hd = L["prerouter"]
        L["prerouter"] = dict(W1=np.zeros_like(hd["W1"]), b1=np.zeros_like(hd["b1"]),
                              W2=np.zeros_like(hd["W2"]), b2=b2)
        layers.append(L)
    x0 = rng.standard_normal((cfg.T, cfg.H))
    res = O.stack_forward(x0, layers, cfg.K, predicted_routing=True)
    tr = res["trace"]
    assert np.array_equal(tr[0]["idx"], tr[0]["true_idx"])
    for l in range(3):
        assert all(list(tr[l]["pred"][t]) == want for t in range(cfg.T))
    for l in (1, 2):
        assert all(list(tr[l]["idx"][t]) == want for t in range(cfg.T))
