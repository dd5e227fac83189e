"""Benchmark of the routed-expert stack on B200.

Default workload: the 35B-shaped MoE stack (40 layers x 256 routed experts,
top-4, hidden 2048, int4 group-64 experts, 8-bit router and shared gate,
shared expert with LoRA r=16, one Prerouter head per layer) decoding one token
per step (batch 1).  A step is one token through all 40 layers.  Every rank is
an independent replica (batch-1 decode does not shard; weak scaling).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line on rank 0.  Beside the headline it reports the 35B-shaped
prefill (3,328 tokens), the 8B-shaped decode and a 64-token batched decode with
predicted routing, and, at N = 1, the float64 oracle timed on the host cores.
``--impl reference`` times only that oracle, on rank 0: each step is one of
its work items for a batch-1 token (route, one routed expert, shared expert,
combine + Prerouter), and seconds per token are taken from the per-kind means.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gen import CONFIGS, inputs  # noqa: E402

METRIC = "MoE-stack decode tok/s (35B-shape, bs=1) & HBM GB/s vs peak; prefill tok/s"
CFG_ID = 1
PREFILL_CFG_ID = 3
DECODE_8B_CFG_ID = 2
BATCHED_CFG_ID = 4
EPS = 1e-6
N_TOKENS = 64  # distinct tokens cycled through the steps


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def token_layer_bytes(cfg) -> int:
    """Algorithmic HBM bytes one token reads in one layer (batch-1 decode)."""
    def mat(out, inp):  # int4 codes + fp16 scale and bias per 64 inputs
        return out * (inp // 2 + 4 * (inp // 64))
    blk = mat(2 * cfg.I, cfg.H) + mat(cfg.H, cfg.I)
    shared = mat(2 * cfg.I_s, cfg.H) + mat(cfg.H, cfg.I_s)
    lora = 2 * (cfg.r * cfg.H * 2 + cfg.I_s * cfg.r * 2) + cfg.r * cfg.I_s * 2 + cfg.H * cfg.r * 2
    router = cfg.E * (cfg.H + 4 * (cfg.H // 64))
    sgate = cfg.H + 4 * (cfg.H // 64)
    pre = cfg.P * cfg.H * 2 + cfg.P * cfg.K * 2 + cfg.P * 2 + cfg.E_next * cfg.P * 2 + cfg.E_next * 2
    return cfg.K * blk + shared + lora + router + sgate + pre


def max_over_ranks(v: float, dist, device) -> float:
    """The largest of every rank's value (the whole job waits for the slowest replica)."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Units per second processed by all ranks together over the (max-over-ranks) time ms."""
    return units_per_rank * world / (ms / 1000.0)


def expert_flops(cfg, T: int) -> float:
    """Algorithmic tensor-core work of one layer's experts: T*K routed slots and T shared-expert rows,
    each 2*(2I*H) for gate/up plus 2*(H*I) for down."""
    return 2.0 * (T * cfg.K + T) * 3 * cfg.H * cfg.I


def prefill_leg(dev, M, passes: int = 5, cfg=None):
    """Prefill (default: the 35B shape, 3,328 tokens through the 40-layer stack; per-layer launches, grouped-GEMM
    experts), plus one layer's expert forward timed alone for the tensor-core fraction."""
    import torch
    cfg = cfg or CONFIGS[PREFILL_CFG_ID]
    T, K = cfg.T, cfg.K
    t_build = time.time()
    stack = M.DeviceStack(cfg, lambda l: inputs.layer(cfg, l), device=dev)
    st = M.StackStructs(stack)
    ws = M.workspace(M.moe_stack_workspace_size(st, T, K, K), device=dev)
    x0 = torch.from_numpy(inputs.bf16_bits_to_f32(inputs.activations(cfg, step=1, T=T))).to(dev)
    x = torch.empty_like(x0)
    err = torch.zeros((1,), dtype=torch.int32, device=dev)
    opts = M.stack_opts(path=M.PATH_LAYERS)
    stream = torch.cuda.current_stream(dev)
    build_s = time.time() - t_build

    def run():
        x.copy_(x0)
        M.moe_stack_decode(st, x, K, K, EPS, ws, err_word=err, opts=opts)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # cold: the first pass after the upload, with L2 flushed by a 512 MB device write
    flush = torch.empty((512 << 20,), dtype=torch.uint8, device=dev)
    flush.fill_(1)
    torch.cuda.synchronize(dev)

    def cold():
        e0.record(stream)
        run()
        e1.record(stream)
        torch.cuda.synchronize(dev)

    _, win_cold = timed_window(cold)
    ms_cold = e0.elapsed_time(e1)
    del flush
    for _ in range(2):
        run()
    torch.cuda.synchronize(dev)

    def warm():
        e0.record(stream)
        for _ in range(passes):
            run()
        e1.record(stream)
        torch.cuda.synchronize(dev)

    _, win = timed_window(warm)
    if int(err.item()) != 0:
        raise RuntimeError(f"prefill: device-side wait timed out (status {int(err.item())})")
    ms_pass = e0.elapsed_time(e1) / passes

    # one layer's expert forward (bucketing, permute, both grouped GEMMs, LoRA, combine) timed alone
    L = stack.layers[1]
    u = torch.empty((T, cfg.H), dtype=torch.int16, device=dev)
    M.moe_rmsnorm_bf16(x0, EPS, u)
    logits = torch.empty((T, cfg.E), device=dev)
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    w = torch.empty((T, K), device=dev)
    M.moe_route_topk(L, u, K, logits, idx, w)
    out = torch.empty((T, cfg.H), device=dev)
    ews = M.workspace(M.moe_workspace_size(L, T, K), device=dev)
    for _ in range(3):
        M.moe_expert_forward(L, u, K, idx, w, out, 0, ews)
    torch.cuda.synchronize(dev)
    reps = 10
    e0.record(stream)
    for _ in range(reps):
        M.moe_expert_forward(L, u, K, idx, w, out, 0, ews)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_ef = e0.elapsed_time(e1) / reps
    touched = int(torch.unique(idx).numel())
    del stack, st, ws, ews
    torch.cuda.empty_cache()
    flops = expert_flops(cfg, T)
    try:
        peak = float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"])
        peak_kind = "measured (burst bf16; the fp16 tensor path has the same nominal rate)"
    except Exception:
        peak, peak_kind = 1590.0, "fallback"
    achieved = flops / (ms_ef / 1000.0) / 1e12
    per_layer = 1 + 2 + 10 + 3  # rmsnorm; router + top-K; expert forward; Prerouter W1, W2, top-K
    return {
        "workload": f"{cfg.name}: {T:,} tokens through {cfg.layers} layers ({cfg.E} experts, top-{cfg.K}, H {cfg.H}, "
                    f"I {cfg.I})" + (f", Zipf({cfg.zipf_s})-offset router" if cfg.zipf_s else ""),
        "value": T / (ms_pass / 1000.0), "unit": "tok/s", "ms_per_pass": ms_pass, "passes": passes,
        "warm": {"value": T / (ms_pass / 1000.0), "ms_per_pass": ms_pass, "passes": passes, "clocks": clock_summary(win),
                 "note": "after two untimed passes; weights and inputs partly L2-resident between passes"},
        "cold": {"value": T / (ms_cold / 1000.0), "ms_per_pass": ms_cold, "clocks": clock_summary(win_cold),
                 "note": "first pass after the weights were uploaded, L2 flushed by a 512 MB device write; "
                         "includes first-call costs (lazy module loading, tensor-map encoding)"},
        "gpu_launches_per_pass": per_layer * cfg.layers, "stack_build_s": build_s,
        "expert_forward": {"ms_per_layer": ms_ef, "algorithmic_tflop_per_layer": flops / 1e12,
                           "touched_experts": touched,
                           "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                                        "frac": achieved / peak, "peak_kind": peak_kind,
                                        "scope": "every kernel of one layer's moe_expert_forward (the two grouped "
                                                 "GEMMs dominate), timed alone",
                                        "traffic": None,
                                        "traffic_note": "DRAM bytes are captured per launch of the gate/up grouped "
                                                        "GEMM (ncu, 3,328 tokens); this roofline spans every kernel "
                                                        "of the layer, so no whole-layer traffic is given"}},
    }


def decode_leg(dev, M, cfg_id: int, steps: int):
    """Batch-1 decode of another stack shape (per token: all layers, one launch when eligible)."""
    import torch
    cfg = CONFIGS[cfg_id]
    stack = M.DeviceStack(cfg, lambda l: inputs.layer(cfg, l), device=dev)
    st = M.StackStructs(stack)
    ws = M.workspace(M.moe_stack_workspace_size(st, 1, cfg.K, cfg.K), device=dev)
    xs = torch.from_numpy(np.stack([inputs.bf16_bits_to_f32(inputs.activations(cfg, step=1 + i, T=1))
                                    for i in range(N_TOKENS)])).to(dev)
    x = torch.empty((1, cfg.H), device=dev)
    err = torch.zeros((1,), dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        x.copy_(xs[i % N_TOKENS])
        M.moe_stack_decode(st, x, cfg.K, cfg.K, EPS, ws, err_word=err)

    for i in range(10):
        step(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed():
        e0.record(stream)
        for i in range(steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)

    _, win = timed_window(timed)
    if int(err.item()) != 0:
        raise RuntimeError(f"device-side wait timed out (status {int(err.item())})")
    ms = e0.elapsed_time(e1) / steps
    del stack, st, ws
    torch.cuda.empty_cache()
    peak, kind = peaks()
    bytes_tok = token_layer_bytes(cfg) * cfg.layers
    gbs = bytes_tok / (ms / 1000.0) / 1e9
    return {"workload": f"{cfg.name}: {cfg.layers} layers, {cfg.E} experts, top-{cfg.K}, H {cfg.H}, I {cfg.I}, batch 1",
            "value": 1000.0 / ms, "unit": "tok/s", "ms_per_token": ms, "steps": steps, "clocks": clock_summary(win),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "peak_kind": kind, "algorithmic_bytes_per_token": bytes_tok}}


def batched_decode_leg(dev, M, steps: int = 20):
    """35B-shaped batched decode: 64 tokens per step, layers >= 1 executing the previous head's prediction,
    LoRA on every routed down projection.  Reports tok/s, the bytes of the experts actually touched per step
    over the step time, and the Prerouter hit rate (|pred_{l-1} & true_l| / K)."""
    import torch
    cfg = CONFIGS[BATCHED_CFG_ID]
    T, K = cfg.T, cfg.K
    stack = M.DeviceStack(cfg, lambda l: inputs.layer(cfg, l), device=dev)
    st = M.StackStructs(stack)
    ws = M.workspace(M.moe_stack_workspace_size(st, T, K, K), device=dev)
    x0 = torch.from_numpy(inputs.bf16_bits_to_f32(inputs.activations(cfg, step=5, T=T))).to(dev)
    x = torch.empty_like(x0)
    err = torch.zeros((1,), dtype=torch.int32, device=dev)
    n = cfg.layers
    idx_all = torch.full((n, T, K), -1, dtype=torch.int32, device=dev)
    true_all = torch.full((n, T, K), -1, dtype=torch.int32, device=dev)
    pred_all = torch.full((n, T, K), -1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(trace):
        x.copy_(x0)
        kw = dict(idx_all=idx_all, true_idx_all=true_all, pred_all=pred_all) if trace else {}
        M.moe_stack_decode(st, x, K, K, EPS, ws, use_predicted_routing=True, err_word=err, **kw)

    step(True)
    torch.cuda.synchronize(dev)
    idx_h, true_h, pred_h = idx_all.cpu().numpy(), true_all.cpu().numpy(), pred_all.cpu().numpy()
    for _ in range(3):
        step(False)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed():
        e0.record(stream)
        for _ in range(steps):
            step(False)
        e1.record(stream)
        torch.cuda.synchronize(dev)

    _, win = timed_window(timed)
    if int(err.item()) != 0:
        raise RuntimeError(f"device-side wait timed out (status {int(err.item())})")
    ms = e0.elapsed_time(e1) / steps
    del stack, st, ws
    torch.cuda.empty_cache()
    hits = [np.mean([len(set(pred_h[l - 1, t]) & set(true_h[l, t])) / K for t in range(T)]) for l in range(1, n)]
    touched = [len(np.unique(idx_h[l])) for l in range(n)]
    mat = lambda out, inp: out * (inp // 2 + 4 * (inp // 64))
    blk = mat(2 * cfg.I, cfg.H) + mat(cfg.H, cfg.I)
    down_lora = cfg.r * cfg.I * 2 + cfg.H * cfg.r * 2
    per_layer_fixed = token_layer_bytes(cfg) - K * blk  # shared expert, its LoRA, router, gate, Prerouter
    step_bytes = sum(t * (blk + down_lora) for t in touched) + n * per_layer_fixed
    peak, kind = peaks()
    gbs = step_bytes / (ms / 1000.0) / 1e9
    return {"workload": "35B-shaped batched decode: 64 tokens per step, 40 layers, predicted routing for layers >= 1, "
                        "LoRA r16 on every routed down projection",
            "value": T / (ms / 1000.0), "unit": "tok/s", "ms_per_step": ms, "steps": steps, "clocks": clock_summary(win),
            "touched_experts_per_layer": float(np.mean(touched)), "prerouter_hit_rate": float(np.mean(hits)),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "peak_kind": kind, "bytes_per_step": step_bytes,
                         "scope": "whole step; bytes = experts touched (with their down LoRA) + per-layer fixed weights"}}


def tiered_leg(dev, M, n_layers: int = 8, n_slots: int = 32, warm_tokens: int = 16, tokens: int = 48):
    """35B-shaped batch-1 decode over the first n_layers layers (Zipf-offset router), each layer's routed experts
    in pinned host memory behind an HBM cache of n_slots expert blocks (moe_tier_*): per-layer launches and one
    host read of the routing per layer.  Four modes on the same tokens, each with fresh caches warmed by
    warm_tokens tokens: every expert resident in HBM; tiered (copies on demand); tiered with Prerouter prefetch
    (layer l's head predicts layer l+1's experts, copied on a side stream as soon as the prediction is read);
    tiered with ideal prefetch (the next layer's true experts, recorded in the resident pass, issued when a
    layer starts) -- the bound for a perfect predictor.  ``cold_ms_per_token`` times the warm-up tokens, the
    first through empty caches."""
    import dataclasses
    import torch
    cfg = dataclasses.replace(CONFIGS[PREFILL_CFG_ID], T=1)
    K, H = cfg.K, cfg.H
    hosts = [inputs.layer(cfg, l) for l in range(n_layers)]
    full = [M.DeviceLayer(cfg, h, device=dev) for h in hosts]
    heads = [M.DeviceHead(cfg, h["prerouter"], device=dev) for h in hosts]
    stride = M.block_stride(cfg.H, cfg.I)
    lean = [M.DeviceLayer(cfg, dict(h, experts={}), device=dev, pool=torch.zeros(stride, dtype=torch.uint8, device=dev))
            for h in hosts]
    pools = [M.host_pool(cfg, h["experts"]) for h in hosts]
    del hosts
    n_tok = warm_tokens + tokens
    xs = torch.from_numpy(np.stack([inputs.bf16_bits_to_f32(inputs.activations(cfg, step=5000 + i, T=1))
                                    for i in range(n_tok)])).to(dev)
    x = torch.empty((1, H), device=dev)
    u = torch.empty((1, H), dtype=torch.int16, device=dev)
    logits = torch.empty((1, cfg.E), device=dev)
    idx = torch.empty((1, K), dtype=torch.int32, device=dev)
    idx_slot = torch.empty_like(idx)
    w = torch.empty((1, K), device=dev)
    pred = torch.empty((1, K), dtype=torch.int32, device=dev)
    scores = torch.empty((1, cfg.E_next), device=dev)
    pws = M.workspace(M.prerouter_workspace_size(heads[0], 1), device=dev)
    ws = M.workspace(M.moe_workspace_size(full[0], 1, K), device=dev)
    side = torch.cuda.Stream(device=dev)
    stream = torch.cuda.current_stream(dev)
    recorded = np.zeros((n_tok, n_layers, K), np.int32)

    def token(i, mode, tiers):
        x.copy_(xs[i])
        for l in range(n_layers):
            if mode == "ideal" and l + 1 < n_layers:
                tiers[l + 1].prefetch(recorded[i, l + 1], stream=side)
            M.moe_rmsnorm_bf16(x, EPS, u)
            M.moe_route_topk(full[l], u, K, logits, idx, w)
            idx_h = idx.cpu().numpy()  # the host reads the routing (one sync per layer)
            if mode == "resident":
                recorded[i, l] = idx_h[0]
                M.moe_expert_forward(full[l], u, K, idx, w, x, 2, ws)
            else:
                tiers[l].acquire(idx_h, idx, idx_slot)
                M.moe_expert_forward(tiers[l], u, K, idx_slot, w, x, 2, tws)
                tiers[l].release()
            M.prerouter_predict(heads[l], u, idx, K, pred, scores, pws)
            if mode == "prerouter" and l + 1 < n_layers:
                tiers[l + 1].prefetch(pred.cpu().numpy(), stream=side)

    out = {"workload": f"{cfg.name} shapes, batch-1 decode over the first {n_layers} layers (Zipf-offset router), "
                       f"routed experts in pinned host memory behind {n_slots} HBM slots per layer "
                       f"({n_slots / cfg.E:.0%} of the experts); per-layer launches, one host read of the routing "
                       "per layer",
           "n_slots": n_slots, "tokens": tokens, "warm_tokens": warm_tokens, "modes": {}}
    tws = None
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    bb = M.block_bytes(cfg.H, cfg.I)
    for mode in ("resident", "tiered", "prerouter", "ideal"):
        tiers = None
        if mode != "resident":
            tiers = [M.TieredPool(lean[l], pools[l], n_slots) for l in range(n_layers)]
            tws = M.workspace(M.moe_workspace_size(tiers[0], 1, K), device=dev)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for i in range(warm_tokens):  # cold: the first tokens through empty caches
            token(i, mode, tiers)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_cold = e0.elapsed_time(e1) / warm_tokens
        before = [t.stats() for t in tiers] if tiers else None

        def timed():
            e0.record(stream)
            for i in range(warm_tokens, n_tok):
                token(i, mode, tiers)
            e1.record(stream)
            torch.cuda.synchronize(dev)

        _, win = timed_window(timed)
        ms = e0.elapsed_time(e1) / tokens
        r = {"ms_per_token": ms, "value": 1000.0 / ms, "unit": "tok/s", "clocks": clock_summary(win),
             "cold_ms_per_token": ms_cold}
        if tiers:
            d = {k: sum(t.stats()[k] - b[k] for t, b in zip(tiers, before)) for k in before[0]}
            r.update({"hit_rate": d["hits"] / max(d["requested"], 1),
                      "prefetch_hit_rate": d["prefetch_hits"] / max(d["requested"], 1),
                      "mb_copied_per_token": (d["bytes_acquired"] + d["bytes_prefetched"]) / tokens / 1e6,
                      "mb_on_demand_per_token": d["bytes_acquired"] / tokens / 1e6,
                      "experts_per_layer_call": d["requested"] / (tokens * n_layers), "block_bytes": bb})
            for t in tiers:
                t.close()
        out["modes"][mode] = r
    return out


def launches_per_step(cfg, single: bool, predicted=False) -> int:
    if single:
        return 1  # the whole stack is one cooperative launch (plus two cudaMemsetAsync, not kernels)
    per_layer = 1 + 2 + 1 + 1 + 1 + 1 + 3  # rmsnorm, router+topk, pre, gate/up, lora-mid, down, prerouter x3
    return cfg.layers * per_layer + (cfg.layers - 1 if predicted else 0)


def headline_line(cfg, world: int, steps: int, warmup: int, ms: float, value: float, e2e_value: float,
                  single: bool, clocks: dict) -> dict:
    """The JSON line of the decode headline from the measured numbers.

    ``ms`` is the max-over-ranks device time of the ``steps`` timed steps and
    ``value`` the whole-job rate from it; the roofline numerator is the
    algorithmic bytes of one step (one stack launch on the single-launch path)
    over the mean step time.
    """
    T = cfg.T
    peak, peak_kind = peaks()
    bytes_step = token_layer_bytes(cfg) * cfg.layers * T
    achieved = bytes_step / (ms / steps / 1000.0) / 1e9
    return {
        "metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": ms / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**decode_config(cfg, world),
                   "l2": "inputs larger than L2: 433 MB of weights read per step, a distinct token per step",
                   "path": "moe_stack_decode, " + ("one cooperative launch per token" if single
                                                     else "per-layer launches")},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": measured_traffic(cfg.layers) if single else None, "peak_kind": peak_kind,
                     "scope": "stack kernel (the whole step)" if single else "whole step (all launches)",
                     "algorithmic_bytes_per_step": bytes_step},
        "e2e": {"value": e2e_value, "unit": "tok/s", "h2d_bytes_per_step": T * cfg.H * 4,
                "d2h_bytes_per_step": T * cfg.H * 4},
        "gpu_launches": launches_per_step(cfg, single) * steps,
        "clocks": clocks,
    }


def smi_gpu_id(local: int) -> str:
    """nvidia-smi ``--id`` of this process's CUDA device ``local``.

    CUDA_VISIBLE_DEVICES renumbers devices for CUDA but not for nvidia-smi, so
    its ``local``-th entry (an index or a GPU UUID) names the GPU; without it
    the CUDA index is the nvidia-smi index.
    """
    vis = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    return vis[local] if local < len(vis) else str(local)


class Clocks:
    """SM clock and throttle-reason samples, read-only, from NVML every 5 ms in a thread (nvidia-smi as the
    fallback), plus one sample at each edge of a timed window; ``summary(window)`` gives a window's median SM
    clock, the maximum clock and the reasons seen.  Started before the warm-up and kept for every leg."""

    REASONS = (("hw_slowdown", "nvmlClocksThrottleReasonHwSlowdown", 0x8),
               ("hw_thermal_slowdown", "nvmlClocksThrottleReasonHwThermalSlowdown", 0x40),
               ("sw_thermal_slowdown", "nvmlClocksThrottleReasonSwThermalSlowdown", 0x20),
               ("sw_power_cap", "nvmlClocksThrottleReasonSwPowerCap", 0x4))

    def __init__(self, dev):
        self.dev = dev
        self.samples = []  # (time, sm MHz, reason names)
        self.max_mhz = None
        self.nv = None
        self.handle = None
        self.thread = None
        self.stop_flag = False
        self.source = None

    def _read(self):
        nv = self.nv
        try:
            sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
            get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            bits = get(self.handle)
        except Exception:
            return
        names = tuple(n for n, attr, dflt in self.REASONS if bits & getattr(nv, attr, dflt))
        self.samples.append((time.time(), float(sm), names))

    def start(self):
        import threading
        try:
            import pynvml as nv
            import torch
            nv.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.dev).uuid)
            self.handle = nv.nvmlDeviceGetHandleByUUID(uuid)
            self.nv = nv
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM))
            self.source = "nvml"
        except Exception:
            self.nv = None
        if self.nv is not None:
            def loop():
                while not self.stop_flag:
                    self._read()
                    time.sleep(0.005)
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
        else:
            self._start_smi()
        return self

    def _start_smi(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={smi_gpu_id(self.dev.index or 0)}",
                                          "--query-gpu=timestamp,clocks.sm,clocks.max.sm,"
                                          "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                                          "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True, bufsize=1)
            self.source = "nvidia-smi"
        except Exception:
            self.proc = None

    def edge(self):
        """One sample now (the edges of a timed window)."""
        if self.nv is not None:
            self._read()

    def stop(self):
        self.stop_flag = True
        if self.thread is not None:
            self.thread.join(timeout=1)
        proc = getattr(self, "proc", None)
        if proc is not None:
            import datetime
            proc.terminate()
            try:
                out, _ = proc.communicate(timeout=5)
            except Exception:
                proc.kill()
                out, _ = proc.communicate()
            for l in out.splitlines():
                f = [x.strip() for x in l.split(",")]
                try:
                    ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    names = tuple(n for (n, _, _), v in zip(self.REASONS, f[3:7]) if v.lower() == "active")
                    self.samples.append((ts, float(f[1]), names))
                    self.max_mhz = float(f[2])
                except (ValueError, IndexError):
                    continue

    def summary(self, window):
        t0, t1 = window
        sel = [x for x in self.samples if t0 - 0.002 <= x[0] <= t1 + 0.002]
        sm = [x[1] for x in sel]
        reasons = sorted({n for x in sel for n in x[2]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(sm), "source": self.source}


CLK = None  # the bench's clock sampler (set in main)


def timed_window(fn):
    """Run fn() between two clock edge samples; returns (fn's result, the wall-clock window)."""
    if CLK is not None:
        CLK.edge()
    t0 = time.time()
    r = fn()
    t1 = time.time()
    if CLK is not None:
        CLK.edge()
    return r, (t0, t1)


def clock_summary(window):
    return CLK.summary(window) if CLK is not None else None


def measured_traffic(layers: int):
    """DRAM bytes per stack-kernel launch from the committed ncu record, or None if the kernel changed since."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "stack_decode_traffic.json")))
        src = b"".join(open(os.path.join(ROOT, f), "rb").read() for f in rec["source_files"])
        if hashlib.sha256(src).hexdigest() != rec["source_sha256"]:
            return None
        return (rec["dram_bytes_read"] + rec["dram_bytes_write"]) * layers / rec["captured_layers"]
    except Exception:
        return None


class OracleTokenPass:
    """Batch-1 tokens through the stack on the float64 oracle, one work item at a time.

    A layer is K + 3 items, taken in the order of the oracle's own layer pass:
    ``route`` (layer input, router logits, top-K, gating weights), ``expert``
    once per routed slot, ``shared`` (shared expert and its sigmoid gate) and
    ``tail`` (weighted combine, residual add, Prerouter prediction).  Every item
    calls the oracle's functions as they stand; ``step`` returns the item's kind
    and its seconds of oracle work.  Inputs are drawn outside the clock: each
    layer's router, shared expert and Prerouter once (then kept), and per layer
    only the experts the token is routed to.  After the last layer the next
    token (a new seeded activation) starts at layer 0.
    """

    KINDS = ("route", "expert", "shared", "tail")

    def __init__(self, cfg, eps: float = EPS):
        from oracle import moe_oracle as O
        self.O, self.cfg, self.eps = O, cfg, eps
        self.static = {}
        self.token, self.layer, self.i = 0, 0, 0
        self.finished = []  # residual streams of completed tokens
        self._new_token()

    def _new_token(self):
        self.x = inputs.bf16_bits_to_f32(inputs.activations(self.cfg, step=self.token, T=1)).astype(np.float64)

    def _layer_static(self, l: int):
        if l not in self.static:
            self.static[l] = (inputs.router(self.cfg, l), inputs.shared(self.cfg, l), inputs.prerouter(self.cfg, l))
        return self.static[l]

    def step(self) -> tuple[str, float]:
        O, cfg, K = self.O, self.cfg, self.cfg.K
        R, S, P = self._layer_static(self.layer)
        i = self.i
        if i == 0:
            kind, t0 = "route", time.perf_counter()
            self.u = O.layer_input(self.x, self.eps)
            logits = O.router_logits(self.u, R)
            self.idx = O.topk(logits, K)
            self.w = O.gating(logits, self.idx)
            dt = time.perf_counter() - t0
            self.experts = {int(e): inputs.expert(cfg, self.layer, int(e)) for e in self.idx[0]}
            self.y = np.zeros((1, K, cfg.H), dtype=np.float64)
        elif i <= K:
            kind, t0 = "expert", time.perf_counter()
            self.y[:, i - 1] = O.routed_outputs(self.u, self.experts, self.idx[:, i - 1:i])[:, 0]
            dt = time.perf_counter() - t0
        elif i == K + 1:
            kind, t0 = "shared", time.perf_counter()
            self.ys = O.shared_expert(self.u, S)
            self.g = O.shared_gate(self.u, S)
            dt = time.perf_counter() - t0
        else:
            kind, t0 = "tail", time.perf_counter()
            self.x = self.x + O.combine(self.w, self.y, self.g, self.ys)
            self.pred = O.prerouter_predict(self.u, self.idx, P, cfg.E, K)[0]
            dt = time.perf_counter() - t0
        self.i += 1
        if self.i == K + 3:
            self.i, self.layer = 0, self.layer + 1
            if self.layer == cfg.layers:
                self.finished.append(self.x)
                self.token, self.layer = self.token + 1, 0
                self._new_token()
        return kind, dt


def oracle_token_seconds(items, cfg) -> float:
    """Oracle seconds per token from timed items: per-kind means times the items of a token.

    With every kind sampled a token costs ``layers * (t_route + K t_expert +
    t_shared + t_tail)``; otherwise the plain item rate is scaled by the
    ``layers * (K + 3)`` items of a token.
    """
    per_layer = {"route": 1, "expert": cfg.K, "shared": 1, "tail": 1}
    by = {k: [t for kind, t in items if kind == k] for k in per_layer}
    if all(by.values()):
        return cfg.layers * sum(n * statistics.fmean(by[k]) for k, n in per_layer.items())
    return sum(t for _, t in items) * cfg.layers * (cfg.K + 3) / len(items)


def blas_threads() -> int:
    """Threads of the host BLAS pool the oracle's matmuls run on (the largest pool if several)."""
    from threadpoolctl import threadpool_info
    return max((p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"), default=1)


def _oracle_layers(cfg, budget_s: float):
    ref = OracleTokenPass(cfg)
    items = []
    while not items or ref.i != 0 or sum(t for _, t in items) < budget_s:
        items.append(ref.step())
    return items


def cpu_baseline(cfg, budget_s: float = 20.0, one_thread_budget_s: float = 10.0):
    """The float64 oracle on the host: whole layers of batch-1 tokens until each time budget is spent.

    The headline figure uses every BLAS thread of the process; a second sample
    with the BLAS pool limited to one thread is reported beside it.
    """
    from threadpoolctl import threadpool_limits
    cores = blas_threads()
    items = _oracle_layers(cfg, budget_s)
    out = {"value": 1.0 / oracle_token_seconds(items, cfg), "unit": "tok/s", "cores": cores, "kind": "oracle",
           "sample": f"{len(items) // (cfg.K + 3)} layer passes of batch-1 tokens through the 35B-shaped stack "
                     f"(float64 numpy, BLAS threads = {cores}), seconds per token = {cfg.layers} x one layer's items"}
    if one_thread_budget_s > 0:
        with threadpool_limits(limits=1, user_api="blas"):
            one = _oracle_layers(cfg, one_thread_budget_s)
        out["one_thread"] = {"value": 1.0 / oracle_token_seconds(one, cfg), "unit": "tok/s", "cores": 1,
                             "sample": f"{len(one) // (cfg.K + 3)} layer passes, BLAS threads = 1"}
    return out


def decode_config(cfg, world: int) -> dict:
    return {"workload": "35B-shaped MoE stack decode, batch 1 (40 layers, 256 experts, top-4, H 2048, "
                        "I 512, shared expert I 512 + LoRA r16, Prerouter P 256)",
            "tokens_per_step": cfg.T, "layers": cfg.layers, "parallelism": f"replicas x{world}"}


def run_reference(args, rank, world):
    """The oracle timed on the host cores (rank 0 only): each step is one oracle work item."""
    if rank != 0:
        return
    cfg = CONFIGS[CFG_ID]
    ref = OracleTokenPass(cfg)
    for _ in range(args.warmup):
        ref.step()
    items = [ref.step() for _ in range(args.steps)]
    v = 1.0 / oracle_token_seconds(items, cfg)
    cores = blas_threads()
    sample = (f"{args.steps} oracle work items (route / one routed expert / shared expert / combine + Prerouter; "
              f"{cfg.K + 3} per layer, {cfg.layers} layers per token) of batch-1 tokens, after {args.warmup} "
              f"warm-up items; float64 numpy, BLAS threads = {cores}")
    config = decode_config(cfg, world)
    config["step"] = "one oracle work item of a token's pass (a bounded sample of the decode step)"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tok/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * sum(t for _, t in items) / len(items),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config,
        "cpu_baseline": {"value": v, "unit": "tok/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# Stamp slots of moe_stack_opts.trace written by the single-launch kernel (see include/moe.h), and the
# spans between them that --diag-stack --trace reports.
TRACE_SPANS = [(0, 1, "A: x received -> RMSNorm done, layer weights landed"),
               (1, 2, "A: router / shared-gate / LoRA-A rows published"),
               (2, 3, "A: shared (gate, up) dots + Prerouter u part (during the logits hop)"),
               (3, 4, "A->B: rest of the logits hop"),
               (4, 5, "B: top-K (every warp)"),
               (5, 6, "B: routed copies issued"),
               (6, 15, "B: copies issued -> first routed rows landed"),
               (6, 7, "B: (gate, up) pairs done"),
               (7, 8, "B: hidden published + previous head's output rows (during the hidden hop)"),
               (8, 9, "B->C: rest of the hidden-vector hop"),
               (9, 10, "C: hidden vector to pair order, sums, LoRA A, down rows landed"),
               (10, 11, "C: down sub-rows"),
               (11, 12, "C: combine, x rows published")]


def _span_stats(v) -> str:
    return (f"mean {v.mean():8.2f}  p90 {np.percentile(v, 90):8.2f}  max {v.max():8.2f}" if v.size
            else "(not recorded)")


def diag_stack(args):
    """Diagnostic run of the batch-1 stack (no JSON line): the first --layers layers of the 35B shape (or
    --cfg), --runs tokens on --path; with --trace, per-phase times from the kernel's %globaltimer stamps."""
    import torch
    import int4_expert_ffn_top_b200 as M
    cfg = CONFIGS[args.cfg]
    stack = M.DeviceStack(cfg, lambda l: inputs.layer(cfg, l), n_layers=args.layers)
    st = M.StackStructs(stack)
    ws = M.workspace(M.moe_stack_workspace_size(st, 1, cfg.K, cfg.K))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    toks = [torch.from_numpy(inputs.bf16_bits_to_f32(inputs.activations(cfg, step=1 + i, T=1))).cuda() for i in range(8)]
    x = torch.empty_like(toks[0])
    trace = torch.zeros((stack.n, M.moe_stack_grid(), 16), dtype=torch.int64, device="cuda") if args.trace else None
    opts = M.stack_opts(path=args.path, trace=trace)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.runs):
        x.copy_(toks[i % len(toks)])
        M.moe_stack_decode(st, x, cfg.K, cfg.K, EPS, ws, err_word=err, opts=opts)
    e1.record()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise SystemExit(f"moe_stack_decode reported status {int(err.item())}")
    print(f"{cfg.name}, {stack.n} layers, path {args.path}: {args.runs} tokens, "
          f"{e0.elapsed_time(e1) / args.runs:.3f} ms per token" + (" (with tracing)" if args.trace else ""))
    if not args.trace:
        return
    raw = trace.cpu().numpy()
    ok = raw != 0
    tr = (raw.astype(np.float64) - raw[ok].min()) / 1000.0  # us
    print("per span, us (mean / p90 / max over CTAs, layers 1..n-1):")
    for i, j, name in TRACE_SPANS:
        m = ok[1:, :, i] & ok[1:, :, j]
        print(f"  {name:78s} {_span_stats((tr[1:, :, j] - tr[1:, :, i])[m])}")
    m = ok[1:, :, 0] & ok[:-1, :, 12]
    print(f"  {'C->A: residual hop (own x rows published -> next layer x received)':78s} "
          f"{_span_stats((tr[1:, :, 0] - tr[:-1, :, 12])[m])}")
    period = np.diff(tr[:, :, 12].max(axis=1))
    print(f"layer period (latest CTA's x rows published), us: mean {period.mean():.2f}")


def diag_expert(args):
    """Diagnostic run of one layer's moe_expert_forward (no JSON line): layer 1 of --cfg (default: the 35B-shaped
    prefill, Zipf-offset router) on --tokens tokens, routed on the GPU, --runs calls; for profilers."""
    import torch
    import int4_expert_ffn_top_b200 as M
    cfg = CONFIGS[args.cfg if args.cfg != CFG_ID else PREFILL_CFG_ID]
    T, K = args.tokens, cfg.K
    lay = M.DeviceLayer(cfg, inputs.layer(cfg, 1))
    u = torch.from_numpy(inputs.activations(cfg, step=9, T=T).view(np.int16)).cuda()
    logits = torch.empty((T, cfg.E), device="cuda")
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_route_topk(lay, u, K, logits, idx, w, err_word=err)
    out = torch.empty((T, cfg.H), device="cuda")
    ws = M.workspace(M.moe_workspace_size(lay, T, K))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.runs):
        M.moe_expert_forward(lay, u, K, idx, w, out, 0, ws, err_word=err)
    e1.record()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise SystemExit(f"moe_expert_forward reported status {int(err.item())}")
    ms = e0.elapsed_time(e1) / args.runs
    print(f"{cfg.name}, one layer's expert forward at {T} tokens: {ms:.3f} ms per call "
          f"({expert_flops(cfg, T) / (ms / 1000.0) / 1e12:.1f} TFLOP/s)")


def diag_route(args):
    """Diagnostic run of one layer's router + top-K and Prerouter (no JSON line): layer 1 of --cfg (default: the
    35B-shaped prefill) on --tokens tokens, --runs calls of each; for profilers."""
    import torch
    import int4_expert_ffn_top_b200 as M
    cfg = CONFIGS[args.cfg if args.cfg != CFG_ID else PREFILL_CFG_ID]
    T, K = args.tokens, cfg.K
    host = inputs.layer(cfg, 1, experts=[])
    lay = M.DeviceLayer(cfg, host)
    head = M.DeviceHead(cfg, host["prerouter"])
    u = torch.from_numpy(inputs.activations(cfg, step=9, T=T).view(np.int16)).cuda()
    logits = torch.empty((T, cfg.E), device="cuda")
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), device="cuda")
    pred = torch.empty((T, K), dtype=torch.int32, device="cuda")
    scores = torch.empty((T, cfg.E), device="cuda")
    pws = M.workspace(M.prerouter_workspace_size(head, T))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    M.moe_route_topk(lay, u, K, logits, idx, w, err_word=err)
    M.prerouter_predict(head, u, idx, K, pred, scores, pws, err_word=err)
    e0.record()
    for _ in range(args.runs):
        M.moe_route_topk(lay, u, K, logits, idx, w, err_word=err)
    e1.record()
    for _ in range(args.runs):
        M.prerouter_predict(head, u, idx, K, pred, scores, pws, err_word=err)
    e2.record()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise SystemExit(f"status {int(err.item())}")
    ms_r, ms_p = e0.elapsed_time(e1) / args.runs, e1.elapsed_time(e2) / args.runs
    fr = 2.0 * T * cfg.H * cfg.E
    fp = 2.0 * T * ((cfg.H + cfg.E) * cfg.P + cfg.P * cfg.E_next)
    print(f"{cfg.name}, {T} tokens: router + top-K {ms_r * 1e3:.1f} us ({fr / (ms_r / 1e3) / 1e12:.1f} TFLOP/s), "
          f"Prerouter {ms_p * 1e3:.1f} us ({fp / (ms_p / 1e3) / 1e12:.1f} TFLOP/s)")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the 3,328-token prefill leg")
    ap.add_argument("--no-extra", action="store_true", help="skip the 8B-shaped and batched decode legs")
    ap.add_argument("--path", type=int, default=0, help="0 auto, 1 per-layer launches, 2 single launch")
    ap.add_argument("--diag-stack", action="store_true",
                    help="diagnostic batch-1 stack run (for profilers and the phase trace); prints no JSON line")
    ap.add_argument("--cfg", type=int, default=CFG_ID, help="--diag-stack: workload shape (gen.configs index)")
    ap.add_argument("--layers", type=int, default=None, help="--diag-stack: first N layers (default: all)")
    ap.add_argument("--runs", type=int, default=4, help="--diag-stack: tokens run through the stack")
    ap.add_argument("--trace", action="store_true", help="--diag-stack: print per-phase times")
    ap.add_argument("--diag-expert", action="store_true",
                    help="diagnostic run of one layer's expert forward (for profilers); prints no JSON line")
    ap.add_argument("--diag-route", action="store_true",
                    help="diagnostic run of one layer's router + top-K and Prerouter; prints no JSON line")
    ap.add_argument("--tokens", type=int, default=3328, help="--diag-expert / --diag-route: tokens per call")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.diag_stack:
        return diag_stack(args)
    if args.diag_expert:
        return diag_expert(args)
    if args.diag_route:
        return diag_route(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import int4_expert_ffn_top_b200 as M

    torch.cuda.set_device(local)
    if dist is not None:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    cfg = CONFIGS[CFG_ID]
    stack = M.DeviceStack(cfg, lambda l: inputs.layer(cfg, l), device=dev)
    st = M.StackStructs(stack)
    T = cfg.T
    ws = M.workspace(M.moe_stack_workspace_size(st, T, cfg.K, cfg.K), device=dev)
    toks = np.stack([inputs.bf16_bits_to_f32(inputs.activations(cfg, step=1 + rank * N_TOKENS + i, T=T))
                     for i in range(N_TOKENS)])
    xpool = torch.from_numpy(toks).to(dev)
    x = torch.empty((T, cfg.H), device=dev)
    stream = torch.cuda.current_stream(dev)

    opts = M.stack_opts(path=args.path)
    err = torch.zeros((1,), dtype=torch.int32, device=dev)
    single = args.path != 1 and T == 1

    def step(i):
        x.copy_(xpool[i % N_TOKENS])
        M.moe_stack_decode(st, x, cfg.K, cfg.K, EPS, ws, err_word=err, opts=opts)

    global CLK
    CLK = Clocks(dev).start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed_run():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for i in range(args.steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1)

    # two timed runs of exactly --steps steps each; the line reports both and their median
    runs, wins = [], []
    for _ in range(2):
        ms_r, win = timed_window(timed_run)
        runs.append(max_over_ranks(ms_r, dist, dev))
        wins.append(win)
    if int(err.item()) != 0:
        raise RuntimeError(f"device-side wait timed out (status {int(err.item())})")
    if dist is not None:
        dist.barrier()
    ms = statistics.median(runs)
    value = whole_job_rate(T * args.steps, world, ms)
    head_clocks = clock_summary((wins[0][0], wins[-1][1]))

    # end to end through the public API with host buffers: H2D of the token, D2H of the result
    xh = torch.from_numpy(toks).pin_memory()
    outh = torch.empty((T, cfg.H), dtype=torch.float32).pin_memory()
    e2e_steps = max(args.steps // 4, 10)
    for i in range(3):
        x.copy_(xh[i], non_blocking=True)
        M.moe_stack_decode(st, x, cfg.K, cfg.K, EPS, ws, err_word=err, opts=opts)
        outh.copy_(x, non_blocking=True)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    e0.record(stream)
    for i in range(e2e_steps):
        x.copy_(xh[i % N_TOKENS], non_blocking=True)
        M.moe_stack_decode(st, x, cfg.K, cfg.K, EPS, ws, err_word=err, opts=opts)
        outh.copy_(x, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_e2e = e0.elapsed_time(e1)
    ms_e2e = max_over_ranks(ms_e2e, dist, dev)
    e2e_value = whole_job_rate(T * e2e_steps, world, ms_e2e)

    out = headline_line(cfg, world, args.steps, args.warmup, ms, value, e2e_value, single, head_clocks)
    out["runs"] = [{"ms_per_step": m / args.steps, "value": whole_job_rate(T * args.steps, world, m)} for m in runs]
    if not args.no_prefill:
        del stack, st, ws, xpool
        torch.cuda.empty_cache()
        pre = prefill_leg(dev, M)
        pre["ms_per_pass"] = max_over_ranks(pre["ms_per_pass"], dist, dev)
        pre["value"] = whole_job_rate(CONFIGS[PREFILL_CFG_ID].T, world, pre["ms_per_pass"])
        out["prefill"] = pre
    if not args.no_extra:
        for key, fn in (("decode_8b", lambda: decode_leg(dev, M, DECODE_8B_CFG_ID, steps=500)),
                        ("batched_decode", lambda: batched_decode_leg(dev, M)),
                        ("prefill_8b", lambda: prefill_leg(dev, M, passes=3,
                                                           cfg=dataclasses.replace(CONFIGS[DECODE_8B_CFG_ID], T=3328,
                                                                               name="8B-shaped prefill"))),
                        ("tiered_pool", lambda: tiered_leg(dev, M))):
            try:
                leg = fn()
                ms_leg = leg.get("ms_per_token", leg.get("ms_per_step"))
                if ms_leg is None and "ms_per_pass" in leg:  # the 8B prefill leg
                    ms_leg = leg["ms_per_pass"]
                if ms_leg is None:  # the tiered-pool leg: its on-demand mode's time
                    ms_leg = leg["modes"]["tiered"]["ms_per_token"]
            except Exception as exc:  # a failing extra leg must not lose the headline line
                leg, ms_leg = {"error": f"{type(exc).__name__}: {exc}"}, -1.0
            # every rank takes this collective, on the error path too
            ms_leg = max_over_ranks(ms_leg, dist, dev)
            if "error" not in leg:
                leg["ms_max_over_ranks"] = ms_leg
            out[key] = leg
    CLK.stop()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(cfg)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
