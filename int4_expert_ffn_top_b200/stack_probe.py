"""Run the single-launch stack kernel on synthetic weights, for profilers and phase tracing.

    python -m int4_expert_ffn_top_b200.stack_probe --cfg 1 --layers 4 --runs 4   # e.g. under ncu
    python -m int4_expert_ffn_top_b200.stack_probe --cfg 1 --trace --runs 50     # per-phase timings

Builds the first ``--layers`` layers of a workload shape (all layers by
default) with the seeded synthetic weights, then runs ``moe_stack_decode`` on
the single-launch path for batch-1 tokens.  With ``--trace`` it passes a
``moe_stack_opts.trace`` buffer (%globaltimer stamps written per CTA at phase
boundaries) and prints the time between phase stamps, mean / p90 over CTAs and
layers 1..n-1, for the last traced run.  Stamps a build did not write (zero)
are left out of the statistics.
"""
from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

# Stamp slots of moe_stack_opts.trace (see include/moe.h).
PHASES = [(0, 1, "A: residual received -> router rows published"), (1, 2, "A->B: logits hop"),
          (2, 3, "B: top-K + routed copies issued"), (3, 4, "B: (gate, up) pairs -> hidden published"),
          (4, 5, "B->C: hidden-vector hop"), (5, 6, "C: down + combine -> residual published"),
          (6, 7, "C: tail (Prerouter, next layer's weight issue)")]
SUB = [(0, 8, "A: residual received -> RMSNorm done"), (8, 9, "A: RMSNorm done -> static weights landed"),
       (9, 1, "A: items"), (2, 10, "B: logits received -> top-K done"), (10, 11, "B: top-K -> barriers armed"),
       (11, 12, "B: copies issued"), (3, 13, "B: copy barrier -> first routed pair landed"),
       (5, 14, "C: hidden received -> down prologue"), (14, 15, "C: prologue -> down rows landed")]


def _stats(v: np.ndarray) -> str:
    return f"mean {v.mean():8.2f}  p90 {np.percentile(v, 90):8.2f}  max {v.max():8.2f}" if v.size else "(not recorded)"


def main(argv=None) -> None:
    import torch

    import int4_expert_ffn_top_b200 as M
    from gen import CONFIGS, inputs

    ap = argparse.ArgumentParser()
    ap.add_argument("--cfg", type=int, default=1, help="workload shape (gen.configs.CONFIGS index)")
    ap.add_argument("--layers", type=int, default=None, help="first N layers (default: all)")
    ap.add_argument("--runs", type=int, default=4, help="tokens run through the stack")
    ap.add_argument("--trace", action="store_true", help="record and print per-phase timings")
    a = ap.parse_args(argv)

    cfg = CONFIGS[a.cfg]
    stack = M.DeviceStack(cfg, lambda l: inputs.layer(cfg, l), n_layers=a.layers)
    st = M.StackStructs(stack)
    ws = M.workspace(M.moe_stack_workspace_size(st, 1, cfg.K, cfg.K))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    toks = [torch.from_numpy(inputs.bf16_bits_to_f32(inputs.activations(cfg, step=1 + i, T=1))).cuda() for i in range(8)]
    x = torch.empty_like(toks[0])
    trace = torch.zeros((stack.n, M.moe_stack_grid(), 16), dtype=torch.int64, device="cuda") if a.trace else None
    opts = M.stack_opts(path=M.PATH_SINGLE, trace=trace)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(a.runs):
        x.copy_(toks[i % len(toks)])
        M.moe_stack_decode(st, x, cfg.K, cfg.K, 1e-6, ws, err_word=err, opts=opts)
    e1.record()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise SystemExit(f"moe_stack_decode reported status {int(err.item())}")
    print(f"{cfg.name}, {stack.n} layers: {a.runs} tokens, {e0.elapsed_time(e1) / a.runs:.3f} ms per token"
          + (" (with tracing)" if a.trace else ""))
    if not a.trace:
        return
    raw = trace.cpu().numpy()
    ok = raw != 0
    tr = (raw.astype(np.float64) - raw[ok].min()) / 1000.0  # us
    print("per phase, us (mean / p90 / max over CTAs, layers 1..n-1):")
    for i, j, name in PHASES + SUB:
        m = ok[1:, :, i] & ok[1:, :, j]
        print(f"  {name:50s} {_stats((tr[1:, :, j] - tr[1:, :, i])[m])}")
    m = ok[1:, :, 0] & ok[:-1, :, 6]
    print(f"  {'C->A: residual hop (own rows published -> next layer)':50s} {_stats((tr[1:, :, 0] - tr[:-1, :, 6])[m])}")
    period = np.diff(tr[:, :, 6].max(axis=1))
    print(f"layer period (latest CTA's residual published), us: mean {period.mean():.2f}")


if __name__ == "__main__":
    main()
