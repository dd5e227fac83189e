"""Plain float64 CPU oracle of the routed-expert layer.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  It shares no code with the CUDA
library and imports nothing from it; it reads the storage formats described in
``gen.inputs`` and nothing else.

Every function is the plain definition of one step, evaluated in float64 with
library matmuls, in the order the Edge0 pages describe the layer:

* 4-bit affine quantisation with group 64 (``w = q*scale + bias``) for experts,
  8 bits for the router gate and the shared-expert gate -- 2kiu.com article
  "iPhone, Mac, Android, Windows measured: Edge0 on five platforms", bullet
  "SSD expert offload" (``group_size: 64, bits: 4``) and the closing paragraph
  on config.json (router gate and shared expert gate lifted to 8 bits).
* Router top-K over the routed experts: K=4 of 256 (35B) and K=8 of 128 (8B) --
  autoark.ai Edge0 blog, tier table; gating weights are the softmax over the K
  selected logits (the pages do not spell this out; the top-K-then-softmax
  reading equals softmax-then-renormalise in exact arithmetic).
* SwiGLU expert FFN (gate/up/down) with an unmerged LoRA delta ``B(Ax)`` added
  to a projection's output before the activation -- 2kiu.com article, bullet
  "Recover-LoRA" (adapter kept separate from the read-only base).
* Shared expert scaled by a per-token sigmoid gate.
* Weighted combine over the K experts in fixed k order.
* Prerouter: an MLP head over the hidden state and the experts executed at this
  layer, giving a top-K prediction for the next layer that is then used as the
  routing -- news18a article on Edge0 (Prerouter paragraph) and the 2kiu.com
  "Prerouter" bullet ("used directly as routing").
* Token buckets (histogram, exclusive prefix sum, stable permutation and its
  inverse) as the plain definition of grouping slots by expert.

Parity of the full layer at real shapes is pinned only by these definitions;
the pieces are pinned by closed forms, invariants and brute force in the tests.
"""
from __future__ import annotations

import numpy as np

GROUP = 64


# ----------------------------------------------------------------------------- formats
def unpack_codes(words: np.ndarray, bits: int) -> np.ndarray:
    """Codes of a packed matrix: element ``k`` of a row sits at bits ``bits*(k % (32/bits))`` of word ``k // (32/bits)``."""
    per = 32 // bits
    mask = np.uint32((1 << bits) - 1)
    shifts = (np.arange(per, dtype=np.uint32) * np.uint32(bits))
    codes = (words[..., None] >> shifts) & mask
    return codes.reshape(words.shape[0], words.shape[1] * per).astype(np.int64)


def dequant(m: dict) -> np.ndarray:
    """Affine group-64 dequantisation ``w[o,k] = q[o,k]*scale[o,k//64] + bias[o,k//64]`` in float64 (exact)."""
    q = unpack_codes(m["q"], m["bits"]).astype(np.float64)
    s = np.repeat(m["s"].astype(np.float64), GROUP, axis=1)
    b = np.repeat(m["b"].astype(np.float64), GROUP, axis=1)
    return q * s + b


def round_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (8 significant bits), ties to even; normal range only."""
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)                      # v = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)


# ----------------------------------------------------------------------------- elementwise
def sigmoid(a: np.ndarray) -> np.ndarray:
    return 0.5 * (1.0 + np.tanh(0.5 * a))


def silu(a: np.ndarray) -> np.ndarray:
    return a * sigmoid(a)


# ----------------------------------------------------------------------------- glue between stacked layers
def rmsnorm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """Weightless RMSNorm ``x / sqrt(mean(x^2) + eps)`` per token (stack glue; the pages omit attention and norms)."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def layer_input(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """``u = bf16(rmsnorm(x))``: the bf16 activations a layer consumes."""
    return round_bf16(rmsnorm(x, eps))


# ----------------------------------------------------------------------------- routing
def router_logits(u: np.ndarray, router: dict) -> np.ndarray:
    """``logits[t,e] = sum_k u[t,k] * W_r[e,k] + beta[e]`` with the 8-bit router gate dequantised."""
    W = dequant(router)
    beta = np.asarray(router.get("beta", np.zeros(W.shape[0])), dtype=np.float64)
    return np.asarray(u, dtype=np.float64) @ W.T + beta


def topk(scores: np.ndarray, K: int) -> np.ndarray:
    """Indices of the K largest scores per row, in descending order; equal scores go to the lower index."""
    T, E = scores.shape
    out = np.empty((T, K), dtype=np.int64)
    ids = np.arange(E)
    for t in range(T):
        out[t] = np.lexsort((ids, -scores[t]))[:K]
    return out


def gating(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Softmax over the selected logits: ``w_k = exp(l_k - max) / sum_j exp(l_j - max)``."""
    sel = np.take_along_axis(np.asarray(logits, dtype=np.float64), idx, axis=1)
    z = np.exp(sel - sel.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


# ----------------------------------------------------------------------------- experts
def lora_delta(x: np.ndarray, lo: dict | None) -> np.ndarray | float:
    """Unmerged LoRA delta ``scale * B (A x)`` on the projection input ``x``."""
    if lo is None:
        return 0.0
    A = lo["A"].astype(np.float64)
    B = lo["B"].astype(np.float64)
    return float(lo.get("scale", 1.0)) * ((x @ A.T) @ B.T)


def expert_ffn(u: np.ndarray, ex: dict, lora_gate=None, lora_up=None, lora_down=None) -> np.ndarray:
    """SwiGLU FFN ``W_d (silu(W_g u + dg) * (W_u u + du)) + dd`` on rows of ``u``; gate/up stacked gate-first."""
    u = np.asarray(u, dtype=np.float64)
    Wgu = dequant(ex["gate_up"])
    I = Wgu.shape[0] // 2
    a = u @ Wgu[:I].T + lora_delta(u, lora_gate)
    b = u @ Wgu[I:].T + lora_delta(u, lora_up)
    h = silu(a) * b
    return h @ dequant(ex["down"]).T + lora_delta(h, lora_down)


def expert_hidden(u: np.ndarray, ex: dict, lora_gate=None, lora_up=None) -> np.ndarray:
    """The SwiGLU hidden activations ``h`` of an expert (intermediate of :func:`expert_ffn`)."""
    u = np.asarray(u, dtype=np.float64)
    Wgu = dequant(ex["gate_up"])
    I = Wgu.shape[0] // 2
    return silu(u @ Wgu[:I].T + lora_delta(u, lora_gate)) * (u @ Wgu[I:].T + lora_delta(u, lora_up))


def shared_expert(u: np.ndarray, sh: dict) -> np.ndarray:
    return expert_ffn(u, sh, sh.get("lora_gate"), sh.get("lora_up"), sh.get("lora_down"))


def shared_gate(u: np.ndarray, sh: dict) -> np.ndarray:
    """Per-token scalar ``g = sigmoid(w_sg . u)`` with the 8-bit shared-expert gate ``[1, H]``."""
    return sigmoid(np.asarray(u, dtype=np.float64) @ dequant(sh["gate"]).T)[:, 0]


def routed_outputs(u: np.ndarray, experts: dict, idx: np.ndarray) -> np.ndarray:
    """``y[t,k] = FFN_{idx[t,k]}(u[t])`` for every slot; ``experts`` maps expert id -> tensors."""
    T, K = idx.shape
    y = np.zeros((T, K, u.shape[1]), dtype=np.float64)
    for e in np.unique(idx):
        ts, ks = np.nonzero(idx == e)
        ex = experts[int(e)]
        y[ts, ks] = expert_ffn(u[ts], ex, ex.get("gate_lora"), ex.get("up_lora"), ex.get("down_lora"))
    return y


def combine(w: np.ndarray, y: np.ndarray, g: np.ndarray, ys: np.ndarray) -> np.ndarray:
    """``out[t] = sum_{k=0}^{K-1} w[t,k] y[t,k] + g[t] ys[t]``, summed in k order."""
    out = np.zeros_like(ys)
    for k in range(w.shape[1]):
        out = out + w[:, k:k + 1] * y[:, k]
    return out + g[:, None] * ys


# ----------------------------------------------------------------------------- prerouter
def multi_hot(sel: np.ndarray, E: int) -> np.ndarray:
    T = sel.shape[0]
    m = np.zeros((T, E), dtype=np.float64)
    m[np.repeat(np.arange(T), sel.shape[1]), sel.reshape(-1)] = 1.0
    return m


def prerouter_scores(u: np.ndarray, sel: np.ndarray, head: dict, E: int) -> np.ndarray:
    """``p = W2 silu(W1 [u ; multi_hot(sel)] + b1) + b2``."""
    W1 = head["W1"].astype(np.float64)
    z = silu(np.concatenate([np.asarray(u, np.float64), multi_hot(sel, E)], axis=1) @ W1.T
             + head["b1"].astype(np.float64))
    return z @ head["W2"].astype(np.float64).T + head["b2"].astype(np.float64)


def prerouter_predict(u: np.ndarray, sel: np.ndarray, head: dict, E: int, K_next: int):
    p = prerouter_scores(u, sel, head, E)
    return topk(p, K_next), p


# ----------------------------------------------------------------------------- buckets
def buckets(idx: np.ndarray, E: int) -> dict:
    """Group the ``T*K`` slots (slot ``t*K+k``) by expert.

    ``count[e]`` slots per expert, ``offset`` its exclusive prefix sum (length E+1),
    ``perm[j]`` the slot at sorted position ``j`` (stable: ascending slot id within an
    expert) and ``inv[slot]`` its sorted position.
    """
    flat = np.asarray(idx, dtype=np.int64).reshape(-1)
    count = np.bincount(flat, minlength=E)
    offset = np.concatenate([[0], np.cumsum(count)])
    perm = np.argsort(flat, kind="stable")
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    return dict(count=count, offset=offset, perm=perm, inv=inv)


# ----------------------------------------------------------------------------- one layer / a stack
def layer_forward(u: np.ndarray, L: dict, K: int, routing: np.ndarray | None = None,
                  K_next: int | None = None) -> dict:
    """One routed-expert layer on bf16-valued inputs ``u [T,H]``.

    ``L`` holds ``router``, ``shared``, ``experts`` (id -> tensors, at least the
    ones used) and optionally ``prerouter``.  ``routing`` overrides the router's
    own top-K (predicted routing); the gating weights are always the softmax of
    this layer's logits at the executed indices.
    """
    u = np.asarray(u, dtype=np.float64)
    logits = router_logits(u, L["router"])
    true_idx = topk(logits, K)
    idx = true_idx if routing is None else np.asarray(routing, dtype=np.int64)
    w = gating(logits, idx)
    y = routed_outputs(u, L["experts"], idx)
    ys = shared_expert(u, L["shared"])
    g = shared_gate(u, L["shared"])
    out = combine(w, y, g, ys)
    res = dict(logits=logits, true_idx=true_idx, idx=idx, w=w, y=y, ys=ys, g=g, out=out)
    if "prerouter" in L:
        E = logits.shape[1]
        pred, p = prerouter_predict(u, idx, L["prerouter"], E, K_next or K)
        res.update(pred=pred, p=p)
    return res


def stack_forward(x0: np.ndarray, layers, K: int, predicted_routing: bool = False, eps: float = 1e-6) -> dict:
    """Free-running stack ``x_{l+1} = x_l + MoE_l(bf16(rmsnorm(x_l)))``; ``layers`` yields layer dicts."""
    x = np.asarray(x0, dtype=np.float64)
    trace = []
    pred = None
    for L in layers:
        u = layer_input(x, eps)
        r = layer_forward(u, L, K, routing=pred if predicted_routing else None)
        x = x + r["out"]
        pred = r.get("pred")
        trace.append(dict(u=u, idx=r["idx"], true_idx=r["true_idx"], pred=pred))
    return dict(x=x, trace=trace)
