"""Device-resident weights in the library's HBM layout.

Uploads host arrays (the storage formats of ``include/moe.h``) into torch-owned
device memory and fills the ``moe_layer`` / ``moe_prerouter`` structs with the
pointers.  Routed experts of a layer go into one pool: expert ``e`` is the
block at ``pool + e*stride`` holding gate/up codes, scales, biases, then down
codes, scales, biases (one contiguous span per expert).
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib


def qrow_bytes(in_dim: int, bits: int) -> int:
    """Bytes of one row record: codes, in/64 fp16 scales, in/64 fp16 biases, padded to 16."""
    return (in_dim * bits // 8 + 4 * (in_dim // 64) + 15) // 16 * 16


def block_bytes(H: int, I: int) -> int:
    return 2 * I * qrow_bytes(H, 4) + H * qrow_bytes(I, 4)


def block_stride(H: int, I: int) -> int:
    return (block_bytes(H, I) + 255) // 256 * 256


def qrows(m: dict) -> np.ndarray:
    """Row records ``[out, qrow_bytes]`` (uint8) of a matrix given as codes / scales / biases."""
    out = m["q"].shape[0]
    in_dim = m["q"].shape[1] * 32 // m["bits"]
    cb, G = in_dim * m["bits"] // 8, in_dim // 64
    rec = np.zeros((out, qrow_bytes(in_dim, m["bits"])), np.uint8)
    rec[:, :cb] = np.ascontiguousarray(m["q"]).view(np.uint8).reshape(out, cb)
    rec[:, cb:cb + 2 * G] = np.ascontiguousarray(m["s"]).view(np.uint8).reshape(out, 2 * G)
    rec[:, cb + 2 * G:cb + 4 * G] = np.ascontiguousarray(m["b"]).view(np.uint8).reshape(out, 2 * G)
    return rec


def expert_block(ex: dict) -> np.ndarray:
    """One expert's bytes: gate/up records interleaved (gate_0, up_0, gate_1, ...), then down records."""
    gu = qrows(ex["gate_up"])
    I = gu.shape[0] // 2
    inter = np.empty_like(gu)
    inter[0::2], inter[1::2] = gu[:I], gu[I:]
    return np.concatenate([inter.reshape(-1), qrows(ex["down"]).reshape(-1)])


def _dev(a: np.ndarray, device) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint32:
        a = a.view(np.int32)
    elif a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(device)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def host_pool(cfg, experts: dict) -> torch.Tensor:
    """The routed expert blocks of a layer in pinned host memory: uint8 ``[E, block_stride]``, expert ``e`` at
    row ``e`` (experts missing from ``experts`` stay zero)."""
    stride = block_stride(cfg.H, cfg.I)
    pool = torch.zeros((cfg.E, stride), dtype=torch.uint8).pin_memory()
    arr = pool.numpy()
    for e, ex in experts.items():
        b = expert_block(ex)
        arr[e, :b.size] = b
    return pool


class DeviceLayer:
    """One layer's tensors on the device and its ``moe_layer`` struct.

    ``host`` is a layer dict as drawn by ``gen.inputs.layer``; experts missing
    from ``host['experts']`` leave their pool blocks zero (never read unless
    routed to).  ``pool`` may be a caller-provided uint8 device tensor view of
    ``E*stride`` bytes (e.g. a slice of one stack-wide allocation).
    """

    def __init__(self, cfg, host: dict, device="cuda", pool: torch.Tensor | None = None):
        self.cfg = cfg
        H, E, I, r = cfg.H, cfg.E, cfg.I, cfg.r
        self.stride = block_stride(H, I)
        R, S = host["router"], host["shared"]
        self.t = {}
        t = self.t
        t["router"] = _dev(qrows(R), device)
        t["router_bias"] = _dev(R["beta"].astype(np.float32), device)
        t["sgate"] = _dev(qrows(S["gate"]), device)
        t["shared"] = _dev(expert_block(S), device)
        for i, p in enumerate(("gate", "up", "down")):
            lo = S.get("lora_" + p)
            t[f"A{i}"] = None if lo is None else _dev(lo["A"], device)
            t[f"B{i}"] = None if lo is None else _dev(lo["B"], device)
        if pool is None:
            pool = torch.zeros(E * self.stride, dtype=torch.uint8, device=device)
        self.pool = pool
        self.fill_experts(host["experts"])
        ex_lora = [e for e in host["experts"].values() if "down_lora" in e]
        if cfg.lora_routed_down:
            A = np.zeros((E, r, I), np.float16)
            B = np.zeros((E, H, r), np.float16)
            for e, ex in host["experts"].items():
                A[e], B[e] = ex["down_lora"]["A"], ex["down_lora"]["B"]
            t["exA"], t["exB"] = _dev(A, device), _dev(B, device)
        else:
            assert not ex_lora
            t["exA"] = t["exB"] = None
        if getattr(cfg, "lora_routed_gate_up", False):
            A = np.zeros((E, 2, r, H), np.float16)
            B = np.zeros((E, 2 * I, r), np.float16)
            for e, ex in host["experts"].items():
                A[e, 0], A[e, 1] = ex["gate_lora"]["A"], ex["up_lora"]["A"]
                B[e, 0::2], B[e, 1::2] = ex["gate_lora"]["B"], ex["up_lora"]["B"]  # the block's interleaved rows
            t["exAgu"], t["exBgu"] = _dev(A, device), _dev(B, device)
        else:
            t["exAgu"] = t["exBgu"] = None
        self.struct = self._make_struct()

    def fill_experts(self, experts: dict):
        if not experts:
            return
        stride = self.stride
        ids = sorted(experts)
        host = np.zeros((len(ids), stride), np.uint8)
        for i, e in enumerate(ids):
            b = expert_block(experts[e])
            host[i, :b.size] = b
        staged = torch.from_numpy(host).pin_memory() if torch.cuda.is_available() else torch.from_numpy(host)
        pool2 = self.pool.view(self.cfg.E, stride)
        if ids == list(range(ids[0], ids[0] + len(ids))):
            pool2[ids[0]:ids[0] + len(ids)].copy_(staged, non_blocking=True)
        else:
            for i, e in enumerate(ids):
                pool2[e].copy_(staged[i], non_blocking=True)
        torch.cuda.current_stream(self.pool.device).synchronize()

    def _make_struct(self) -> _lib.moe_layer:
        c, t = self.cfg, self.t
        L = _lib.moe_layer()
        L.H, L.E, L.I, L.I_s, L.r = c.H, c.E, c.I, c.I_s, c.r
        L.router = _lib.moe_qrows(_ptr(t["router"]), c.E, c.H, 8)
        L.router_bias = _ptr(t["router_bias"])
        L.shared_gate = _lib.moe_qrows(_ptr(t["sgate"]), 1, c.H, 8)
        L.shared_block = _ptr(t["shared"])
        for i in range(3):
            L.sh_lora_A[i] = _ptr(t[f"A{i}"])
            L.sh_lora_B[i] = _ptr(t[f"B{i}"])
        L.lora_scale = 1.0
        L.pool = self.pool.data_ptr()
        L.expert_stride = self.stride
        L.ex_lora_A, L.ex_lora_B = _ptr(t["exA"]), _ptr(t["exB"])
        L.ex_lora_A_gu, L.ex_lora_B_gu = _ptr(t["exAgu"]), _ptr(t["exBgu"])
        return L


class DeviceHead:
    """One Prerouter head on the device and its ``moe_prerouter`` struct."""

    def __init__(self, cfg, head: dict, device="cuda"):
        self.t = {k: _dev(v, device) for k, v in head.items()}
        s = _lib.moe_prerouter()
        s.W1, s.b1, s.W2, s.b2 = (self.t["W1"].data_ptr(), self.t["b1"].data_ptr(), self.t["W2"].data_ptr(),
                                  self.t["b2"].data_ptr())
        s.H, s.E, s.P, s.E_next = cfg.H, cfg.E, cfg.P, cfg.E_next
        self.struct = s


class DeviceStack:
    """All layers of a stack: one pool allocation for every routed expert of every layer.

    ``layer_fn(l)`` returns the host layer dict of layer ``l`` (storage formats of
    ``include/moe.h``); host copies are dropped after upload.
    """

    def __init__(self, cfg, layer_fn, device="cuda", n_layers: int | None = None, with_heads: bool = True):
        self.cfg = cfg
        n = n_layers or cfg.layers
        stride = block_stride(cfg.H, cfg.I)
        span = cfg.E * stride
        self.pool = torch.empty(n * span, dtype=torch.uint8, device=device)
        self.layers, self.heads = [], []
        for l in range(n):
            host = layer_fn(l)
            self.layers.append(DeviceLayer(cfg, host, device, pool=self.pool[l * span:(l + 1) * span]))
            if with_heads:
                self.heads.append(DeviceHead(cfg, host["prerouter"], device))
            del host
        self.layer_array = (_lib.moe_layer * n)(*[d.struct for d in self.layers])
        self.head_array = (_lib.moe_prerouter * n)(*[h.struct for h in self.heads]) if with_heads else None
        self.n = n
