"""B200 routed-expert layer: Python binding of libmoe.so.

The functions here have the names of the C entry points in ``include/moe.h``
and only marshal arguments (torch tensors -> device pointers, the caller's
current CUDA stream) and turn a non-zero status into ``MoEError``.  Every step
of the computation runs in the library's CUDA kernels; there is no other path.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib
from .weights import DeviceHead, DeviceLayer, DeviceStack, block_bytes, block_stride, host_pool, qrow_bytes  # noqa: F401

OUT_F32, OUT_BF16, OUT_ADD_F32 = 0, 1, 2


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {moe_status_string(code)} ({code})")
        self.code = code


def lib() -> ctypes.CDLL:
    return _lib.load()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _p(t) -> int | None:
    return None if t is None else t.data_ptr()


# Tensors that hold bf16 values may be typed bf16 or carry the bits as a 16-bit integer.
BF16_BITS = tuple(d for d in (torch.bfloat16, torch.int16, getattr(torch, "uint16", None)) if d is not None)
F32, I32, I64 = (torch.float32,), (torch.int32,), (torch.int64,)


def _arg(fn: str, name: str, t, dtypes, numel: int = 0, optional: bool = False) -> int | None:
    """Address of a tensor argument after checking it can be handed to the library.

    The library reads and writes device memory through the raw address, so a
    host tensor, a strided view, a wrong element type or a buffer smaller than
    the call touches is refused here, before any launch.
    """
    if t is None:
        if optional:
            return None
        raise ValueError(f"{fn}: {name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{fn}: {name} must be a torch.Tensor, got {type(t).__name__}")
    if t.device.type != "cuda":
        raise ValueError(f"{fn}: {name} must be a CUDA tensor, got one on {t.device}")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{fn}: {name} has dtype {t.dtype}, expected {' or '.join(str(d) for d in dtypes)}")
    if not t.is_contiguous():
        raise ValueError(f"{fn}: {name} must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{fn}: {name} holds {t.numel()} elements, the call needs {numel}")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{fn}: {name} is on {t.device}, the current device is cuda:{torch.cuda.current_device()}")
    return t.data_ptr()


def _rows(fn: str, name: str, t, width: int, dtypes) -> int:
    """Row count of a 2-D ``[T, width]`` tensor argument (checked like :func:`_arg`)."""
    if not isinstance(t, torch.Tensor) or t.dim() != 2 or t.shape[1] != width:
        shape = tuple(t.shape) if isinstance(t, torch.Tensor) else type(t).__name__
        raise ValueError(f"{fn}: {name} must be [T, {width}], got {shape}")
    _arg(fn, name, t, dtypes)
    return t.shape[0]


def _ws(fn: str, t) -> tuple[int, int]:
    """Address and byte size of a workspace tensor (its size is checked by the library)."""
    return _arg(fn, "workspace", t, None), t.numel() * t.element_size()


def _check(fn: str, code: int):
    if code != _lib.MOE_OK:
        raise MoEError(fn, code)


def moe_status_string(code: int) -> str:
    return lib().moe_status_string(code).decode()


def moe_qrow_bytes(in_dim: int, bits: int) -> int:
    return lib().moe_qrow_bytes(in_dim, bits)


def moe_expert_block_bytes(H: int, I: int) -> int:
    return lib().moe_expert_block_bytes(H, I)


def moe_rmsnorm_bf16(x: torch.Tensor, eps: float, u: torch.Tensor, stream=None):
    fn = "moe_rmsnorm_bf16"
    if not isinstance(x, torch.Tensor) or x.dim() != 2:
        raise ValueError(f"{fn}: x must be [T, H]")
    T, H = x.shape
    px, pu = _arg(fn, "x", x, F32), _arg(fn, "u", u, BF16_BITS, T * H)
    _check(fn, lib().moe_rmsnorm_bf16(px, T, H, eps, pu, _stream(stream)))


def moe_route_topk(layer: DeviceLayer, u: torch.Tensor, K: int, logits: torch.Tensor, idx: torch.Tensor,
                   w: torch.Tensor, err_word: torch.Tensor | None = None, stream=None):
    fn, L = "moe_route_topk", layer.struct
    T = _rows(fn, "u", u, L.H, BF16_BITS)
    args = (_arg(fn, "logits", logits, F32, T * L.E), _arg(fn, "idx", idx, I32, T * K), _arg(fn, "w", w, F32, T * K))
    err = _arg(fn, "err_word", err_word, I32, 1, optional=True)
    _check(fn, lib().moe_route_topk(ctypes.byref(L), _p(u), T, K, *args, err, _stream(stream)))


def moe_workspace_size(layer: DeviceLayer, T: int, K: int) -> int:
    return lib().moe_workspace_size(ctypes.byref(layer.struct), T, K)


def _expert_args(fn: str, layer: DeviceLayer, u, K: int, idx, w, out, out_mode: int, perm_out):
    L = layer.struct
    T = _rows(fn, "u", u, L.H, BF16_BITS)
    out_types = BF16_BITS if out_mode == OUT_BF16 else F32
    return T, (_arg(fn, "idx", idx, I32, T * K), _arg(fn, "w", w, F32, T * K), _arg(fn, "out", out, out_types, T * L.H),
               out_mode, _arg(fn, "perm_out", perm_out, I32, T * K, optional=True))


def moe_expert_forward(layer: DeviceLayer, u: torch.Tensor, K: int, idx: torch.Tensor, w: torch.Tensor,
                       out: torch.Tensor, out_mode: int, workspace: torch.Tensor, perm_out: torch.Tensor | None = None,
                       err_word: torch.Tensor | None = None, stream=None):
    fn = "moe_expert_forward"
    T, args = _expert_args(fn, layer, u, K, idx, w, out, out_mode, perm_out)
    err = _arg(fn, "err_word", err_word, I32, 1, optional=True)
    _check(fn, lib().moe_expert_forward(ctypes.byref(layer.struct), _p(u), T, K, *args, *_ws(fn, workspace), err,
                                        _stream(stream)))


def moe_noalloc_scratch_bytes() -> int:
    return lib().moe_noalloc_scratch_bytes()


def moe_expert_forward_noalloc(layer: DeviceLayer, u: torch.Tensor, K: int, idx: torch.Tensor, w: torch.Tensor,
                               out: torch.Tensor, out_mode: int, perm_out: torch.Tensor | None = None,
                               err_word: torch.Tensor | None = None, stream=None):
    """moe_expert_forward without a workspace: scratch is the library's fixed per-device array.

    For callers that cannot allocate device memory.  Calls share that array, so
    calls that overlap on the GPU race; the first call on a device should come
    before any stream capture on it.
    """
    fn = "moe_expert_forward_noalloc"
    T, args = _expert_args(fn, layer, u, K, idx, w, out, out_mode, perm_out)
    err = _arg(fn, "err_word", err_word, I32, 1, optional=True)
    _check(fn, lib().moe_expert_forward_noalloc(ctypes.byref(layer.struct), _p(u), T, K, *args, err, _stream(stream)))


def prerouter_workspace_size(head: DeviceHead, T: int) -> int:
    return lib().prerouter_workspace_size(ctypes.byref(head.struct), T)


def prerouter_predict(head: DeviceHead, u: torch.Tensor, sel: torch.Tensor, K_next: int, pred: torch.Tensor,
                      scores: torch.Tensor, workspace: torch.Tensor, err_word: torch.Tensor | None = None, stream=None):
    fn, P = "prerouter_predict", head.struct
    if not isinstance(sel, torch.Tensor) or sel.dim() != 2:
        raise ValueError(f"{fn}: sel must be [T, K]")
    T, K = sel.shape
    if _rows(fn, "u", u, P.H, BF16_BITS) != T:
        raise ValueError(f"{fn}: u has {u.shape[0]} rows, sel has {T}")
    args = (_arg(fn, "sel", sel, I32), K_next, _arg(fn, "pred", pred, I32, T * K_next),
            _arg(fn, "scores", scores, F32, T * P.E_next))
    err = _arg(fn, "err_word", err_word, I32, 1, optional=True)
    _check(fn, lib().prerouter_predict(ctypes.byref(P), _p(u), args[0], T, K, *args[1:], *_ws(fn, workspace), err,
                                       _stream(stream)))


class TieredPool:
    """A layer's routed experts in pinned host memory behind an HBM cache of ``n_slots`` expert blocks
    (``moe_tier_*``).  Its ``struct`` is the layer view that ``moe_expert_forward`` takes with slot ids (pass the
    TieredPool as the layer): pool = the slot array, E = n_slots, no routed LoRA; ``moe_expert_forward`` reads
    neither the router nor any expert outside the pool."""

    def __init__(self, layer: DeviceLayer, host_blocks: torch.Tensor, n_slots: int, device=None):
        fn = "moe_tier_create"
        c = layer.cfg
        if not isinstance(host_blocks, torch.Tensor) or host_blocks.dtype != torch.uint8 or \
                host_blocks.dim() != 2 or host_blocks.shape[0] != c.E or not host_blocks.is_pinned():
            raise ValueError(f"{fn}: host_blocks must be a pinned uint8 [E, stride] tensor")
        if layer.struct.ex_lora_A:
            raise ValueError(f"{fn}: routed LoRA is not served from a tiered pool")
        self.layer, self.host = layer, host_blocks
        self.stride = block_stride(c.H, c.I)
        self.n_slots = n_slots
        self.slots = torch.zeros(n_slots * self.stride, dtype=torch.uint8,
                                 device=device if device is not None else layer.pool.device)
        h = ctypes.c_void_p()
        _check(fn, lib().moe_tier_create(host_blocks.data_ptr(), host_blocks.stride(0), c.E, block_bytes(c.H, c.I),
                                         self.slots.data_ptr(), self.stride, n_slots, ctypes.byref(h)))
        self.handle = h
        v = _lib.moe_layer()
        ctypes.memmove(ctypes.byref(v), ctypes.byref(layer.struct), ctypes.sizeof(v))
        v.E = n_slots
        v.router = _lib.moe_qrows(layer.struct.router.rows, n_slots, c.H, 8)
        v.pool, v.expert_stride = self.slots.data_ptr(), self.stride
        v.ex_lora_A = v.ex_lora_B = None
        self.struct = v  # a TieredPool stands in for the layer in moe_expert_forward / moe_workspace_size

    def acquire(self, experts, idx: torch.Tensor, idx_slot: torch.Tensor, err_word: torch.Tensor | None = None,
                stream=None):
        fn = "moe_tier_acquire"
        ex = np.ascontiguousarray(np.asarray(experts, dtype=np.int32).reshape(-1))
        n = idx.numel()
        a = _arg(fn, "idx", idx, I32, n)
        b = _arg(fn, "idx_slot", idx_slot, I32, n)
        err = _arg(fn, "err_word", err_word, I32, 1, optional=True)
        _check(fn, lib().moe_tier_acquire(self.handle, ex.ctypes.data, ex.size, a, n, b, err, _stream(stream)))

    def release(self, stream=None):
        _check("moe_tier_release", lib().moe_tier_release(self.handle, _stream(stream)))

    def prefetch(self, experts, stream=None):
        ex = np.ascontiguousarray(np.asarray(experts, dtype=np.int32).reshape(-1))
        _check("moe_tier_prefetch", lib().moe_tier_prefetch(self.handle, ex.ctypes.data, ex.size, _stream(stream)))

    def stats(self) -> dict:
        st = _lib.moe_tier_stats()
        _check("moe_tier_get_stats", lib().moe_tier_get_stats(self.handle, ctypes.byref(st)))
        return {n: getattr(st, n) for n, _ in st._fields_}

    def close(self):
        if getattr(self, "handle", None):
            lib().moe_tier_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_tier_create(layer: DeviceLayer, host_blocks: torch.Tensor, n_slots: int, device=None) -> TieredPool:
    return TieredPool(layer, host_blocks, n_slots, device)


def moe_tier_destroy(tier: TieredPool):
    tier.close()


def moe_tier_acquire(tier: TieredPool, experts, idx: torch.Tensor, idx_slot: torch.Tensor,
                     err_word: torch.Tensor | None = None, stream=None):
    tier.acquire(experts, idx, idx_slot, err_word, stream)


def moe_tier_release(tier: TieredPool, stream=None):
    tier.release(stream)


def moe_tier_prefetch(tier: TieredPool, experts, stream=None):
    tier.prefetch(experts, stream)


def moe_tier_get_stats(tier: TieredPool) -> dict:
    return tier.stats()


class StackStructs:
    """Contiguous host arrays of ``moe_layer`` / ``moe_prerouter`` structs for the stack entry points."""

    def __init__(self, layers, heads=None):
        # The structs hold raw device addresses: keep the tensors behind them alive as long as this object.
        self._owners = (layers, heads)
        if isinstance(layers, DeviceStack):
            self.n, self.layers, self.heads = layers.n, layers.layer_array, layers.head_array
            return
        self.n = len(layers)
        if self.n == 0:
            raise ValueError("StackStructs: a stack needs at least one layer")
        if heads is not None and len(heads) != self.n:
            raise ValueError(f"StackStructs: {len(heads)} Prerouter heads for {self.n} layers")
        self.layers = (_lib.moe_layer * self.n)(*[l.struct for l in layers])
        self.heads = None if heads is None else (_lib.moe_prerouter * self.n)(*[h.struct for h in heads])

    def heads_ptr(self):
        return None if self.heads is None else ctypes.cast(self.heads, ctypes.POINTER(_lib.moe_prerouter))


def moe_stack_workspace_size(stack: StackStructs, T: int, K: int, K_next: int) -> int:
    return lib().moe_stack_workspace_size(stack.layers, stack.heads_ptr(), stack.n, T, K, K_next)


PATH_AUTO, PATH_LAYERS, PATH_SINGLE = 0, 1, 2


def stack_opts(timeout_ns: int = 0, path: int = PATH_AUTO, drop_layer: int = -1, drop_cta: int = -1,
               trace: torch.Tensor | None = None):
    """moe_stack_opts; drop_layer/drop_cta (>= 0) arm the timeout-path test hook.

    ``trace``: int64 device tensor of ``n_layers * moe_stack_grid() * 16`` stamps
    (checked against the stack when the options are used).
    """
    o = _lib.moe_stack_opts(timeout_ns, path, drop_layer + 1 if drop_layer >= 0 else 0, drop_cta,
                            _arg("stack_opts", "trace", trace, I64, optional=True))
    o.trace_tensor = trace  # keeps the buffer alive and lets moe_stack_decode check its size
    return o


def moe_stack_grid() -> int:
    return lib().moe_stack_grid()


def moe_stack_decode(stack: StackStructs, x: torch.Tensor, K: int, K_next: int, eps: float, workspace: torch.Tensor,
                     x_trace=None, u_trace=None, idx_all=None, true_idx_all=None, pred_all=None,
                     use_predicted_routing=False, err_word=None, opts=None, stream=None):
    fn, n, H = "moe_stack_decode", stack.n, stack.layers[0].H
    T = _rows(fn, "x", x, H, F32)
    ptrs = (_arg(fn, "x_trace", x_trace, F32, n * T * H, optional=True),
            _arg(fn, "u_trace", u_trace, BF16_BITS, n * T * H, optional=True),
            _arg(fn, "idx_all", idx_all, I32, n * T * K, optional=True),
            _arg(fn, "true_idx_all", true_idx_all, I32, n * T * K, optional=True),
            _arg(fn, "pred_all", pred_all, I32, n * T * K_next, optional=True))
    err = _arg(fn, "err_word", err_word, I32, 1, optional=True)
    trace = getattr(opts, "trace_tensor", None) if opts is not None else None
    if trace is not None:
        _arg(fn, "opts.trace", trace, I64, n * moe_stack_grid() * 16)
    elif opts is not None and opts.trace:
        raise ValueError(f"{fn}: opts.trace was set without a tensor; build the options with stack_opts()")
    _check(fn, lib().moe_stack_decode(
        stack.layers, stack.heads_ptr(), n, T, K, K_next, eps, _p(x), *ptrs, int(bool(use_predicted_routing)), err,
        None if opts is None else ctypes.byref(opts), *_ws(fn, workspace), _stream(stream)))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A device scratch buffer (256-byte aligned by the caching allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
