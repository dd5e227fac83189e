"""B200 routed-expert layer: Python binding of libmoe.so.

The functions here have the names of the C entry points in ``include/moe.h``
and only marshal arguments (torch tensors -> device pointers, the caller's
current CUDA stream) and turn a non-zero status into ``MoEError``.  Every step
of the computation runs in the library's CUDA kernels; there is no other path.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from .weights import DeviceHead, DeviceLayer, DeviceStack, block_bytes, block_stride, qrow_bytes  # noqa: F401

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
    T, H = x.shape
    _check("moe_rmsnorm_bf16", lib().moe_rmsnorm_bf16(_p(x), T, H, eps, _p(u), _stream(stream)))


def moe_route_topk(layer: DeviceLayer, u: torch.Tensor, K: int, logits: torch.Tensor, idx: torch.Tensor,
                   w: torch.Tensor, stream=None):
    T = u.shape[0]
    _check("moe_route_topk", lib().moe_route_topk(ctypes.byref(layer.struct), _p(u), T, K, _p(logits), _p(idx),
                                                  _p(w), _stream(stream)))


def moe_workspace_size(layer: DeviceLayer, T: int, K: int) -> int:
    return lib().moe_workspace_size(ctypes.byref(layer.struct), T, K)


def moe_expert_forward(layer: DeviceLayer, u: torch.Tensor, K: int, idx: torch.Tensor, w: torch.Tensor,
                       out: torch.Tensor, out_mode: int, workspace: torch.Tensor, perm_out: torch.Tensor | None = None,
                       stream=None):
    T = u.shape[0]
    _check("moe_expert_forward", lib().moe_expert_forward(
        ctypes.byref(layer.struct), _p(u), T, K, _p(idx), _p(w), _p(out), out_mode, _p(perm_out), _p(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


def moe_noalloc_scratch_bytes() -> int:
    return lib().moe_noalloc_scratch_bytes()


def moe_expert_forward_noalloc(layer: DeviceLayer, u: torch.Tensor, K: int, idx: torch.Tensor, w: torch.Tensor,
                               out: torch.Tensor, out_mode: int, perm_out: torch.Tensor | None = None, stream=None):
    """moe_expert_forward without a workspace: scratch is the library's fixed per-device array.

    For callers that cannot allocate device memory.  Calls share that array, so
    calls that overlap on the GPU race; the first call on a device should come
    before any stream capture on it.
    """
    T = u.shape[0]
    _check("moe_expert_forward_noalloc", lib().moe_expert_forward_noalloc(
        ctypes.byref(layer.struct), _p(u), T, K, _p(idx), _p(w), _p(out), out_mode, _p(perm_out), _stream(stream)))


def prerouter_workspace_size(head: DeviceHead, T: int) -> int:
    return lib().prerouter_workspace_size(ctypes.byref(head.struct), T)


def prerouter_predict(head: DeviceHead, u: torch.Tensor, sel: torch.Tensor, K_next: int, pred: torch.Tensor,
                      scores: torch.Tensor, workspace: torch.Tensor, stream=None):
    T, K = sel.shape
    _check("prerouter_predict", lib().prerouter_predict(
        ctypes.byref(head.struct), _p(u), _p(sel), T, K, K_next, _p(pred), _p(scores), _p(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))


class StackStructs:
    """Contiguous host arrays of ``moe_layer`` / ``moe_prerouter`` structs for the stack entry points."""

    def __init__(self, layers, heads=None):
        if isinstance(layers, DeviceStack):
            self.n, self.layers, self.heads = layers.n, layers.layer_array, layers.head_array
            return
        self.n = len(layers)
        self.layers = (_lib.moe_layer * self.n)(*[l.struct for l in layers])
        self.heads = None if heads is None else (_lib.moe_prerouter * self.n)(*[h.struct for h in heads])

    def heads_ptr(self):
        return None if self.heads is None else ctypes.cast(self.heads, ctypes.POINTER(_lib.moe_prerouter))


def moe_stack_workspace_size(stack: StackStructs, T: int, K: int, K_next: int) -> int:
    return lib().moe_stack_workspace_size(stack.layers, stack.heads_ptr(), stack.n, T, K, K_next)


PATH_AUTO, PATH_LAYERS, PATH_SINGLE = 0, 1, 2


def stack_opts(timeout_ns: int = 0, path: int = PATH_AUTO, drop_layer: int = -1, drop_cta: int = -1,
               trace: torch.Tensor | None = None):
    """moe_stack_opts; drop_layer/drop_cta (>= 0) arm the timeout-path test hook; trace: int64 device tensor."""
    return _lib.moe_stack_opts(timeout_ns, path, drop_layer + 1 if drop_layer >= 0 else 0, drop_cta, _p(trace))


def moe_stack_grid() -> int:
    return lib().moe_stack_grid()


def moe_stack_decode(stack: StackStructs, x: torch.Tensor, K: int, K_next: int, eps: float, workspace: torch.Tensor,
                     x_trace=None, u_trace=None, idx_all=None, true_idx_all=None, pred_all=None,
                     use_predicted_routing=False, err_word=None, opts=None, stream=None):
    T = x.shape[0]
    _check("moe_stack_decode", lib().moe_stack_decode(
        stack.layers, stack.heads_ptr(), stack.n, T, K, K_next, eps, _p(x), _p(x_trace), _p(u_trace), _p(idx_all),
        _p(true_idx_all), _p(pred_all), int(bool(use_predicted_routing)), _p(err_word),
        None if opts is None else ctypes.byref(opts), _p(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A device scratch buffer (256-byte aligned by the caching allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
