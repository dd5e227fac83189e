"""ctypes view of libmoe.so: struct layouts and raw entry points of ``include/moe.h``."""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int32, c_int64, c_size_t, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, MOE_ERR_RANGE = range(7)
MOE_MAX_TOKENS = 524280  # most tokens one call takes


class moe_qrows(ctypes.Structure):
    _fields_ = [("rows", c_void_p), ("out_dim", c_int32), ("in_dim", c_int32), ("bits", c_int32)]


class moe_layer(ctypes.Structure):
    _fields_ = [("H", c_int32), ("E", c_int32), ("I", c_int32), ("I_s", c_int32), ("r", c_int32),
                ("router", moe_qrows), ("router_bias", c_void_p), ("shared_gate", moe_qrows),
                ("shared_block", c_void_p),
                ("sh_lora_A", c_void_p * 3), ("sh_lora_B", c_void_p * 3), ("lora_scale", c_float),
                ("pool", c_void_p), ("expert_stride", c_int64), ("ex_lora_A", c_void_p), ("ex_lora_B", c_void_p),
                ("ex_lora_A_gu", c_void_p), ("ex_lora_B_gu", c_void_p)]


class moe_stack_opts(ctypes.Structure):
    _fields_ = [("timeout_ns", c_int64), ("path", c_int32), ("test_drop_layer", c_int32), ("test_drop_cta", c_int32),
                ("trace", c_void_p)]


class moe_prerouter(ctypes.Structure):
    _fields_ = [("W1", c_void_p), ("b1", c_void_p), ("W2", c_void_p), ("b2", c_void_p),
                ("H", c_int32), ("E", c_int32), ("P", c_int32), ("E_next", c_int32)]


class moe_tier_stats(ctypes.Structure):
    _fields_ = [(n, c_int64) for n in ("acquires", "requested", "hits", "prefetch_hits", "misses", "prefetched",
                                       "bytes_acquired", "bytes_prefetched")]


# name -> (restype, argtypes); mirrors include/moe.h
SIGNATURES = {
    "moe_status_string": (c_char_p, [c_int32]),
    "moe_qrow_bytes": (c_size_t, [c_int32, c_int32]),
    "moe_expert_block_bytes": (c_size_t, [c_int32, c_int32]),
    "moe_rmsnorm_bf16": (c_int32, [c_void_p, c_int32, c_int32, c_float, c_void_p, c_void_p]),
    "moe_route_topk": (c_int32, [POINTER(moe_layer), c_void_p, c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_void_p]),
    "moe_expert_forward": (c_int32, [POINTER(moe_layer), c_void_p, c_int32, c_int32, c_void_p, c_void_p, c_void_p,
                                     c_int32, c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
    "moe_workspace_size": (c_size_t, [POINTER(moe_layer), c_int32, c_int32]),
    "prerouter_predict": (c_int32, [POINTER(moe_prerouter), c_void_p, c_void_p, c_int32, c_int32, c_int32, c_void_p,
                                    c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
    "prerouter_workspace_size": (c_size_t, [POINTER(moe_prerouter), c_int32]),
    "moe_stack_decode": (c_int32, [POINTER(moe_layer), POINTER(moe_prerouter), c_int32, c_int32, c_int32, c_int32,
                                   c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int32,
                                   c_void_p, POINTER(moe_stack_opts), c_void_p,
                                   c_size_t, c_void_p]),
    "moe_expert_forward_noalloc": (c_int32, [POINTER(moe_layer), c_void_p, c_int32, c_int32, c_void_p, c_void_p,
                                             c_void_p, c_int32, c_void_p, c_void_p, c_void_p]),
    "moe_noalloc_scratch_bytes": (c_size_t, []),
    "moe_tier_create": (c_int32, [c_void_p, c_int64, c_int32, c_int64, c_void_p, c_int64, c_int32, POINTER(c_void_p)]),
    "moe_tier_destroy": (None, [c_void_p]),
    "moe_tier_acquire": (c_int32, [c_void_p, c_void_p, c_int32, c_void_p, c_int32, c_void_p, c_void_p, c_void_p]),
    "moe_tier_release": (c_int32, [c_void_p, c_void_p]),
    "moe_tier_prefetch": (c_int32, [c_void_p, c_void_p, c_int32, c_void_p]),
    "moe_tier_get_stats": (c_int32, [c_void_p, POINTER(moe_tier_stats)]),
    "moe_stack_grid": (c_int32, []),
    "moe_stack_workspace_size": (c_size_t, [POINTER(moe_layer), POINTER(moe_prerouter), c_int32, c_int32, c_int32,
                                            c_int32]),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoe.so; raises if it is missing (there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"libmoe.so not built at {path}; run int4_expert_ffn_top_b200.build.build()")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
