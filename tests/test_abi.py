"""CPU checks of the C ABI: the library loads, exports every declared symbol, and
rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

from int4_expert_ffn_top_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    from int4_expert_ffn_top_b200 import _lib
    return _lib.load()


def declared_functions():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", src, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while")))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "moe_route_topk" in names and "moe_expert_forward" in names and "prerouter_predict" in names
    for n in names:
        assert hasattr(lib, n), n


def test_python_binding_mirrors_the_header():
    import int4_expert_ffn_top_b200 as M
    from int4_expert_ffn_top_b200 import _lib
    for n in declared_functions():
        assert n in _lib.SIGNATURES, n
        assert hasattr(M, n), n


def test_tier_host_side_rejections(lib):
    """The tiered pool's entry points refuse null handles, pointers and bad sizes before any CUDA call."""
    from int4_expert_ffn_top_b200 import _lib
    h = ctypes.c_void_p()
    bad = _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_tier_create(None, 4096, 16, 4096, None, 4096, 4, ctypes.byref(h)) == bad and not h.value
    assert lib.moe_tier_create(1 << 20, 4096, 0, 4096, 1 << 21, 4096, 4, ctypes.byref(h)) == bad  # no experts
    assert lib.moe_tier_create(1 << 20, 4096, 300, 4096, 1 << 21, 4096, 4, ctypes.byref(h)) == bad  # > 256
    assert lib.moe_tier_create(1 << 20, 4096, 16, 4096, 1 << 21, 4000, 4, ctypes.byref(h)) == bad  # stride < block
    assert lib.moe_tier_create(1 << 20, 4096, 16, 4096, (1 << 21) + 16, 4096, 4, ctypes.byref(h)) == bad  # align
    assert lib.moe_tier_create(1 << 20, 4096, 16, 4096, 1 << 21, 4096, 4, None) == bad
    assert lib.moe_tier_acquire(None, None, 0, None, 0, None, None, None) == bad
    assert lib.moe_tier_release(None, None) == bad
    assert lib.moe_tier_prefetch(None, None, 0, None) == bad
    st = _lib.moe_tier_stats()
    assert lib.moe_tier_get_stats(None, ctypes.byref(st)) == bad
    lib.moe_tier_destroy(None)  # a null handle is ignored


def test_status_strings(lib):
    from int4_expert_ffn_top_b200 import moe_status_string
    assert moe_status_string(0) == "ok"
    assert "workspace" in moe_status_string(3)
    assert moe_status_string(99) == "unknown status"


def test_expert_block_bytes(lib):
    from int4_expert_ffn_top_b200 import block_bytes, moe_expert_block_bytes, moe_qrow_bytes, qrow_bytes
    # gate/up 1024 x (1024 B codes + 64 B scales + 64 B biases) + down 2048 x (256 + 16 + 16)
    assert moe_expert_block_bytes(2048, 512) == 1024 * 1152 + 2048 * 288 == 1769472
    # records pad to 16 bytes: 64 + 4 + 4 -> 80
    assert moe_qrow_bytes(128, 4) == 80 and moe_qrow_bytes(2048, 8) == 2048 + 128
    for H, I in ((256, 128), (2048, 512), (4096, 1024)):
        assert moe_expert_block_bytes(H, I) == block_bytes(H, I)
        assert moe_qrow_bytes(H, 4) == qrow_bytes(H, 4)
    assert moe_expert_block_bytes(2048, 100) == 0 and moe_qrow_bytes(100, 4) == 0


def test_host_side_rejections(lib):
    from int4_expert_ffn_top_b200 import _lib
    L = _lib.moe_layer()
    # null layer / null pointers / bad shapes fail before any launch
    assert lib.moe_route_topk(None, None, 1, 4, None, None, None, None, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_rmsnorm_bf16(None, -1, 2048, 1e-6, None, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_rmsnorm_bf16(None, 0, 2048, 1e-6, None, None) == _lib.MOE_OK
    L.H, L.E, L.I, L.I_s, L.r = 2048, 256, 512, 512, 16
    assert lib.moe_route_topk(ctypes.byref(L), None, 1, 9, None, None, None, None, None) == _lib.MOE_ERR_UNSUPPORTED
    L.H = 2000
    assert lib.moe_route_topk(ctypes.byref(L), None, 1, 4, None, None, None, None, None) == _lib.MOE_ERR_UNSUPPORTED
    L.H = 2048
    L.r = 12  # LoRA ranks are multiples of 8
    assert lib.moe_route_topk(ctypes.byref(L), None, 1, 4, None, None, None, None, None) == _lib.MOE_ERR_UNSUPPORTED
    L.r = 16
    # router matrix missing
    assert lib.moe_route_topk(ctypes.byref(L), None, 1, 4, None, None, None, None, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_forward(ctypes.byref(L), None, 1, 4, None, None, None, 0, None, None, 0,
                                  None, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_expert_forward(ctypes.byref(L), None, 1, 4, None, None, None, 7, None, None, 0,
                                  None, None) == _lib.MOE_ERR_INVALID_ARG
    P = _lib.moe_prerouter()
    P.H, P.E, P.P, P.E_next = 2048, 256, 256, 256
    assert lib.prerouter_predict(ctypes.byref(P), None, None, 1, 4, 9, None, None, None, 0,
                                 None, None) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.prerouter_predict(ctypes.byref(P), None, None, 1, 4, 4, None, None, None, 0,
                                 None, None) == _lib.MOE_ERR_INVALID_ARG
    assert lib.moe_stack_decode(None, None, 0, 1, 4, 4, 1e-6, None, None, None, None, None, None, 0, None, None,
                                None, 0, None) == _lib.MOE_ERR_INVALID_ARG


def test_token_limit_is_rejected_on_the_host(lib):
    import re as _re

    from int4_expert_ffn_top_b200 import _lib
    hdr = open(os.path.join(ROOT, "include", "moe.h")).read()
    assert int(_re.search(r"#define MOE_MAX_TOKENS (\d+)", hdr).group(1)) == _lib.MOE_MAX_TOKENS == 65535 * 8
    L = _lib.moe_layer()
    L.H, L.E, L.I, L.I_s, L.r = 2048, 256, 512, 512, 16
    big = _lib.MOE_MAX_TOKENS + 1
    assert lib.moe_route_topk(ctypes.byref(L), None, big, 4, None, None, None, None, None) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.moe_expert_forward(ctypes.byref(L), None, big, 4, None, None, None, 0, None, None, 0,
                                  None, None) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.moe_workspace_size(ctypes.byref(L), big, 4) == 0
    assert lib.moe_workspace_size(ctypes.byref(L), _lib.MOE_MAX_TOKENS, 4) > 0
    P = _lib.moe_prerouter()
    P.H, P.E, P.P, P.E_next = 2048, 256, 256, 256
    assert lib.prerouter_predict(ctypes.byref(P), None, None, big, 4, 4, None, None, None, 0,
                                 None, None) == _lib.MOE_ERR_UNSUPPORTED
    assert lib.prerouter_workspace_size(ctypes.byref(P), big) == 0
    assert lib.moe_stack_workspace_size(ctypes.byref(L), None, 1, big, 4, 4) == 0


def test_workspace_sizes_grow_with_tokens(lib):
    from int4_expert_ffn_top_b200 import _lib
    L = _lib.moe_layer()
    L.H, L.E, L.I, L.I_s, L.r = 2048, 256, 512, 512, 16
    a = lib.moe_workspace_size(ctypes.byref(L), 1, 4)
    b = lib.moe_workspace_size(ctypes.byref(L), 64, 4)
    assert 0 < a < b and a % 256 == 0 and b % 256 == 0
    # h for (T*K + T) slots x I fp16 dominates
    assert b >= (64 * 4 + 64) * 512 * 2


def test_bench_diagnostic_mode_parses_its_arguments():
    """The profiling/tracing mode named in profiles/ (bench.py --diag-stack) parses its options without a GPU."""
    import subprocess
    import sys
    r = subprocess.run([sys.executable, "bench.py", "--help"],
                       cwd=os.path.dirname(os.path.dirname(os.path.abspath(__file__))), capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and "--diag-stack" in r.stdout and "--trace" in r.stdout


def test_expert_block_layout_decodes_back_to_the_expert():
    """The HBM expert block: gate/up records interleaved (gate_j, up_j), then down records; each record is
    codes (nibble k at bits 4(k%2) of byte k/2), then in/64 fp16 scales, then in/64 fp16 biases."""
    import numpy as np

    from gen import CONFIGS, inputs
    from int4_expert_ffn_top_b200.weights import expert_block, qrow_bytes
    from oracle import moe_oracle as O

    cfg = CONFIGS[0]
    ex = inputs.layer(cfg, 0, experts=[5])["experts"][5]
    blk = expert_block(ex)
    H, I = cfg.H, cfg.I

    def decode(rec, in_dim):
        cb, G = in_dim // 2, in_dim // 64
        q = np.empty(in_dim)
        q[0::2], q[1::2] = rec[:cb] & 15, rec[:cb] >> 4
        s = rec[cb:cb + 2 * G].view(np.float16).astype(np.float64)
        b = rec[cb + 2 * G:cb + 4 * G].view(np.float16).astype(np.float64)
        return q * np.repeat(s, 64) + np.repeat(b, 64)

    rgu, rdn = qrow_bytes(H, 4), qrow_bytes(I, 4)
    assert blk.size == 2 * I * rgu + H * rdn
    gu = O.dequant(ex["gate_up"])
    dn = O.dequant(ex["down"])
    for j in (0, 1, I // 2, I - 1):
        assert np.array_equal(decode(blk[(2 * j) * rgu:(2 * j + 1) * rgu], H), gu[j])          # gate row j
        assert np.array_equal(decode(blk[(2 * j + 1) * rgu:(2 * j + 2) * rgu], H), gu[I + j])  # up row j
    off = 2 * I * rgu
    for o in (0, 7, H - 1):
        assert np.array_equal(decode(blk[off + o * rdn:off + (o + 1) * rdn], I), dn[o])


# Well-formed structs whose pointers are aligned stand-in addresses.  The calls
# below end at a host-side check (a zero-byte workspace at the latest), so no
# address is ever used on a device.
def _fake_layer(base: int):
    from int4_expert_ffn_top_b200 import _lib
    from int4_expert_ffn_top_b200.weights import block_stride
    L = _lib.moe_layer()
    L.H, L.E, L.I, L.I_s, L.r = 2048, 256, 512, 512, 16
    L.router = _lib.moe_qrows(base + 0x1000, 256, 2048, 8)
    L.shared_gate = _lib.moe_qrows(base + 0x2000, 1, 2048, 8)
    L.shared_block = base + 0x3000
    for i in range(3):
        L.sh_lora_A[i], L.sh_lora_B[i] = base + 0x4000 + 0x100 * i, base + 0x5000 + 0x100 * i
    L.lora_scale = 1.0
    L.pool = base + 0x100000
    L.expert_stride = block_stride(2048, 512)
    return L


def _fake_head(base: int):
    from int4_expert_ffn_top_b200 import _lib
    P = _lib.moe_prerouter()
    P.W1, P.b1, P.W2, P.b2 = base + 0x6000, base + 0x7000, base + 0x8000, base + 0x9000
    P.H, P.E, P.P, P.E_next = 2048, 256, 256, 256
    return P


FAKE_WS = 0x7f0000000000  # 256-byte aligned, never dereferenced: every call is refused before it


def test_well_formed_calls_pass_every_host_check(lib):
    from int4_expert_ffn_top_b200 import _lib
    L, P = _fake_layer(0x10000000), _fake_head(0x20000000)
    dev = 0x30000000
    assert lib.moe_expert_forward(ctypes.byref(L), dev, 1, 4, dev, dev, dev, 0, None, FAKE_WS, 0,
                                  None, None) == _lib.MOE_ERR_WORKSPACE
    assert lib.prerouter_predict(ctypes.byref(P), dev, dev, 1, 4, 4, dev, dev, FAKE_WS, 0,
                                 None, None) == _lib.MOE_ERR_WORKSPACE
    layers = (_lib.moe_layer * 3)(*[_fake_layer(0x10000000 * (l + 1)) for l in range(3)])
    heads = (_lib.moe_prerouter * 3)(*[_fake_head(0x40000000 * (l + 1)) for l in range(3)])
    assert lib.moe_stack_decode(layers, heads, 3, 1, 4, 4, 1e-6, dev, None, None, None, None, None, 0, None, None,
                                FAKE_WS, 0, None) == _lib.MOE_ERR_WORKSPACE


def test_stack_weights_of_every_layer_are_checked_before_any_launch(lib):
    from int4_expert_ffn_top_b200 import _lib

    def stack_status(edit_layer=None, edit_head=None, K_next=4):
        layers = (_lib.moe_layer * 3)(*[_fake_layer(0x10000000 * (l + 1)) for l in range(3)])
        heads = (_lib.moe_prerouter * 3)(*[_fake_head(0x40000000 * (l + 1)) for l in range(3)])
        if edit_layer:
            edit_layer(layers[2])
        if edit_head:
            edit_head(heads[2])
        return lib.moe_stack_decode(layers, heads, 3, 1, 4, K_next, 1e-6, 0x30000000, None, None, None, None, None,
                                    0, None, None, FAKE_WS, 0, None)

    def no_pool(L):
        L.pool = None

    def short_stride(L):
        L.expert_stride = 256

    def half_lora(L):
        L.sh_lora_B[1] = None

    def no_w1(P):
        P.W1 = None

    def odd_w2(P):
        P.W2 = P.W2 + 8

    def small_e_next(P):
        P.E_next = 2

    for edit in (no_pool, short_stride, half_lora):
        assert stack_status(edit_layer=edit) == _lib.MOE_ERR_INVALID_ARG, edit.__name__
    for edit in (no_w1, odd_w2):
        assert stack_status(edit_head=edit) == _lib.MOE_ERR_INVALID_ARG, edit.__name__
    assert stack_status(edit_head=small_e_next) == _lib.MOE_ERR_UNSUPPORTED
    assert stack_status(K_next=9) == _lib.MOE_ERR_UNSUPPORTED
    assert stack_status() == _lib.MOE_ERR_WORKSPACE


def test_header_is_plain_c99_and_the_library_links_from_c(lib):
    """A C program (no C++, no torch) compiles against include/moe.h with -pedantic -Werror, links libmoe.so and
    calls the host-only entry points; the one compute entry point it calls is refused before any launch."""
    import shutil
    import subprocess

    from int4_expert_ffn_top_b200 import build as B
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    out_dir = os.path.join(ROOT, "_build", "c_abi_check")
    os.makedirs(out_dir, exist_ok=True)
    src, exe = os.path.join(out_dir, "main.c"), os.path.join(out_dir, "main")
    with open(src, "w") as f:
        f.write(r'''
#include <stdio.h>
#include <string.h>
#include "moe.h"
int main(void) {
  moe_layer L;
  memset(&L, 0, sizeof L);
  L.H = 2048; L.E = 256; L.I = 512; L.I_s = 512; L.r = 16;
  printf("%s|%zu|%zu|%d|%zu\n", moe_status_string(MOE_ERR_WORKSPACE), moe_expert_block_bytes(2048, 512),
         moe_qrow_bytes(2048, 8), (int)moe_route_topk(&L, NULL, 1, 4, NULL, NULL, NULL, NULL, NULL),
         moe_workspace_size(&L, MOE_MAX_TOKENS + 1, 4));
  return 0;
}
''')
    lib_dir = os.path.dirname(B.LIB)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    src, "-o", exe, "-L", lib_dir, "-lmoe", f"-Wl,-rpath,{lib_dir}"], check=True, timeout=120)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60, check=True)
    assert r.stdout.strip() == "workspace too small|1769472|2176|1|0"  # router rows missing -> invalid argument
