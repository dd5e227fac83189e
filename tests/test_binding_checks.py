"""CPU checks of the Python binding's argument marshalling.

The binding hands raw device addresses to the C ABI, so it refuses host
tensors, wrong element types, strided views and buffers smaller than the call
touches before the library is called.  Here the library is replaced by a
recorder and tensors are host tensors that report a CUDA device, so the checks
and the argument order of every entry point run without a GPU.
"""
import ctypes
import weakref

import pytest
import torch

import int4_expert_ffn_top_b200 as M
from int4_expert_ffn_top_b200 import _lib

H, E, I, K, T = 256, 16, 128, 2, 5


class FakeCuda(torch.Tensor):
    @property
    def device(self):
        return torch.device("cuda", 0)


def cu(t: torch.Tensor) -> torch.Tensor:
    return torch.Tensor._make_subclass(FakeCuda, t)


class Recorder:
    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        def fn(*args):
            self.calls.append((name, args))
            return {"moe_stack_grid": 4, "moe_status_string": b"ok"}.get(name, _lib.MOE_OK)
        return fn


class FakeLayer:
    def __init__(self):
        self.struct = _lib.moe_layer()
        self.struct.H, self.struct.E, self.struct.I, self.struct.I_s, self.struct.r = H, E, I, I, 8


class FakeHead:
    def __init__(self):
        self.struct = _lib.moe_prerouter()
        self.struct.H, self.struct.E, self.struct.P, self.struct.E_next = H, E, 64, E


@pytest.fixture
def rec(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(M, "lib", lambda: r)
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    return r


def u16(rows=T, width=H):
    return cu(torch.zeros((rows, width), dtype=torch.int16))


def f32(*shape):
    return cu(torch.zeros(shape, dtype=torch.float32))


def i32(*shape):
    return cu(torch.zeros(shape, dtype=torch.int32))


def ws():
    return cu(torch.zeros(4096, dtype=torch.uint8))


# ----------------------------------------------------------------------------- accepted calls reach the ABI in order
def test_expert_forward_passes_arguments_in_abi_order(rec):
    u, idx, w, out, perm, work = u16(), i32(T, K), f32(T, K), f32(T, H), i32(T * K), ws()
    M.moe_expert_forward(FakeLayer(), u, K, idx, w, out, M.OUT_F32, work, perm_out=perm, stream=0)
    name, a = rec.calls[-1]
    assert name == "moe_expert_forward"
    assert a[1:] == (u.data_ptr(), T, K, idx.data_ptr(), w.data_ptr(), out.data_ptr(), 0, perm.data_ptr(),
                     work.data_ptr(), 4096, None, 0)
    err = i32(1)
    M.moe_expert_forward(FakeLayer(), u, K, idx, w, out, M.OUT_F32, work, err_word=err, stream=0)
    assert rec.calls[-1][1][-2:] == (err.data_ptr(), 0)
    out16 = u16()
    M.moe_expert_forward_noalloc(FakeLayer(), u, K, idx, w, out16, M.OUT_BF16, stream=0)
    name, a = rec.calls[-1]
    assert name == "moe_expert_forward_noalloc"
    assert a[1:] == (u.data_ptr(), T, K, idx.data_ptr(), w.data_ptr(), out16.data_ptr(), 1, None, None, 0)


def test_zero_tokens_and_a_larger_output_are_accepted(rec):
    M.moe_expert_forward(FakeLayer(), u16(rows=0), K, i32(0, K), f32(0, K), f32(1, H), M.OUT_F32, ws(), stream=0)
    assert rec.calls[-1][1][2] == 0


def test_route_rmsnorm_prerouter_argument_order(rec):
    u, logits, idx, w = u16(), f32(T, E), i32(T, K), f32(T, K)
    M.moe_route_topk(FakeLayer(), u, K, logits, idx, w, stream=0)
    assert rec.calls[-1][1][1:] == (u.data_ptr(), T, K, logits.data_ptr(), idx.data_ptr(), w.data_ptr(), None, 0)
    x = f32(T, H)
    M.moe_rmsnorm_bf16(x, 1e-6, u, stream=0)
    assert rec.calls[-1] == ("moe_rmsnorm_bf16", (x.data_ptr(), T, H, 1e-6, u.data_ptr(), 0))
    sel, pred, scores, work = i32(T, K), i32(T, 3), f32(T, E), ws()
    M.prerouter_predict(FakeHead(), u, sel, 3, pred, scores, work, stream=0)
    assert rec.calls[-1][1][1:] == (u.data_ptr(), sel.data_ptr(), T, K, 3, pred.data_ptr(), scores.data_ptr(),
                                    work.data_ptr(), 4096, None, 0)


def test_stack_decode_argument_order_and_trace_size(rec):
    layers = [FakeLayer(), FakeLayer()]
    st = M.StackStructs(layers)
    n = 2
    x, err = f32(1, H), i32(1)
    tr = dict(x_trace=f32(n, 1, H), u_trace=u16(rows=n, width=H), idx_all=i32(n, 1, K), true_idx_all=i32(n, 1, K),
              pred_all=i32(n, 1, K))
    work = ws()
    trace = cu(torch.zeros((n, 4, 16), dtype=torch.int64))
    opts = M.stack_opts(path=M.PATH_SINGLE, trace=trace)
    M.moe_stack_decode(st, x, K, K, 1e-6, work, err_word=err, opts=opts, stream=0, **tr)
    name, a = rec.calls[-1]
    assert name == "moe_stack_decode"
    assert a[2:7] == (n, 1, K, K, 1e-6) and a[7] == x.data_ptr()
    assert a[8:13] == tuple(tr[k].data_ptr() for k in ("x_trace", "u_trace", "idx_all", "true_idx_all", "pred_all"))
    assert a[13] == 0 and a[14] == err.data_ptr() and a[16:] == (work.data_ptr(), 4096, 0)
    with pytest.raises(ValueError, match="opts.trace"):  # one stamp row short of n * grid * 16
        M.moe_stack_decode(st, x, K, K, 1e-6, work,
                           opts=M.stack_opts(trace=cu(torch.zeros((n, 3, 16), dtype=torch.int64))), stream=0)
    raw = _lib.moe_stack_opts(0, 0, 0, -1, trace.data_ptr())  # a bare struct gives no size to check
    with pytest.raises(ValueError, match="stack_opts"):
        M.moe_stack_decode(st, x, K, K, 1e-6, work, opts=raw, stream=0)


# ----------------------------------------------------------------------------- refused before the library is called
@pytest.mark.parametrize("case", ["host", "dtype", "strided", "short", "width", "missing", "out_bf16", "out_f32",
                                  "perm_short", "not_tensor"])
def test_bad_arguments_never_reach_the_library(rec, case):
    args = dict(u=u16(), idx=i32(T, K), w=f32(T, K), out=f32(T, H), mode=M.OUT_F32, perm=None)
    if case == "host":
        args["idx"] = torch.zeros((T, K), dtype=torch.int32)
    elif case == "dtype":
        args["idx"] = cu(torch.zeros((T, K), dtype=torch.int64))
    elif case == "strided":
        args["w"] = cu(torch.zeros((K, T), dtype=torch.float32)).t()
    elif case == "short":
        args["w"] = f32(T, K - 1)
    elif case == "width":
        args["u"] = u16(width=H // 2)
    elif case == "missing":
        args["out"] = None
    elif case == "out_bf16":  # fp32 output mode with a 16-bit buffer
        args["out"] = u16()
    elif case == "out_f32":  # bf16 output mode with an fp32 buffer
        args["mode"] = M.OUT_BF16
    elif case == "perm_short":
        args["perm"] = i32(T * K - 1)
    elif case == "not_tensor":
        args["idx"] = [[0, 1]] * T
    with pytest.raises((ValueError, TypeError)):
        M.moe_expert_forward(FakeLayer(), args["u"], K, args["idx"], args["w"], args["out"], args["mode"], ws(),
                             perm_out=args["perm"], stream=0)
    assert rec.calls == []


def test_host_tensor_is_refused_with_its_device_named():
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        M._arg("f", "x", torch.zeros(4), (torch.float32,))


def test_stack_structs_keep_the_device_tensors_alive():
    layer = FakeLayer()
    ref = weakref.ref(layer)
    st = M.StackStructs([layer])
    del layer
    assert ref() is not None and st.n == 1
    assert isinstance(st.layers, ctypes.Array)


def test_stack_structs_refuse_an_empty_stack_or_mismatched_heads():
    with pytest.raises(ValueError, match="at least one layer"):
        M.StackStructs([])
    with pytest.raises(ValueError, match="heads"):
        M.StackStructs([FakeLayer(), FakeLayer()], [FakeHead()])
    st = M.StackStructs([FakeLayer()], [FakeHead()])
    assert st.heads_ptr() is not None


def test_tier_calls_pass_arguments_in_abi_order(rec):
    tp = object.__new__(M.TieredPool)  # the constructor needs pinned host memory; the calls do not
    tp.handle = ctypes.c_void_p(1234)
    try:
        idx, slot, err = i32(T, K), i32(T, K), i32(1)
        tp.acquire([3, 1], idx, slot, err_word=err, stream=0)
        name, a = rec.calls[-1]
        assert name == "moe_tier_acquire"
        assert a[0] is tp.handle and a[2] == 2 and a[3:] == (idx.data_ptr(), T * K, slot.data_ptr(), err.data_ptr(), 0)
        n = len(rec.calls)
        with pytest.raises(ValueError):
            tp.acquire([3], idx, i32(T * K - 1), stream=0)  # idx_slot smaller than idx
        with pytest.raises(ValueError):
            tp.acquire([3], cu(torch.zeros((T, K), dtype=torch.int64)), slot, stream=0)  # wrong element type
        assert len(rec.calls) == n  # neither reached the library
        tp.prefetch([5, 6, 7], stream=0)
        name, a = rec.calls[-1]
        assert name == "moe_tier_prefetch" and a[0] is tp.handle and a[2] == 3 and a[3] == 0
        tp.release(stream=0)
        assert rec.calls[-1] == ("moe_tier_release", (tp.handle, 0))
    finally:
        tp.handle = None  # the fake handle must never reach the real library
