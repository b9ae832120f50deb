"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/respin.h declares, and rejects bad arguments (and
injected faults) before touching the device."""
import ctypes
import os
import re

import pytest

import rotation_post_quantization_b200 as rq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "respin.h")

# fake, suitably aligned device addresses: validation never dereferences them
A16 = 0x10000
A16B = 0x20000
MIS = 0x10008


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(
        r"^\s*(?:respin_status_t|const char\*)\s+(\w+)\s*\(", src, flags=re.M)))


def test_header_symbols_exported():
    names = declared_functions()
    assert len(names) >= 8
    assert set(names) == set(rq.EXPORTED)
    for n in names:
        assert hasattr(rq.lib, n), n


def test_header_flag_values_match_binding():
    src = open(HEADER).read()
    flags = dict((m, int(v)) for m, v in re.findall(r"#define (RESPIN_\w+) (\d+)u", src))
    assert flags == {"RESPIN_H_FP32_DEBUG": rq.RESPIN_H_FP32_DEBUG,
                     "RESPIN_ACT_INT3": rq.RESPIN_ACT_INT3}


def test_version():
    assert "sm_100a" in rq.version()


def call_create(D, r, U=None, V=None, flags=0):
    h = ctypes.c_void_p()
    fp = ctypes.POINTER(ctypes.c_float)
    buf = (ctypes.c_float * 8)()
    up = ctypes.cast(buf, fp) if U else None
    vp = ctypes.cast(buf, fp) if V else None
    return rq.lib.respin_plan_create(ctypes.byref(h), D, r, up, vp, flags), h


@pytest.mark.parametrize("D,r,U,V,flags,want", [
    (100, 0, False, False, 0, rq.RESPIN_ERR_UNSUPPORTED),     # D % 128
    (0, 0, False, False, 0, rq.RESPIN_ERR_UNSUPPORTED),
    (4096, 12, True, True, 0, rq.RESPIN_ERR_UNSUPPORTED),     # r % 8
    (4096, 136, True, True, 0, rq.RESPIN_ERR_UNSUPPORTED),    # r > 128
    (4096, -8, True, True, 0, rq.RESPIN_ERR_UNSUPPORTED),
    (4096, 32, False, True, 0, rq.RESPIN_ERR_INVALID_ARG),    # NULL U
    (4096, 32, True, False, 0, rq.RESPIN_ERR_INVALID_ARG),    # NULL V
    (4096, 32, True, True, 4, rq.RESPIN_ERR_INVALID_ARG),     # unknown flag
])
def test_plan_create_validation(D, r, U, V, flags, want):
    st, h = call_create(D, r, U, V, flags)
    assert st == want
    assert not h.value
    assert rq.last_error()


def test_plan_create_null_out():
    assert rq.lib.respin_plan_create(None, 4096, 0, None, None, 0) == \
        rq.RESPIN_ERR_INVALID_ARG


def test_fault_hook_plan_alloc(monkeypatch):
    monkeypatch.setenv("RESPIN_FAULT", "plan_alloc")
    st, h = call_create(4096, 0)
    assert st == rq.RESPIN_ERR_OOM
    assert "injected" in rq.last_error()
    with pytest.raises(rq.RespinError) as ei:
        rq.Plan(4096, 0)
    assert ei.value.status == rq.RESPIN_ERR_OOM


def test_unknown_plan_rejected():
    assert rq.lib.respin_plan_destroy(None) == rq.RESPIN_OK
    assert rq.lib.respin_plan_destroy(ctypes.c_void_p(0x1234)) == \
        rq.RESPIN_ERR_INVALID_ARG
    st = rq.lib.respin_boundary_forward(ctypes.c_void_p(0x1234), A16, A16, 4,
                                        A16, A16, A16, None)
    assert st == rq.RESPIN_ERR_INVALID_ARG
    assert "plan" in rq.last_error()


def gemm(qa=A16, sa=A16, qw=A16B, sw=A16B, N=4, K=256, O=32, out=A16):
    return rq.lib.w4a4_gemm(qa, sa, qw, sw, N, K, O, out, None)


@pytest.mark.parametrize("kw,want", [
    (dict(K=100), rq.RESPIN_ERR_UNSUPPORTED),
    (dict(K=0), rq.RESPIN_ERR_UNSUPPORTED),
    (dict(K=131072), rq.RESPIN_ERR_UNSUPPORTED),
    (dict(O=24), rq.RESPIN_ERR_UNSUPPORTED),
    (dict(O=0), rq.RESPIN_ERR_UNSUPPORTED),
    (dict(N=-1), rq.RESPIN_ERR_INVALID_ARG),
    (dict(qa=None), rq.RESPIN_ERR_INVALID_ARG),
    (dict(sw=None), rq.RESPIN_ERR_INVALID_ARG),
    (dict(out=None), rq.RESPIN_ERR_INVALID_ARG),
    (dict(qa=MIS), rq.RESPIN_ERR_ALIGNMENT),
    (dict(out=MIS), rq.RESPIN_ERR_ALIGNMENT),
    (dict(sa=A16 + 2), rq.RESPIN_ERR_ALIGNMENT),
    (dict(sw=A16B + 4), rq.RESPIN_ERR_ALIGNMENT),
])
def test_gemm_validation(kw, want):
    assert gemm(**kw) == want
    assert rq.last_error()


def test_gemm_empty_is_noop():
    assert gemm(N=0, qa=None, out=None) == rq.RESPIN_OK


def test_gemm_i32_validation():
    assert rq.lib.w4a4_gemm_i32(A16, A16B, 4, 96, 32, A16, None) == \
        rq.RESPIN_ERR_UNSUPPORTED
    assert rq.lib.w4a4_gemm_i32(MIS, A16B, 4, 128, 32, A16, None) == \
        rq.RESPIN_ERR_ALIGNMENT


def test_fault_hook_launch(monkeypatch):
    monkeypatch.setenv("RESPIN_FAULT", "launch")
    assert gemm() == rq.RESPIN_ERR_CUDA
    assert "injected" in rq.last_error()
    with pytest.raises(rq.RespinError):
        rq._check(gemm())


def test_last_error_cleared_on_success():
    gemm(K=100)
    assert rq.last_error()
    assert gemm(N=0) == rq.RESPIN_OK
    assert rq.last_error() == ""


def test_device_status_null():
    assert rq.lib.respin_device_status(None) == rq.RESPIN_ERR_INVALID_ARG


def test_selftest_limit_validation():
    assert rq.lib.respin_selftest_wait_limit(0, None) == rq.RESPIN_ERR_INVALID_ARG
    assert rq.lib.respin_selftest_wait_limit(2000001, None) == rq.RESPIN_ERR_INVALID_ARG
    assert "limit_us" in rq.last_error()


def test_gemm_rowmax_validation():
    f = rq.lib.w4a4_gemm_rowmax
    # no rowmax buffer
    assert f(A16, A16, A16B, A16B, 256, 256, 32, A16, None, None) == rq.RESPIN_ERR_INVALID_ARG
    # few tokens: the weight-streaming kernel writes no maxima
    assert f(A16, A16, A16B, A16B, 128, 256, 32, A16, A16, None) == rq.RESPIN_ERR_UNSUPPORTED
    # misaligned maxima buffer
    assert f(A16, A16, A16B, A16B, 256, 256, 32, A16, A16 + 2, None) == rq.RESPIN_ERR_ALIGNMENT
    assert f(A16, A16, A16B, A16B, 256, 100, 32, A16, A16, None) == rq.RESPIN_ERR_UNSUPPORTED
    assert rq.last_error()


def test_quantize_rowmax_validation():
    f = rq.lib.respin_quantize_rowmax
    assert f(A16, A16, 4, 300, A16, A16, 0, None) == rq.RESPIN_ERR_UNSUPPORTED      # D % 256
    assert f(A16, A16, -1, 256, A16, A16, 0, None) == rq.RESPIN_ERR_INVALID_ARG      # N < 0
    assert f(A16, A16, 0, 256, A16, A16, 0, None) == rq.RESPIN_OK                   # N == 0
    assert f(None, A16, 4, 256, A16, A16, 0, None) == rq.RESPIN_ERR_INVALID_ARG
    assert f(MIS, A16, 4, 256, A16, A16, 0, None) == rq.RESPIN_ERR_ALIGNMENT
    assert f(A16, A16, 4, 256, A16, A16, 8, None) == rq.RESPIN_ERR_INVALID_ARG       # unknown flag
    assert rq.last_error()
