"""Python binding of the ReSpinQuant block-boundary library (librespin.so).

Argument marshalling only: every step of the path runs in the CUDA kernels
behind the C ABI declared in include/respin.h. torch tensors supply device
memory and the current CUDA stream. There is no CPU fallback: if the built
library is missing, importing this package raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librespin.so")

RESPIN_OK = 0
RESPIN_ERR_INVALID_ARG = 1
RESPIN_ERR_ALIGNMENT = 2
RESPIN_ERR_UNSUPPORTED = 3
RESPIN_ERR_CUDA = 4
RESPIN_ERR_OOM = 5
RESPIN_ERR_DEVICE_CHECK = 6
RESPIN_H_FP32_DEBUG = 1
RESPIN_ACT_INT3 = 2

# Every entry point include/respin.h declares (checked by the tests).
EXPORTED = ("respin_plan_create", "respin_plan_create_subspace", "respin_plan_destroy",
            "respin_boundary_forward", "w4a4_gemm", "w4a4_gemm_i32",
            "w4a4_gemm_rowmax", "respin_quantize_rowmax",
            "respin_factors_from_subspace", "respin_factors_from_transition",
            "respin_fuse_weight", "respin_quantize_weight",
            "respin_device_status", "respin_selftest_wait_limit",
            "respin_last_error", "respin_version")


class RespinError(RuntimeError):
    """A library call returned a status other than RESPIN_OK."""

    def __init__(self, status: int, message: str):
        super().__init__(f"respin status {status}: {message}")
        self.status = status
        self.message = message


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python rotation_post_quantization_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, u32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint
    fp = ctypes.POINTER(ctypes.c_float)
    lib.respin_plan_create.argtypes = [ctypes.POINTER(vp), i32, i32, fp, fp, u32]
    lib.respin_plan_create_subspace.argtypes = [ctypes.POINTER(vp), i32, i32, fp, fp, u32]
    lib.respin_plan_destroy.argtypes = [vp]
    lib.respin_boundary_forward.argtypes = [vp, vp, vp, i32, vp, vp, vp, vp]
    lib.w4a4_gemm.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp, vp]
    lib.w4a4_gemm_i32.argtypes = [vp, vp, i32, i32, i32, vp, vp]
    lib.w4a4_gemm_rowmax.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp, vp, vp]
    lib.respin_quantize_rowmax.argtypes = [vp, vp, i32, i32, vp, vp, u32, vp]
    dp = ctypes.POINTER(ctypes.c_double)
    lib.respin_factors_from_subspace.argtypes = [i32, i32, fp, fp, fp, fp]
    lib.respin_factors_from_transition.argtypes = [i32, i32, fp, ctypes.c_double, fp, fp, dp]
    lib.respin_fuse_weight.argtypes = [i32, i32, fp, fp, fp, fp]
    lib.respin_quantize_weight.argtypes = [i32, i32, fp, i32, vp, fp]
    lib.respin_device_status.argtypes = [ctypes.POINTER(ctypes.c_int)]
    lib.respin_selftest_wait_limit.argtypes = [u32, vp]
    for name in EXPORTED[:-2]:
        getattr(lib, name).restype = ctypes.c_int
    lib.respin_last_error.restype = ctypes.c_char_p
    lib.respin_last_error.argtypes = []
    lib.respin_version.restype = ctypes.c_char_p
    lib.respin_version.argtypes = []
    return lib


lib = _load()


def _check(status: int) -> None:
    if status != RESPIN_OK:
        raise RespinError(status, lib.respin_last_error().decode())


def last_error() -> str:
    return lib.respin_last_error().decode()


def version() -> str:
    return lib.respin_version().decode()


def _ptr(t):
    """Device pointer of a tensor (or None), as an int for ctypes."""
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


class Plan:
    """respin_plan_create / respin_plan_destroy: one block boundary's factors."""

    def __init__(self, D: int, r: int, U_r=None, V_r=None, flags: int = 0):
        self.D, self.r, self.flags = int(D), int(r), int(flags)
        self.handle = ctypes.c_void_p()
        fp = ctypes.POINTER(ctypes.c_float)
        U = V = None
        if U_r is not None:
            U = np.ascontiguousarray(U_r, dtype=np.float32)
            V = np.ascontiguousarray(V_r, dtype=np.float32)
            if U.shape != (self.D, self.r) or V.shape != (self.D, self.r):
                raise ValueError("U_r and V_r must be [D, r]")
        up = U.ctypes.data_as(fp) if U is not None else None
        vp_ = V.ctypes.data_as(fp) if V is not None else None
        _check(lib.respin_plan_create(ctypes.byref(self.handle), self.D,
                                      self.r, up, vp_, self.flags))

    def destroy(self) -> None:
        if self.handle:
            h, self.handle = self.handle, ctypes.c_void_p()
            _check(lib.respin_plan_destroy(h))

    def __del__(self):
        try:
            self.destroy()
        except Exception:
            pass


class SubspacePlan(Plan):
    """respin_plan_create_subspace: a boundary from its stored subspace form
    (host fp32 basis Q [D, r] and rotation R_sub [r, r])."""

    def __init__(self, D: int, r: int, Q, R_sub, flags: int = 0):
        self.D, self.r, self.flags = int(D), int(r), int(flags)
        self.handle = ctypes.c_void_p()
        fp = ctypes.POINTER(ctypes.c_float)
        Qa = np.ascontiguousarray(Q, dtype=np.float32)
        Ra = np.ascontiguousarray(R_sub, dtype=np.float32)
        if Qa.shape != (self.D, self.r) or Ra.shape != (self.r, self.r):
            raise ValueError("Q must be [D, r] and R_sub [r, r]")
        _check(lib.respin_plan_create_subspace(ctypes.byref(self.handle), self.D, self.r,
                                               Qa.ctypes.data_as(fp), Ra.ctypes.data_as(fp),
                                               self.flags))


def respin_plan_create(D, r, U_r=None, V_r=None, flags=0) -> Plan:
    return Plan(D, r, U_r, V_r, flags)


def respin_plan_create_subspace(D, r, Q, R_sub, flags=0) -> SubspacePlan:
    return SubspacePlan(D, r, Q, R_sub, flags)


def respin_plan_destroy(plan: Plan) -> None:
    plan.destroy()


def respin_boundary_forward(plan: Plan, x, residual, h_out, q_packed, scale,
                            stream=None) -> None:
    """h' = residual (I + U_r V_r^T) + x, then per-token INT4 codes and scales
    (3-bit codes in the same nibbles for a plan made with RESPIN_ACT_INT3).

    x, residual, h_out: [N, D] CUDA tensors (bf16; h_out fp32 for a plan made
    with RESPIN_H_FP32_DEBUG; residual / h_out may be None); q_packed: uint8
    [N, D/2]; scale: fp32 [N].
    """
    N = int(x.shape[0]) if x is not None else 0
    _check(lib.respin_boundary_forward(
        plan.handle, _ptr(x), _ptr(residual), N, _ptr(h_out), _ptr(q_packed),
        _ptr(scale), _stream(stream)))


def w4a4_gemm(q_act, scale_act, q_w, scale_w, out, stream=None) -> None:
    """out[N, O] (bf16) = (acc * scale_act[n]) * scale_w[o], acc exact int."""
    N, K2 = q_act.shape
    O = q_w.shape[0]
    _check(lib.w4a4_gemm(_ptr(q_act), _ptr(scale_act), _ptr(q_w),
                         _ptr(scale_w), int(N), int(2 * K2), int(O), _ptr(out),
                         _stream(stream)))


def w4a4_gemm_i32(q_act, q_w, acc_out, stream=None) -> None:
    """acc_out[N, O] (int32) = exact integer dot products of the codes."""
    N, K2 = q_act.shape
    O = q_w.shape[0]
    _check(lib.w4a4_gemm_i32(_ptr(q_act), _ptr(q_w), int(N), int(2 * K2),
                             int(O), _ptr(acc_out), _stream(stream)))


def w4a4_gemm_rowmax(q_act, scale_act, q_w, scale_w, out, rowmax, stream=None) -> None:
    """w4a4_gemm, and rowmax[N, ceil(O / 256)] = max |out| per token and
    256-channel tile (N > 128)."""
    N, K2 = q_act.shape
    O = q_w.shape[0]
    _check(lib.w4a4_gemm_rowmax(_ptr(q_act), _ptr(scale_act), _ptr(q_w), _ptr(scale_w),
                                int(N), int(2 * K2), int(O), _ptr(out), _ptr(rowmax),
                                _stream(stream)))


def respin_quantize_rowmax(u, rowmax, q_packed, scale, flags: int = 0, stream=None) -> None:
    """Per-token codes and scales of bf16 u [N, D] from its partial row
    maxima rowmax [N, D / 256]."""
    N, D = u.shape
    _check(lib.respin_quantize_rowmax(_ptr(u), _ptr(rowmax), int(N), int(D), _ptr(q_packed),
                                      _ptr(scale), ctypes.c_uint(flags), _stream(stream)))


def _host_f32(a, shape, name):
    a = np.ascontiguousarray(a, dtype=np.float32)
    if a.shape != shape:
        raise ValueError(f"{name} must have shape {shape}")
    return a


def respin_factors_from_subspace(Q, R_sub):
    """(U_r, V_r) = (Q, Q (R_sub - I)) for the plan, from the subspace form
    (host fp32 arrays Q [D, r] and R_sub [r, r])."""
    Q = np.ascontiguousarray(Q, dtype=np.float32)
    D, r = Q.shape
    R = _host_f32(R_sub, (r, r), "R_sub")
    fp = ctypes.POINTER(ctypes.c_float)
    U = np.empty((D, r), np.float32)
    V = np.empty((D, r), np.float32)
    _check(lib.respin_factors_from_subspace(D, r, Q.ctypes.data_as(fp), R.ctypes.data_as(fp),
                                            U.ctypes.data_as(fp), V.ctypes.data_as(fp)))
    return U, V


def respin_factors_from_transition(T, r: int, gap_tol: float = 1e-6):
    """(U_r, V_r, sigma) = top-r factors of T - I for the plan (host fp32
    T [D, D]); sigma holds s_1 .. s_(r+1). Raises RespinError
    (RESPIN_ERR_UNSUPPORTED) when s_r - s_(r+1) <= gap_tol s_1."""
    T = np.ascontiguousarray(T, dtype=np.float32)
    D = T.shape[0]
    if T.shape != (D, D):
        raise ValueError("T must be square")
    fp = ctypes.POINTER(ctypes.c_float)
    U = np.empty((D, int(r)), np.float32)
    V = np.empty((D, int(r)), np.float32)
    sig = np.zeros(int(r) + 1, np.float64)
    _check(lib.respin_factors_from_transition(D, int(r), T.ctypes.data_as(fp), float(gap_tol),
                                              U.ctypes.data_as(fp), V.ctypes.data_as(fp),
                                              sig.ctypes.data_as(ctypes.POINTER(ctypes.c_double))))
    return U, V, sig


def respin_fuse_weight(W, R_in, R_out=None):
    """W_fused = R_out^T W R_in (or W R_in) for host fp32 arrays W [O, K],
    R_in [K, K], R_out [O, O]; float64 products on the host."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    O, K = W.shape
    Ri = _host_f32(R_in, (K, K), "R_in")
    Ro = None if R_out is None else _host_f32(R_out, (O, O), "R_out")
    fp = ctypes.POINTER(ctypes.c_float)
    out = np.empty((O, K), np.float32)
    _check(lib.respin_fuse_weight(O, K, W.ctypes.data_as(fp), Ri.ctypes.data_as(fp),
                                  None if Ro is None else Ro.ctypes.data_as(fp), out.ctypes.data_as(fp)))
    return out


def respin_quantize_weight(W, qmax: int = 7):
    """(packed codes uint8 [O, K/2], scales fp32 [O]) of host fp32 W [O, K],
    symmetric per output channel (qmax 7: INT4, 3: INT3)."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    O, K = W.shape
    q = np.empty((O, K // 2), np.uint8)
    sc = np.empty(O, np.float32)
    fp = ctypes.POINTER(ctypes.c_float)
    _check(lib.respin_quantize_weight(O, K, W.ctypes.data_as(fp), int(qmax), q.ctypes.data,
                                      sc.ctypes.data_as(fp)))
    return q, sc


def respin_selftest_wait_limit(limit_us: int, stream=None) -> None:
    """Enqueue the failure-detection self test: a bounded wait that nothing
    completes gives up after limit_us microseconds and records site 901."""
    _check(lib.respin_selftest_wait_limit(int(limit_us), _stream(stream)))


def respin_device_status() -> int:
    """Synchronize and return (and clear) the device status word."""
    code = ctypes.c_int(0)
    st = lib.respin_device_status(ctypes.byref(code))
    if st not in (RESPIN_OK, RESPIN_ERR_DEVICE_CHECK):
        _check(st)
    return code.value
