"""ctypes front end of the C++ oracle (respin_oracle_native.cpp).

TEST INFRASTRUCTURE ONLY: only tests/, the smoke check and the benchmark's
CPU-baseline / reference leg may use it. It computes what respin_oracle.py
computes (same readings of the explainer pages), in plain single-threaded
C++ loops; the tests pin it to hand-worked cases, brute force and the numpy
oracle. The library is built in place with g++ on first use (or by build()).
"""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "respin_oracle_native.cpp")
LIB_PATH = os.path.join(HERE, "librespin_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (-O2, no contraction, no fast-math)."""
    if not force and os.path.exists(LIB_PATH) and os.path.getmtime(LIB_PATH) >= os.path.getmtime(SRC):
        return LIB_PATH
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        raise RuntimeError("no C++ compiler for the native oracle")
    tmp = LIB_PATH + ".tmp"
    subprocess.run([cxx, "-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off",
                    "-fno-fast-math", "-o", tmp, SRC], check=True, capture_output=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB_PATH)
        vp, i32 = ctypes.c_void_p, ctypes.c_int
        L.oracle_boundary.argtypes = [i32, i32, i32, vp, vp, vp, vp, i32, vp, vp, vp, vp]
        L.oracle_boundary_subspace.argtypes = [i32, i32, i32, vp, vp, vp, vp, i32, vp, vp, vp, vp]
        L.oracle_pack.argtypes = [i32, i32, vp, vp]
        L.oracle_w4a4.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp]
        for f in (L.oracle_boundary, L.oracle_boundary_subspace, L.oracle_pack, L.oracle_w4a4):
            f.restype = i32
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def boundary_reference(x_bits, res_bits, U32, V32, qmax: int = 7, want_h64: bool = True):
    """(h64 or None, h bf16 bits, codes int8, scale float32) for bf16 bit
    arrays x_bits, res_bits ([N, D] uint16; res_bits may be None) and float32
    factors [D, r]."""
    x = np.ascontiguousarray(x_bits, np.uint16)
    N, D = x.shape
    res = None if res_bits is None else np.ascontiguousarray(res_bits, np.uint16)
    U = np.ascontiguousarray(U32, np.float32)
    V = np.ascontiguousarray(V32, np.float32)
    r = U.shape[1] if U.ndim == 2 else 0
    h64 = np.empty((N, D), np.float64) if want_h64 else None
    hb = np.empty((N, D), np.uint16)
    codes = np.empty((N, D), np.int8)
    scale = np.empty(N, np.float32)
    st = lib().oracle_boundary(N, D, r, _p(x), _p(res), _p(U), _p(V), int(qmax), _p(h64), _p(hb),
                               _p(codes), _p(scale))
    if st != 0:
        raise ValueError("oracle_boundary: bad arguments")
    return h64, hb, codes, scale


def boundary_reference_subspace(x_bits, res_bits, Q32, R32, qmax: int = 7, want_h64: bool = True):
    """As boundary_reference, for a plan in the stored subspace form: float32
    basis Q [D, r] and rotation R_sub [r, r] (zh §2.2)."""
    x = np.ascontiguousarray(x_bits, np.uint16)
    N, D = x.shape
    res = None if res_bits is None else np.ascontiguousarray(res_bits, np.uint16)
    Q = np.ascontiguousarray(Q32, np.float32)
    R = np.ascontiguousarray(R32, np.float32)
    r = Q.shape[1] if Q.ndim == 2 else 0
    h64 = np.empty((N, D), np.float64) if want_h64 else None
    hb = np.empty((N, D), np.uint16)
    codes = np.empty((N, D), np.int8)
    scale = np.empty(N, np.float32)
    st = lib().oracle_boundary_subspace(N, D, r, _p(x), _p(res), _p(Q), _p(R), int(qmax), _p(h64),
                                        _p(hb), _p(codes), _p(scale))
    if st != 0:
        raise ValueError("oracle_boundary_subspace: bad arguments")
    return h64, hb, codes, scale


def pack(codes) -> np.ndarray:
    c = np.ascontiguousarray(codes, np.int8)
    rows, K = c.shape
    out = np.empty((rows, K // 2), np.uint8)
    if lib().oracle_pack(rows, K, _p(c), _p(out)) != 0:
        raise ValueError("oracle_pack: bad arguments")
    return out


def w4a4_gemm(qa, sa, qw, sw):
    """(acc int64 [N, O], bf16 bits [N, O] of the binary32 epilogue, or None
    when sa / sw are None)."""
    qa = np.ascontiguousarray(qa, np.uint8)
    qw = np.ascontiguousarray(qw, np.uint8)
    N, K2 = qa.shape
    O = qw.shape[0]
    acc = np.empty((N, O), np.int64)
    out = None
    sa_ = sw_ = None
    if sa is not None:
        sa_ = np.ascontiguousarray(sa, np.float32)
        sw_ = np.ascontiguousarray(sw, np.float32)
        out = np.empty((N, O), np.uint16)
    st = lib().oracle_w4a4(N, 2 * K2, O, _p(qa), _p(sa_), _p(qw), _p(sw_), _p(acc), _p(out))
    if st == -2:
        raise ValueError("accumulator not exactly representable in binary32")
    if st != 0:
        raise ValueError("oracle_w4a4: bad arguments")
    return acc, out
