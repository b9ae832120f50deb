"""The C++ oracle (oracle/respin_oracle_native.cpp) against what pins it: the
hand-worked quantizer cases, pure-Python brute force on tiny inputs, naive
integer loops and a selection-matrix GEMM, and bit equality with the numpy
oracle on the pages' workload shapes (no GPU)."""
import json
import os

import numpy as np
import pytest

import oracle as O
import workloads as W
from oracle import native as N

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def bits_of(values):
    return O.bf16_bits(np.asarray(values, np.float64))


def test_quantizer_golden_cases_native():
    gold = json.load(open(os.path.join(GOLDEN, "quantizer_cases.json")))
    for key, qmax in (("tokens", 7), ("int3_tokens", 3)):
        for t in gold[key]:
            x = bits_of([t["g"]])
            _, hb, codes, scale = N.boundary_reference(x, None, np.zeros((x.shape[1], 0), np.float32),
                                                       np.zeros((x.shape[1], 0), np.float32), qmax)
            assert np.array_equal(hb, x)
            assert codes[0].tolist() == t["codes"]
            assert scale[0] == np.float32(t["scale"])
    for p in gold["packing"]:
        assert N.pack(np.array([p["codes"]], np.int8))[0].tolist() == p["bytes"]


def test_boundary_brute_force_tiny():
    """D = 16, r = 2: the fix written out as Python loops over exact floats."""
    rs = np.random.default_rng(7)
    D, r, n = 16, 2, 3
    x = bits_of(rs.standard_normal((n, D)))
    res = bits_of(rs.standard_normal((n, D)) * 3)
    U = rs.standard_normal((D, r)).astype(np.float32)
    V = rs.standard_normal((D, r)).astype(np.float32)
    h64, hb, _, _ = N.boundary_reference(x, res, U, V)
    Uq, Vq = O.round_to_bf16(U), O.round_to_bf16(V)
    xf, rf = O.bf16_bits_to_f32(x).astype(float), O.bf16_bits_to_f32(res).astype(float)
    for t in range(n):
        for d in range(D):
            corr = 0.0
            for j in range(r):
                y = sum(rf[t, e] * Uq[e, j] for e in range(D))
                corr += y * Vq[d, j]
            want = (rf[t, d] + xf[t, d]) + corr
            assert abs(h64[t, d] - want) <= 1e-12 * max(1.0, abs(want))


@pytest.mark.parametrize("name,N_,qmax", [("tiny", None, 7), ("llama2_7b", 48, 7), ("llama2_7b", 48, 3),
                                          ("llama2_70b", 8, 7)])
def test_boundary_equals_numpy_oracle(name, N_, qmax):
    fx = W.workload_fixture(name, N=N_) if N_ else W.workload_fixture(name)
    import torch
    xb = fx.x.view(torch.int16).numpy().view(np.uint16)
    rb = fx.residual.view(torch.int16).numpy().view(np.uint16)
    U32, V32 = fx.U.astype(np.float32), fx.V.astype(np.float32)
    h64, hb, codes, scale = N.boundary_reference(xb, rb, U32, V32, qmax)
    h64o, hbo, codeso, scaleo = O.boundary_reference(fx.x.float().numpy(), fx.residual.float().numpy(),
                                                     U32, V32, qmax)
    assert np.max(np.abs(h64 - h64o) / np.maximum(np.abs(h64o), 1e-6)) <= 1e-12
    assert np.array_equal(hb, hbo)
    assert np.array_equal(codes, codeso)
    assert np.array_equal(scale.view(np.uint32), scaleo.view(np.uint32))


def test_gemm_naive_loops_and_epilogue():
    rs = np.random.default_rng(13)
    Nn, K, O_ = 5, 64, 7
    qa = W.int4_packed_random(Nn, K, 1, W.TID_ACODES)
    qw = W.int4_packed_random(O_, K, 1, W.TID_WEIGHTS)
    sa = rs.uniform(0.01, 1, Nn).astype(np.float32)
    sw = rs.uniform(0.01, 1, O_).astype(np.float32)
    acc, out = N.w4a4_gemm(qa, sa, qw, sw)
    a, w = O.unpack_int4(qa), O.unpack_int4(qw)
    for n in range(Nn):
        for o in range(O_):
            assert acc[n, o] == sum(int(a[n, k]) * int(w[o, k]) for k in range(K))
    assert np.array_equal(out, O.w4a4_epilogue_bits(acc, sa, sw))


def test_gemm_selection_and_extremes():
    Nn, K, O_ = 9, 256, 12
    qa = W.int4_packed_random(Nn, K, 2, W.TID_ACODES)
    sel = np.random.default_rng(3).integers(0, K, O_)
    cw = np.zeros((O_, K), np.int8)
    cw[np.arange(O_), sel] = 1
    acc, _ = N.w4a4_gemm(qa, None, O.pack_int4(cw), None)
    assert np.array_equal(acc, O.unpack_int4(qa)[:, sel].astype(np.int64))
    full = np.full((2, K // 2), 0x88, np.uint8)
    acc2, _ = N.w4a4_gemm(full, None, full, None)
    assert np.all(acc2 == 64 * K)


def test_gemm_equals_numpy_oracle_workload_rows():
    K, O_ = 4096, 256
    qa = W.int4_packed_random(16, K, 0, W.TID_ACODES)
    qw = W.int4_packed_random(O_, K, 0, W.TID_WEIGHTS)
    sa = W.activation_scales(16, 0)
    sw = W.weight_scales(O_, K, 0)
    acc, out = N.w4a4_gemm(qa, sa, qw, sw)
    ref = O.w4a4_acc(qa, qw)
    assert np.array_equal(acc, ref)
    assert np.array_equal(out, O.w4a4_epilogue_bits(ref, sa, sw))


def test_subspace_boundary_brute_force_tiny():
    """D = 16, r = 4, stored subspace form: the three steps of zh §2.2 written
    out as Python loops over the plan's rounded values."""
    rs = np.random.default_rng(17)
    D, r, n = 16, 4, 3
    x = bits_of(rs.standard_normal((n, D)))
    res = bits_of(rs.standard_normal((n, D)))
    Q = np.linalg.qr(rs.standard_normal((D, r)))[0].astype(np.float32)
    R = (np.eye(r) + 0.2 * rs.standard_normal((r, r))).astype(np.float32)
    h64, hb, codes, scale = N.boundary_reference_subspace(x, res, Q, R)
    Qq = O.round_to_bf16(Q)
    M = [[float(np.float32(float(R[i, j]) - (1.0 if i == j else 0.0))) for j in range(r)] for i in range(r)]
    xf, rf = O.bf16_bits_to_f32(x), O.bf16_bits_to_f32(res)
    for t in range(n):
        y = [sum(float(rf[t, d]) * float(Qq[d, j]) for d in range(D)) for j in range(r)]
        z = [sum(y[j] * M[i][j] for j in range(r)) for i in range(r)]
        for d in range(D):
            want = float(xf[t, d]) + float(rf[t, d]) + sum(z[i] * float(Qq[d, i]) for i in range(r))
            assert abs(h64[t, d] - want) <= 1e-13 * max(1.0, abs(want))
    assert np.array_equal(hb, O.bf16_bits(h64))


@pytest.mark.parametrize("name", ["tiny", "llama2_7b"])
def test_subspace_native_matches_numpy(name):
    fx = W.workload_fixture(name, N=24)
    Qr, R = W.subspace_factors(fx.Q, fx.theta, fx.r)
    Q32, R32 = Qr.astype(np.float32), R.astype(np.float32)
    xb = O.bf16_bits(fx.x.float().numpy())
    rb = O.bf16_bits(fx.residual.float().numpy())
    a = N.boundary_reference_subspace(xb, rb, Q32, R32)
    b = O.boundary_reference_subspace(fx.x.float().numpy(), fx.residual.float().numpy(), Q32, R32)
    assert np.max(np.abs(a[0] - b[0])) <= 1e-12 * np.max(np.abs(b[0]))
    assert np.array_equal(a[1], b[1])
    assert np.array_equal(a[2], b[2])
    assert np.array_equal(a[3].view(np.uint32), b[3].view(np.uint32))
