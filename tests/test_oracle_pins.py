"""Pins for the CPU oracle: each checks it against something other than itself.

Sources are the gist.science explainer pages of "ReSpinQuant: Efficient
Layer-Wise LLM Quantization via Subspace Residual Rotation Approximation",
cited by language and section.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fixture(D, k, nu, seed=0):
    Q = W.orthonormal_basis(D, k, seed)
    th = W.plane_angles(k, nu)
    R_in, R_out = O.rotation_pair(Q, th)
    T = O.transition_matrix(R_in, R_out)
    return Q, th, T


# ---------------------------------------------------------------- rotations

@pytest.mark.parametrize("D", [2, 16, 256])
def test_hadamard_matches_library(D):
    # Sylvester construction vs scipy's Hadamard matrix (zh §2.1 init).
    np.testing.assert_allclose(O.hadamard(D),
                               scipy.linalg.hadamard(D) / math.sqrt(D),
                               rtol=0, atol=0)
    H = O.hadamard(D)
    np.testing.assert_allclose(H @ H.T, np.eye(D), atol=1e-13)


@pytest.mark.parametrize("D,k,nu", [(256, 8, 0.05), (1024, 64, 0.1),
                                    (512, 128, 1.0)])
def test_transition_matrix_orthogonal(D, k, nu):
    # T = R_out^T R_in is orthogonal (both factors are rotations).
    _, _, T = _fixture(D, k, nu)
    assert np.max(np.abs(T.T @ T - np.eye(D))) <= 1e-5
    assert np.max(np.abs(T.T @ T - np.eye(D))) <= 1e-12


def test_transition_identity_for_equal_rotations():
    # Global rotation: R_in = R_out gives T = I (it §2B; nl §2B).
    rs = np.random.default_rng(5)
    R, _ = np.linalg.qr(rs.standard_normal((128, 128)))
    np.testing.assert_allclose(O.transition_matrix(R, R), np.eye(128),
                               atol=1e-13)
    Q = W.orthonormal_basis(64, 8)
    R_in, R_out = O.rotation_pair(Q, np.zeros(4))
    np.testing.assert_allclose(O.transition_matrix(R_in, R_out), np.eye(64),
                               atol=1e-15)


def test_transition_direction_matters():
    # A transposed operand must not pass: R_out R_in^T differs from R_out^T R_in.
    _, _, T = _fixture(64, 8, 1.0)
    Q = W.orthonormal_basis(64, 8)
    R_in, R_out = O.rotation_pair(Q, W.plane_angles(8, 1.0))
    assert not np.allclose(R_out @ R_in.T, T, atol=1e-3)
    np.testing.assert_allclose(O.transition_matrix(R_in, R_out), T, atol=0)


def test_skew_norm_is_nu():
    # Fixture: Frobenius norm of the generator equals nu.
    Q = W.orthonormal_basis(300, 64)
    A = O.skew_from_planes(Q, W.plane_angles(64, 0.1))
    assert abs(np.linalg.norm(A) - 0.1) < 1e-14
    np.testing.assert_allclose(A, -A.T, atol=0)


# ---------------------------------------------------------------- SVD / factors

@pytest.mark.parametrize("D,k", [(256, 8), (1024, 64)])
def test_singular_values_closed_form(D, k):
    # sigma of T - I: each plane gives 2|sin(theta/2)| twice, the rest is 0.
    Q, th, T = _fixture(D, k, 0.1)
    s = np.linalg.svd(T - np.eye(D), compute_uv=False)
    want = np.sort(np.repeat(2 * np.abs(np.sin(th / 2)), 2))[::-1]
    np.testing.assert_allclose(s[:k], want, rtol=1e-10, atol=1e-13)
    assert np.max(s[k:]) < 1e-12


@pytest.mark.parametrize("D,k,r", [(256, 8, 8), (512, 64, 32), (1024, 64, 16)])
def test_fixture_factors_match_svd(D, k, r):
    # The fixture's closed-form factors equal the library SVD's top-r product.
    Q, th, T = _fixture(D, k, 0.1)
    U, V = W.lowrank_factors(Q, th, r)
    Us, Vs, _ = O.top_r_factors(T, r)
    np.testing.assert_allclose(U @ V.T, Us @ Vs.T, atol=1e-12)
    # and the unique product is what the pages' truncation means:
    # ||dT - U V^T||_F^2 = sum of the dropped sigma^2
    s = np.linalg.svd(T - np.eye(D), compute_uv=False)
    err = np.linalg.norm(T - np.eye(D) - U @ V.T) ** 2
    assert abs(err - np.sum(s[r:] ** 2)) < 1e-12


def test_exact_rank_equals_dense():
    # Delta T built exactly rank r: the rank-r path equals the dense T product.
    D, k = 256, 8
    Q, th, T = _fixture(D, k, 0.05)
    U, V = W.lowrank_factors(Q, th, k)
    rs = np.random.default_rng(1)
    res, x = rs.standard_normal((7, D)), rs.standard_normal((7, D))
    np.testing.assert_allclose(O.boundary_fp64(x, res, U, V),
                               O.dense_boundary_fp64(x, res, T),
                               rtol=0, atol=1e-12)


def test_full_rank_reproduces_dense():
    # r = D: the approximation reproduces h T up to rounding.
    D = 64
    Q, th, T = _fixture(D, D, 1.0)
    U, V, _ = O.top_r_factors(T, D)
    rs = np.random.default_rng(2)
    res, x = rs.standard_normal((5, D)), rs.standard_normal((5, D))
    np.testing.assert_allclose(O.boundary_fp64(x, res, U, V),
                               O.dense_boundary_fp64(x, res, T), atol=1e-12)


@pytest.mark.parametrize("r", [16, 32, 48, 64])
def test_eckart_young_bound(r):
    # ||h_r - h_dense|| <= sigma_{r+1} ||res|| per token (rank-r truncation).
    D, k = 512, 128
    Q, th, T = _fixture(D, k, 0.1)
    U, V = W.lowrank_factors(Q, th, r)
    s = np.linalg.svd(T - np.eye(D), compute_uv=False)
    rs = np.random.default_rng(3)
    res, x = rs.standard_normal((16, D)), rs.standard_normal((16, D))
    diff = O.boundary_fp64(x, res, U, V) - O.dense_boundary_fp64(x, res, T)
    lhs = np.linalg.norm(diff, axis=1)
    rhs = s[r] * np.linalg.norm(res, axis=1)
    assert np.all(lhs <= rhs * (1 + 1e-9) + 1e-12)
    assert np.max(lhs) > 0


def test_truncated_fix_preserves_norm():
    # Block-aligned truncation keeps I + U V^T orthogonal: ||res + corr|| = ||res||.
    D = 512
    Q, th, _ = _fixture(D, 64, 0.3)
    U, V = W.lowrank_factors(Q, th, 32)
    rs = np.random.default_rng(4)
    res = rs.standard_normal((9, D))
    h = O.boundary_fp64(np.zeros_like(res), res, U, V)
    np.testing.assert_allclose(np.linalg.norm(h, axis=1),
                               np.linalg.norm(res, axis=1), rtol=1e-13)


def test_brute_force_loops_tiny():
    # Pure-Python dense O(D^2) loops vs the rank-r oracle on a tiny case.
    D, k = 16, 16
    Q, th, T = _fixture(D, k, 0.7)
    U, V = W.lowrank_factors(Q, th, k)
    rs = np.random.default_rng(6)
    res, x = rs.standard_normal((3, D)), rs.standard_normal((3, D))
    ref = np.zeros((3, D))
    for n in range(3):
        for j in range(D):
            acc = x[n, j]
            for i in range(D):
                acc += res[n, i] * T[i, j]
            ref[n, j] = acc
    np.testing.assert_allclose(O.boundary_fp64(x, res, U, V), ref, atol=1e-12)


def test_subspace_form_equals_row_factor_form():
    # zh §2.2 column form x + Q (M Q^T x) == row form h + (h Q)(Q M)^T.
    D, r = 96, 12
    rs = np.random.default_rng(7)
    Q, _ = np.linalg.qr(rs.standard_normal((D, r)))
    M = 0.1 * rs.standard_normal((r, r))
    xs = rs.standard_normal((D, 5))
    col = O.subspace_residual_rotation(xs, Q, np.eye(r) + M)
    row = O.boundary_fp64(np.zeros((5, D)), xs.T, Q, Q @ M)
    np.testing.assert_allclose(col.T, row, atol=1e-13)
    # the transposed transform would be a different operator
    wrong = O.boundary_fp64(np.zeros((5, D)), xs.T, Q, Q @ M.T)
    assert not np.allclose(col.T, wrong, atol=1e-6)


def test_subspace_basis_reproduces_exact_rank_T():
    # Q from the SVD and M = Q^T dT Q reproduce an exactly rank-r T (column form).
    D, k = 128, 16
    _, _, T = _fixture(D, k, 0.2)
    Qb, M = O.subspace_basis(T, k)
    rs = np.random.default_rng(8)
    xs = rs.standard_normal((D, 4))
    np.testing.assert_allclose(
        O.subspace_residual_rotation(xs, Qb, np.eye(k) + M), T @ xs,
        atol=1e-12)


# ---------------------------------------------------------------- bfloat16

def test_bf16_rounding_matches_torch():
    rs = np.random.default_rng(9)
    with np.errstate(over="ignore"):   # some draws overflow to inf: filtered below
        big = (rs.standard_normal(2000) * 1e38).astype(np.float32)
    vals = [rs.standard_normal(20000).astype(np.float32),
            (rs.standard_normal(2000) * 1e-39).astype(np.float32),  # subnormal
            big,
            # exact ties: low 16 bits = 0x8000
            ((rs.integers(0, 2**15, 4000, dtype=np.uint32) << 16) | 0x8000
             ).astype(np.uint32).view(np.float32),
            np.array([0.0, -0.0, 1.0, -1.0, 3.3895314e38, 3.39e38],
                     np.float32)]
    for v in vals:
        v = v[np.isfinite(v)]
        want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16)
        want = want.numpy().view(np.uint16)
        got = O.bf16_bits(v)
        assert np.array_equal(got, want)


def test_bf16_roundtrip_exact():
    rs = np.random.default_rng(10)
    bits = rs.integers(0, 2**16, 5000).astype(np.uint16)
    f = O.bf16_bits_to_f32(bits)
    ok = np.isfinite(f)
    assert np.array_equal(O.bf16_bits(f[ok]), bits[ok])


# ---------------------------------------------------------------- quantizer

def test_quantizer_golden_cases():
    with open(os.path.join(GOLDEN, "quantizer_cases.json")) as fh:
        gold = json.load(fh)
    for t in gold["tokens"]:
        codes, scale = O.quantize_int4_per_token(np.array([t["g"]], np.float32))
        assert codes[0].tolist() == t["codes"]
        assert scale[0] == np.float32(t["scale"])
    for p in gold["packing"]:
        assert O.pack_int4(np.array(p["codes"])).tolist() == p["bytes"]
        assert O.unpack_int4(np.array(p["bytes"], np.uint8)).tolist() == p["codes"]
    for t in gold["int3_tokens"]:
        codes, scale = O.quantize_int3_per_token(np.array([t["g"]], np.float32))
        assert codes[0].tolist() == t["codes"]
        assert scale[0] == np.float32(t["scale"])


@pytest.mark.parametrize("qmax", [7, 3])
def test_quantizer_invariants(qmax):
    rs = np.random.default_rng(11)
    g = rs.standard_normal((64, 256)).astype(np.float32)
    g[:, 3] *= 50
    g[5] = 0.0
    codes, scale = O.quantize_per_token(g, qmax)
    assert codes.min() >= -qmax - 1 and codes.max() <= qmax
    nz = np.any(g != 0, axis=1)
    assert np.all(np.max(np.abs(codes[nz]), axis=1) == qmax)
    assert scale[5] == 0 and not np.any(codes[5])
    # dequantization error within half a step (plus binary32 slack), in fp64
    err = np.abs(g.astype(np.float64) - codes * scale[:, None].astype(np.float64))
    assert np.all(err <= scale[:, None] * (0.5 + 2e-6))
    # and the code is the nearest integer to g * qmax / amax up to that slack
    amax = np.max(np.abs(g), axis=1).astype(np.float64)
    t = g[nz] * (qmax / amax[nz, None])
    assert np.all(np.abs(t - codes[nz]) <= 0.5 + 1e-5)


def test_quantizer_int3_brute_force_nearest():
    """INT3 codes are the nearest of the 8 levels -4..3 to g*3/amax, brute
    force over the levels (ties, which have measure zero here, excluded)."""
    rs = np.random.default_rng(21)
    g = rs.standard_normal((32, 96)).astype(np.float32)
    codes, scale = O.quantize_int3_per_token(g)
    t = g.astype(np.float64) * (3.0 / np.max(np.abs(g), axis=1, keepdims=True))
    levels = np.arange(-4, 4)
    dist = np.abs(t[..., None] - levels)
    best = levels[np.argmin(dist, axis=-1)]
    srt = np.sort(dist, axis=-1)
    clear = srt[..., 1] - srt[..., 0] > 1e-5
    assert np.array_equal(codes[clear], best[clear])
    assert np.allclose(scale, np.max(np.abs(g), axis=1) / 3.0, rtol=2 ** -23)


@pytest.mark.parametrize("qmax", [7, 3])
def test_quantizer_tiny_amax_is_zero_token(qmax):
    g = np.array([[1e-38, -2e-38, 0.0, 0.0], [3e-38, 0, 0, 0]], np.float32)
    codes, scale = O.quantize_per_token(g, qmax)
    assert scale[0] == 0 and not codes[0].any()
    assert scale[1] > 0 and codes[1, 0] == qmax


def test_pack_roundtrip():
    rs = np.random.default_rng(12)
    c = rs.integers(-8, 8, (10, 64)).astype(np.int8)
    assert np.array_equal(O.unpack_int4(O.pack_int4(c)), c)
    b = rs.integers(0, 256, (10, 32)).astype(np.uint8)
    assert np.array_equal(O.pack_int4(O.unpack_int4(b)), b)


# ---------------------------------------------------------------- GEMM

def test_gemm_naive_loops():
    rs = np.random.default_rng(13)
    a = rs.integers(0, 256, (3, 8), dtype=np.uint8)
    w = rs.integers(0, 256, (5, 8), dtype=np.uint8)
    ca, cw = O.unpack_int4(a), O.unpack_int4(w)
    ref = [[sum(int(ca[n, k]) * int(cw[o, k]) for k in range(16))
            for o in range(5)] for n in range(3)]
    assert O.w4a4_acc(a, w).tolist() == ref


def test_gemm_fp64_form_matches_integer_definition():
    rs = np.random.default_rng(16)
    a = rs.integers(0, 256, (37, 256), dtype=np.uint8)
    w = rs.integers(0, 256, (29, 256), dtype=np.uint8)
    assert np.array_equal(O.w4a4_acc_fp64(a, w), O.w4a4_acc(a, w))
    ext_a = np.full((3, 64), 0x88, np.uint8)   # all -8: |acc| = 64 K
    assert np.all(O.w4a4_acc_fp64(ext_a, ext_a) == 64 * 128)


def test_gemm_selection_matrix():
    # One +1 per weight row selects one activation code: a gather.
    rs = np.random.default_rng(14)
    K, O_ = 64, 12
    a = rs.integers(0, 256, (4, K // 2), dtype=np.uint8)
    sel = rs.integers(0, K, O_)
    cw = np.zeros((O_, K), np.int8)
    cw[np.arange(O_), sel] = 1
    acc = O.w4a4_acc(a, O.pack_int4(cw))
    assert np.array_equal(acc, O.unpack_int4(a)[:, sel].astype(np.int64))


def test_gemm_epilogue():
    acc = np.array([[3, -5], [0, 100]], np.int64)
    sa = np.array([0.5, 2.0], np.float32)
    sw = np.array([2.0, 0.25], np.float32)
    bits = O.w4a4_epilogue_bits(acc, sa, sw)
    vals = O.bf16_bits_to_f32(bits)
    assert vals.tolist() == [[3.0, -0.625], [0.0, 50.0]]
    rs = np.random.default_rng(15)
    acc = rs.integers(-50000, 50000, (32, 48))
    sa = rs.uniform(0.1, 2, 32).astype(np.float32)
    sw = rs.uniform(1e-3, 1e-2, 48).astype(np.float32)
    out = O.bf16_bits_to_f32(O.w4a4_epilogue_bits(acc, sa, sw)).astype(np.float64)
    ref = O.w4a4_dequant_fp64(acc, sa, sw)
    assert np.linalg.norm(out - ref) / np.linalg.norm(ref) < 1e-2
    assert np.max(np.abs(out - ref) / np.maximum(np.abs(ref), 1e-30)) <= 2 ** -8


# ---------------------------------------------------------------- composite

def test_boundary_reference_pipeline():
    fx = W.workload_fixture("tiny")
    U32, V32 = fx.U.astype(np.float32), fx.V.astype(np.float32)
    x = fx.x.float().numpy()
    res = fx.residual.float().numpy()
    h64, hb, codes, scale = O.boundary_reference(x, res, U32, V32)
    # exact rank (k = r): with the plan's bfloat16 factors the result stays
    # close to the dense product per token; the correction term itself carries
    # the factors' bfloat16 precision (relative error of order 2^-8).
    R_in, R_out = O.rotation_pair(fx.Q, fx.theta)
    T = O.transition_matrix(R_in, R_out)
    dense = O.dense_boundary_fp64(x, res, T)
    tok = np.linalg.norm(h64 - dense, axis=1) / np.linalg.norm(dense, axis=1)
    assert np.max(tok) < 1e-4
    corr_d, corr_p = res @ T - res, h64 - res - x
    crel = (np.linalg.norm(corr_p - corr_d, axis=1)
            / np.linalg.norm(corr_d, axis=1))
    assert np.max(crel) < 1e-2
    assert codes.min() >= -7 and codes.max() <= 7
    assert np.all(np.max(np.abs(codes), axis=1) == 7)


# ---------------------------------------------------------------- page counts

def test_page_counts():
    with open(os.path.join(GOLDEN, "paper_counts.json")) as fh:
        g = json.load(fh)
    on = O.online_factor_params(g["layers"], g["D"], g["r"])
    assert on == 8388608
    assert round(on / 1e6, 1) == g["online_params_M"]
    tr = O.training_rotation_params(g["layers"], g["D"]) / 1e6
    assert round(tr + g["spinquant_training_params_M"], 1) == g["training_params_M"]


# ---------------------------------------------------------------- subspace form (device Q-form plans)

def test_subspace_row_form_equals_column_form():
    # zh §2.2 steps 1-3 in the row form (y = res Q, z = y M^T, res + z Q^T)
    # against the column-form function on the same vectors; the transposed
    # transform and a dropped step fail.
    D, r = 96, 12
    rs = np.random.default_rng(21)
    Q, _ = np.linalg.qr(rs.standard_normal((D, r)))
    M = 0.1 * rs.standard_normal((r, r))
    res, x = rs.standard_normal((5, D)), rs.standard_normal((5, D))
    col = O.subspace_residual_rotation(res.T, Q, np.eye(r) + M).T + x
    np.testing.assert_allclose(O.boundary_subspace_fp64(x, res, Q, M), col, atol=1e-13)
    assert not np.allclose(O.boundary_subspace_fp64(x, res, Q, M.T), col, atol=1e-6)
    assert not np.allclose(O.boundary_subspace_fp64(x, res, Q, np.zeros((r, r))), col, atol=1e-6)


@pytest.mark.parametrize("D,k,nu", [(256, 8, 0.05), (512, 32, 1.0)])
def test_subspace_fixture_exact_rank_equals_dense_T(D, k, nu):
    # Exact rank (r = k): the fixture's stored form (Q_r, R_sub) reproduces the
    # dense T = R_out^T R_in built independently through scipy's expm.
    Q, th, T = _fixture(D, k, nu)
    Qr, R = W.subspace_factors(Q, th, k)
    rs = np.random.default_rng(22)
    res, x = rs.standard_normal((6, D)), rs.standard_normal((6, D))
    np.testing.assert_allclose(O.boundary_subspace_fp64(x, res, Qr, R - np.eye(k)),
                               O.dense_boundary_fp64(x, res, T), atol=1e-12)
    # and the rotation is orthogonal with det 1 (a product of plane rotations)
    np.testing.assert_allclose(R.T @ R, np.eye(k), atol=1e-15)
    assert abs(np.linalg.det(R) - 1.0) < 1e-12


def test_subspace_plan_factors_round_once():
    # M = R_sub - I is formed exactly and rounded once to binary32; Q is
    # rounded to bfloat16. Hand-worked: 1 - 2^-24 (a float32) minus 1 is
    # -2^-24, exact; -(1 - 2^-24) minus 1 = -(2 - 2^-24) rounds to -2 in
    # binary32 (spacing 2^-22 below 2: 2^-24 away from -2, 3 2^-24 from the
    # next value); 0.75 off the diagonal stays 0.75.
    R = np.array([[1 - 2.0 ** -24, 0.75], [0.0, -(1 - 2.0 ** -24)]], np.float32)
    Q = np.array([[1.0 + 2.0 ** -8, 0.3], [2.0 ** -20, -0.5]], np.float32)
    Qq, M = O.subspace_plan_factors(Q, R)
    assert M.tolist() == [[-2.0 ** -24, 0.75], [0.0, -2.0]]
    assert Qq[0, 0] == 1.0          # 1 + 2^-8 is a bf16 tie: to even
    assert Qq[1, 1] == -0.5
    assert Qq[1, 0] == 2.0 ** -20


def test_subspace_reference_matches_factor_form_on_fixture():
    # With V = Qq M (no further rounding) the factor-form oracle gives the
    # same h as the subspace-form oracle (different summation order only).
    fx = W.workload_fixture("tiny")
    Qr, R = W.subspace_factors(fx.Q, fx.theta, fx.r)
    Qq, M = O.subspace_plan_factors(Qr.astype(np.float32), R.astype(np.float32))
    x, res = fx.x.float().numpy(), fx.residual.float().numpy()
    np.testing.assert_allclose(O.boundary_subspace_fp64(x, res, Qq, M),
                               O.boundary_fp64(x, res, Qq, Qq @ M), rtol=0, atol=1e-12)
