"""GPU parity of the fused boundary kernel against the CPU oracle.

The boundary is the rank-r residual-path basis fix of the ReSpinQuant
explainers (zh §2.2 steps 1-3; fr §2B-§2C) followed by per-token symmetric
INT4 quantization (zh §3-§4). Every case runs the C ABI on seeded inputs and
compares element by element with the oracle.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from parity_util import (check_bf16_output, check_codes_end_to_end,
                         check_codes_on_own_h, check_corr, check_h_f32,
                         oracle_boundary, run_boundary)

pytestmark = pytest.mark.gpu

# (name, D, N, r, k, nu, n_outlier, outlier_scale, dist)
CASES = [
    ("tiny", 256, 64, 8, 8, 0.05, 2, 20.0, "normal"),
    ("tiny_nu1", 256, 64, 8, 8, 1.0, 2, 20.0, "normal"),
    ("d4096_ragged", 4096, 200, 32, 64, 0.1, 8, 50.0, "normal"),
    ("d4096_nu1", 4096, 77, 32, 64, 1.0, 8, 50.0, "normal"),
    ("decode_n1", 4096, 1, 32, 32, 0.05, 2, 20.0, "normal"),
    ("decode_n8", 4096, 8, 32, 32, 0.05, 2, 20.0, "normal"),
    ("decode_n33", 4096, 33, 32, 32, 0.05, 2, 20.0, "normal"),
    ("d4096_r16", 4096, 50, 16, 64, 0.1, 8, 50.0, "normal"),
    ("d4096_r64", 4096, 50, 64, 64, 0.1, 8, 50.0, "normal"),
    ("d8192_r32", 8192, 70, 32, 128, 0.1, 16, 100.0, "student_t3"),
    ("d8192_r64", 8192, 40, 64, 128, 0.1, 16, 100.0, "student_t3"),
    ("d1024_r128", 1024, 40, 128, 128, 0.5, 4, 50.0, "normal"),
    ("d8192_r128", 8192, 24, 128, 128, 0.1, 16, 100.0, "student_t3"),
    # above the small-call threshold: row-tile kernel (16 whole tokens per CTA)
    ("rowtile_d4096_ragged", 4096, 1301, 32, 64, 0.1, 8, 50.0, "normal"),
    ("rowtile_d4096_nu1", 4096, 1296, 32, 64, 1.0, 8, 50.0, "normal"),
    ("rowtile_d2048_r16", 2048, 1290, 16, 32, 0.5, 4, 20.0, "student_t3"),
    # at least 256 tokens with padded rank 64 / 128: the tensor-core passes
    # (ragged token tiles, several K splits, one K split at D = 1024)
    ("tc_d8192_r64", 8192, 300, 64, 128, 0.1, 16, 100.0, "student_t3"),
    ("tc_d8192_r128", 8192, 333, 128, 128, 0.1, 16, 100.0, "student_t3"),
    ("tc_d4096_r48", 4096, 520, 48, 64, 0.1, 8, 50.0, "normal"),
    ("tc_d1024_r128", 1024, 700, 128, 128, 0.5, 4, 50.0, "normal"),
    # more token tiles (201) than SMs: the projection and re-projection grids
    # take more than one wave
    ("tc_d1024_r48_many_tiles", 1024, 25637, 48, 64, 0.1, 4, 50.0, "normal"),
    # rank 16 / 32 at D = 8192 (register-factor cluster plans) from 4096 tokens
    ("tc_d8192_r32", 8192, 4100, 32, 128, 0.1, 16, 100.0, "student_t3"),
    ("tc_d8192_r16", 8192, 4096, 16, 128, 0.1, 16, 100.0, "student_t3"),
]


def fixture(case):
    name, D, N, r, k, nu, no, os_, dist = case
    return W.boundary_fixture(D, N, r, k=k, nu=nu, n_outlier=no,
                              outlier_scale=os_, dist=dist)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_boundary_f32_debug_matches_fp64(case):
    fx = fixture(case)
    got = run_boundary(fx, f32=True)
    h64, hb, codes_ref, scale_ref = oracle_boundary(fx)
    check_h_f32(got["h"], h64)
    Uq, Vq = O.plan_factors(fx.U.astype(np.float32), fx.V.astype(np.float32))
    check_corr(got["h"], fx.x.float().numpy().astype(np.float64),
               fx.residual.float().numpy().astype(np.float64), Uq, Vq)
    check_codes_on_own_h(O.bf16_bits(got["h"]), got["q"], got["scale"])
    check_codes_end_to_end(got["q"], codes_ref)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_boundary_bf16_matches_oracle(case):
    fx = fixture(case)
    got = run_boundary(fx, f32=False)
    h64, hb, codes_ref, scale_ref = oracle_boundary(fx)
    check_bf16_output(got["h"], h64)
    check_codes_on_own_h(got["h"], got["q"], got["scale"])
    check_codes_end_to_end(got["q"], codes_ref)
    # every nonzero token uses the full code range
    c = O.unpack_int4(got["q"])
    assert c.min() >= -8 and c.max() <= 7
    assert np.all(np.max(np.abs(c), axis=1) == 7)


def test_boundary_full_size_llama2_7b():
    """Full 2048 x 4096, r = 32 workload, launch configuration of the bench."""
    fx = W.workload_fixture("llama2_7b")
    got = run_boundary(fx, f32=False)
    h64, hb, codes_ref, _ = oracle_boundary(fx)
    check_bf16_output(got["h"], h64)
    check_codes_on_own_h(got["h"], got["q"], got["scale"])
    check_codes_end_to_end(got["q"], codes_ref)


def test_boundary_full_size_llama2_70b_sampled():
    """8192 x 8192 (Student-t, 16 outlier channels x100), r = 32; the oracle
    checks a seeded sample of 256 rows."""
    w = W.WORKLOADS["llama2_70b"]
    fx = W.workload_fixture("llama2_70b")
    got = run_boundary(fx, f32=False)
    rows = np.sort(np.random.default_rng(0).choice(w.N, 256, replace=False))
    h64, hb, codes_ref, _ = oracle_boundary(fx, rows=rows)
    check_bf16_output(got["h"][rows], h64)
    check_codes_on_own_h(got["h"][rows], got["q"][rows], got["scale"][rows])
    check_codes_end_to_end(got["q"][rows], codes_ref)


@pytest.mark.parametrize("f32", [False, True])
def test_quant_only_no_residual(f32):
    """r = 0, residual NULL: plain per-token quantization of x (the input of
    the 14336 -> 4096 down projection)."""
    fx = W.boundary_fixture(14336, 20, 0, k=2, nu=0.1, n_outlier=8,
                            outlier_scale=50.0)
    got = run_boundary(fx, f32=f32, residual=False)
    x = fx.x.float().numpy()
    h = got["h"] if f32 else O.bf16_bits_to_f32(got["h"])
    assert np.array_equal(np.asarray(h, np.float32), x)
    codes, sc = O.quantize_int4_per_token(x)
    assert np.array_equal(got["q"], O.pack_int4(codes))
    assert np.array_equal(got["scale"], sc)


def test_r0_with_residual():
    fx = W.boundary_fixture(4096, 37, 0, k=2, nu=0.1, n_outlier=8,
                            outlier_scale=50.0)
    got = run_boundary(fx, f32=False)
    # in the kernel's precision: one binary32 addition, then bf16 rounding
    x = fx.x.float().numpy()
    res = fx.residual.float().numpy()
    hb = O.bf16_bits((res + x).astype(np.float32))
    assert np.array_equal(got["h"], hb)
    check_codes_on_own_h(got["h"], got["q"], got["scale"])


def test_residual_none_ignores_factors():
    fx = W.boundary_fixture(4096, 19, 32, k=64, nu=0.1, n_outlier=8,
                            outlier_scale=50.0)
    got = run_boundary(fx, f32=False, residual=False)
    assert np.array_equal(O.bf16_bits_to_f32(got["h"]), fx.x.float().numpy())


def test_h_out_null_still_quantizes():
    fx = W.boundary_fixture(4096, 45, 32, k=64, nu=0.1, n_outlier=8,
                            outlier_scale=50.0)
    ref = run_boundary(fx, f32=False)
    got = run_boundary(fx, f32=False, h_out=False)
    assert np.array_equal(ref["q"], got["q"])
    assert np.array_equal(ref["scale"], got["scale"])


def test_identity_transition_is_plain_sum():
    """T = I (global rotation, it §2B): zero factors give h' = residual + x."""
    fx = W.boundary_fixture(4096, 40, 32, k=64, nu=0.0, n_outlier=8,
                            outlier_scale=50.0)
    assert not np.any(fx.U @ fx.V.T)
    got = run_boundary(fx, f32=False)
    x = fx.x.float().numpy()
    res = fx.residual.float().numpy()
    assert np.array_equal(got["h"], O.bf16_bits((res + x).astype(np.float32)))


def test_edge_tokens():
    """All-zero token, constant token, single nonzero element."""
    D, N = 4096, 5
    fx = W.boundary_fixture(D, N, 32, k=64, nu=0.1, n_outlier=8,
                            outlier_scale=50.0)
    x = torch.zeros(N, D, dtype=torch.bfloat16)
    res = torch.zeros(N, D, dtype=torch.bfloat16)
    x[1] = 0.75
    x[2, 123] = -3.0
    x[3] = fx.x[3]
    res[3] = fx.residual[3]
    x[4, 7] = 1e-39       # tiny amax: treated as a zero token
    fx.x, fx.residual = x, res
    got = run_boundary(fx, f32=False)
    h64, hb, codes_ref, scale_ref = oracle_boundary(fx)
    check_bf16_output(got["h"], h64)
    check_codes_on_own_h(got["h"], got["q"], got["scale"])
    c = O.unpack_int4(got["q"])
    assert got["scale"][0] == 0 and not c[0].any()
    assert got["scale"][4] == 0 and not c[4].any()
    assert np.all(c[1] == 7)
    assert c[2, 123] == -7 and np.count_nonzero(c[2]) == 1


def test_transposed_convention_swaps_factors():
    """Column convention P = T^T is the same kernel with U and V swapped."""
    fx = W.boundary_fixture(1024, 30, 16, k=16, nu=0.5, n_outlier=2,
                            outlier_scale=20.0)
    fx2 = W.BoundaryFixture(fx.D, fx.N, fx.r, fx.Q, fx.theta, fx.V, fx.U,
                            fx.x, fx.residual)
    got = run_boundary(fx2, f32=True)
    R_in, R_out = O.rotation_pair(fx.Q, fx.theta)
    T = O.transition_matrix(R_in, R_out)
    dense_t = O.dense_boundary_fp64(fx.x.float().numpy(),
                                    fx.residual.float().numpy(), T.T)
    tok = (np.linalg.norm(got["h"] - dense_t, axis=1)
           / np.linalg.norm(dense_t, axis=1))
    assert np.max(tok) < 1e-4


def test_repeat_calls_deterministic():
    fx = W.boundary_fixture(4096, 100, 32, k=64, nu=0.1, n_outlier=8,
                            outlier_scale=50.0)
    a = run_boundary(fx, f32=False)
    b = run_boundary(fx, f32=False)
    for k in a:
        assert np.array_equal(a[k], b[k])


def test_rank_sweep_eckart_young_70b():
    """Config-5 rank sweep on 256 tokens (D = 8192, Student-t, 16 outlier
    channels x100, rank-128 Delta T): the fp32 h' of the rank-r fix against
    the dense h = residual T + x (exact rank-128 factors, float64). Per token
    the error stays within the Eckart-Young bound s_(r+1) |residual| plus the
    bf16 rounding of the plan's factors (at most 1 % of s_1 |residual|) and
    fp32 arithmetic, and its mean falls as r grows (it §2C, fr §2C: top-r
    SVD; s_j = 2 |sin(theta_j / 2)|, each twice)."""
    w = W.WORKLOADS["llama2_70b"]
    D, k, nu, n = w.D, w.k, w.nu, 256
    Q = W.orthonormal_basis(D, k, 0)
    th = W.plane_angles(k, nu)
    Uk, Vk = W.lowrank_factors(Q, th, k)
    sig = np.repeat(2 * np.abs(np.sin(th / 2)), 2)
    means = []
    for r in w.extra["ranks"]:
        fx = W.boundary_fixture(D, n, r, k=k, nu=nu, n_outlier=w.n_outlier,
                                outlier_scale=w.outlier_scale, dist=w.dist)
        got = run_boundary(fx, f32=True)
        x = fx.x.float().numpy().astype(np.float64)
        res = fx.residual.float().numpy().astype(np.float64)
        # the kernel's correction against its own (plan-rounded) rank-r factors
        check_corr(got["h"], x, res, *O.plan_factors(fx.U.astype(np.float32), fx.V.astype(np.float32)))
        hd = O.boundary_fp64(x, res, Uk, Vk)
        e = np.linalg.norm(got["h"].astype(np.float64) - hd, axis=1)
        rn = np.linalg.norm(res, axis=1)
        bound = (sig[r] if r < k else 0.0) * rn + 0.01 * sig[0] * rn + 1e-5 * np.linalg.norm(hd, axis=1)
        assert np.all(e <= bound), (r, float(np.max(e / bound)))
        means.append(float(np.mean(e / rn)))
    assert all(a > b for a, b in zip(means, means[1:])), means
