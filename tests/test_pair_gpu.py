"""GPU parity of the pair boundary kernel (plans made from the stored
subspace form, zh §2.2 steps 1-3: y = residual Q, z = y (R_sub - I)^T,
h' = residual + x + z Q^T, then per-token INT4 / INT3 quantization) against
the CPU oracle, element by element on seeded inputs."""
import numpy as np
import pytest
import torch

import oracle as O
import rotation_post_quantization_b200 as rq
import workloads as W
from parity_util import (check_bf16_output, check_codes_end_to_end, check_codes_on_own_h, check_corr,
                         check_h_f32, oracle_boundary_subspace, run_boundary_subspace,
                         subspace_corr_factors, subspace_of)

pytestmark = pytest.mark.gpu

# (name, D, N, r, k, nu, n_outlier, outlier_scale, dist)
CASES = [
    ("d4096_n1", 4096, 1, 32, 64, 0.1, 8, 50.0, "normal"),
    ("d4096_n7", 4096, 7, 32, 64, 0.1, 8, 50.0, "normal"),
    ("d4096_n33", 4096, 33, 32, 32, 0.05, 2, 20.0, "normal"),
    ("d4096_ragged", 4096, 301, 32, 64, 0.1, 8, 50.0, "normal"),
    ("d4096_nu1", 4096, 200, 32, 64, 1.0, 8, 50.0, "normal"),
    ("d4096_many_tiles", 4096, 2459, 32, 64, 0.1, 8, 50.0, "normal"),
    ("d4096_r16", 4096, 150, 16, 64, 0.1, 8, 50.0, "normal"),
    ("d2048_r32", 2048, 333, 32, 32, 0.5, 4, 20.0, "student_t3"),
    ("d2048_r8", 2048, 97, 8, 16, 1.0, 4, 20.0, "normal"),
    ("d4096_n4096", 4096, 4096, 32, 64, 0.1, 8, 50.0, "normal"),
    ("d4096_r24", 4096, 64, 24, 64, 0.3, 8, 50.0, "normal"),
]


def fixture(case):
    name, D, N, r, k, nu, no, os_, dist = case
    return W.boundary_fixture(D, N, r, k=k, nu=nu, n_outlier=no, outlier_scale=os_, dist=dist)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_pair_f32_debug_matches_fp64(case):
    fx = fixture(case)
    got = run_boundary_subspace(fx, f32=True)
    h64, hb, codes_ref, scale_ref = oracle_boundary_subspace(fx)
    check_h_f32(got["h"], h64)
    Uq, Vq = subspace_corr_factors(fx)
    check_corr(got["h"], fx.x.float().numpy().astype(np.float64),
               fx.residual.float().numpy().astype(np.float64), Uq, Vq)
    check_codes_on_own_h(O.bf16_bits(got["h"]), got["q"], got["scale"])
    check_codes_end_to_end(got["q"], codes_ref)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_pair_bf16_output(case):
    fx = fixture(case)
    got = run_boundary_subspace(fx, f32=False)
    h64, hb, codes_ref, scale_ref = oracle_boundary_subspace(fx)
    check_bf16_output(got["h"], h64)
    check_codes_on_own_h(got["h"], got["q"], got["scale"])
    check_codes_end_to_end(got["q"], codes_ref)


def test_pair_int3_codes():
    fx = fixture(CASES[3])
    got = run_boundary_subspace(fx, f32=False, qmax=3)
    h64, hb, codes_ref, _ = oracle_boundary_subspace(fx, qmax=3)
    check_bf16_output(got["h"], h64)
    check_codes_on_own_h(got["h"], got["q"], got["scale"], qmax=3)
    check_codes_end_to_end(got["q"], codes_ref)


def test_pair_no_residual_and_no_h_out():
    fx = fixture(CASES[3])
    got = run_boundary_subspace(fx, f32=False, residual=False)
    h64, _, codes_ref, scale_ref = oracle_boundary_subspace(fx, residual=False)
    check_bf16_output(got["h"], h64)
    assert np.array_equal(got["q"], O.pack_int4(codes_ref))
    got2 = run_boundary_subspace(fx, f32=False, h_out=False)
    _, hb, _, _ = oracle_boundary_subspace(fx)
    got3 = run_boundary_subspace(fx, f32=False)
    assert np.array_equal(got2["q"], got3["q"])
    assert np.array_equal(got2["scale"].view(np.uint32), got3["scale"].view(np.uint32))


def test_pair_exact_rank_equals_dense_T():
    # k = r: the stored form reproduces the dense transition up to the plan's
    # bfloat16 basis (per-token error far below the bf16 output rounding)
    fx = W.boundary_fixture(4096, 96, 32, k=32, nu=0.5, n_outlier=2, outlier_scale=20.0)
    got = run_boundary_subspace(fx, f32=True)
    R_in, R_out = O.rotation_pair(fx.Q, fx.theta)
    dense = O.dense_boundary_fp64(fx.x.float().numpy(), fx.residual.float().numpy(),
                                  O.transition_matrix(R_in, R_out))
    tok = np.linalg.norm(got["h"] - dense, axis=1) / np.linalg.norm(dense, axis=1)
    assert np.max(tok) < 2e-4, np.max(tok)


def test_pair_edge_tokens():
    # zero, constant, single-nonzero and tiny tokens through the pair kernel
    D, N = 4096, 24
    fx = W.boundary_fixture(D, N, 32, k=64, nu=0.1, n_outlier=8, outlier_scale=50.0)
    x = fx.x.clone()
    res = fx.residual.clone()
    x[0] = 0; res[0] = 0
    x[1] = 0.5; res[1] = 0
    x[2] = 0; res[2] = 0; x[2, 1234] = -3.0
    x[3] = 0; res[3] = 0; x[3, 7] = 1e-38
    fx.x, fx.residual = x, res
    got = run_boundary_subspace(fx, f32=False)
    h64, hb, codes_ref, scale_ref = oracle_boundary_subspace(fx)
    check_codes_on_own_h(got["h"], got["q"], got["scale"])
    assert got["scale"][0] == 0.0 and not got["q"][0].any()
    assert got["scale"][3] == 0.0
    assert np.array_equal(got["h"][:4], hb[:4])


def test_pair_full_size_llama2_7b():
    # the headline workload at its full size (D = 4096, 2048 tokens, r = 32),
    # every row against the oracle
    fx = W.workload_fixture("llama2_7b")
    got = run_boundary_subspace(fx, f32=False)
    h64, hb, codes_ref, scale_ref = oracle_boundary_subspace(fx)
    check_bf16_output(got["h"], h64)
    check_codes_on_own_h(got["h"], got["q"], got["scale"])
    check_codes_end_to_end(got["q"], codes_ref)
    got32 = run_boundary_subspace(fx, f32=True)
    check_h_f32(got32["h"], h64)
    Uq, Vq = subspace_corr_factors(fx)
    check_corr(got32["h"], fx.x.float().numpy().astype(np.float64),
               fx.residual.float().numpy().astype(np.float64), Uq, Vq)


def test_pair_unsupported_shapes():
    Q = np.zeros((1024, 8), np.float32)
    R = np.eye(8, dtype=np.float32)
    with pytest.raises(rq.RespinError) as ei:
        rq.SubspacePlan(1024, 8, Q, R)
    assert ei.value.status == rq.RESPIN_ERR_UNSUPPORTED
    with pytest.raises(rq.RespinError) as ei:
        rq.SubspacePlan(4096, 40, np.zeros((4096, 40), np.float32), np.eye(40, dtype=np.float32))
    assert ei.value.status == rq.RESPIN_ERR_UNSUPPORTED
