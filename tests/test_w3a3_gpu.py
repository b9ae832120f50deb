"""GPU parity of the W3A3 path (3-bit activation codes) against the oracle.

W3A3 is the second quantization setting the ReSpinQuant explainers report
beside W4A4 (zh §3-§4, it §3-§4, nl §3-§4, es §3-§4, fr §4); the pages give
no quantizer for either. Reading (same as the oracle's): the per-token
symmetric quantizer with bound 3 (inv = 3/amax, scale = amax/3, codes in
[-3, 3]) in the same nibble containers, so the integer GEMM is unchanged. Every boundary kernel family is
run with the RESPIN_ACT_INT3 plan flag; the codes feed the W4A4 GEMM with
3-bit weights.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rotation_post_quantization_b200 as rq
import workloads as W
from parity_util import (check_bf16_output, check_codes_end_to_end,
                         check_codes_on_own_h, check_corr, check_h_f32,
                         oracle_boundary, run_boundary)

pytestmark = pytest.mark.gpu

# (name, D, N, r, k, nu, n_outlier, outlier_scale, dist): one per kernel family
CASES = [
    ("tiny_rf1", 256, 64, 8, 8, 0.05, 2, 20.0, "normal"),                 # register-factor, 1 CTA
    ("decode_n8", 4096, 8, 32, 32, 0.05, 2, 20.0, "normal"),              # small call: 4-CTA cluster
    ("d8192_r32", 8192, 70, 32, 128, 0.1, 16, 100.0, "student_t3"),       # register-factor, 8 CTAs
    ("d4096_r64", 4096, 50, 64, 64, 0.1, 8, 50.0, "normal"),              # shared-memory factors
    ("d8192_r128", 8192, 24, 128, 128, 0.1, 16, 100.0, "student_t3"),     # V from L2
    ("rowtile_d4096_ragged", 4096, 1301, 32, 64, 0.1, 8, 50.0, "normal"),  # row tile
]


def fixture(case):
    name, D, N, r, k, nu, no, os_, dist = case
    return W.boundary_fixture(D, N, r, k=k, nu=nu, n_outlier=no,
                              outlier_scale=os_, dist=dist)


def check_int3_range(q_packed):
    c = O.unpack_int4(q_packed)
    assert c.min() >= -3 and c.max() <= 3
    return c


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_w3a3_boundary_bf16(case):
    fx = fixture(case)
    got = run_boundary(fx, f32=False, qmax=3)
    h64, hb, codes_ref, scale_ref = oracle_boundary(fx, qmax=3)
    check_bf16_output(got["h"], h64)
    check_codes_on_own_h(got["h"], got["q"], got["scale"], qmax=3)
    check_codes_end_to_end(got["q"], codes_ref)
    c = check_int3_range(got["q"])
    assert np.all(np.max(np.abs(c), axis=1) == 3)


@pytest.mark.parametrize("case", CASES[:3], ids=[c[0] for c in CASES[:3]])
def test_w3a3_boundary_f32_debug(case):
    fx = fixture(case)
    got = run_boundary(fx, f32=True, qmax=3)
    h64, hb, codes_ref, _ = oracle_boundary(fx, qmax=3)
    check_h_f32(got["h"], h64)
    Uq, Vq = O.plan_factors(fx.U.astype(np.float32), fx.V.astype(np.float32))
    check_corr(got["h"], fx.x.float().numpy().astype(np.float64),
               fx.residual.float().numpy().astype(np.float64), Uq, Vq)
    check_codes_on_own_h(O.bf16_bits(got["h"]), got["q"], got["scale"], qmax=3)
    check_codes_end_to_end(got["q"], codes_ref)


def test_w3a3_quant_only():
    """r = 0, no residual: 3-bit codes of x itself (row-wise kernel)."""
    fx = W.boundary_fixture(14336, 33, 0, k=2, nu=0.1, n_outlier=8, outlier_scale=50.0)
    got = run_boundary(fx, f32=False, residual=False, qmax=3)
    x = fx.x.float().numpy()
    codes, sc = O.quantize_int3_per_token(x)
    assert np.array_equal(got["scale"].view(np.uint32), sc.view(np.uint32))
    assert np.array_equal(got["q"], O.pack_int4(codes))
    assert np.array_equal(got["h"], O.bf16_bits(x))
    check_int3_range(got["q"])


def test_w3a3_boundary_then_gemm():
    """3-bit activation codes from the row-tile boundary (full 2048-token
    workload) times 3-bit weight codes: exact accumulators, bit-exact bf16."""
    fx = W.workload_fixture("llama2_7b")
    got = run_boundary(fx, f32=False, qmax=3)
    check_codes_on_own_h(got["h"], got["q"], got["scale"], qmax=3)
    N, K, O_ = fx.N, fx.D, 1040
    rs = np.random.default_rng(5)
    qw = O.pack_int4(rs.integers(-4, 4, (O_, K)).astype(np.int8))
    sw = W.weight_scales(O_, K, 5)
    d = "cuda"
    out = torch.empty(N, O_, dtype=torch.bfloat16, device=d)
    acc = torch.empty(N, O_, dtype=torch.int32, device=d)
    tq, tsa = torch.from_numpy(got["q"]).to(d), torch.from_numpy(got["scale"]).to(d)
    tqw, tsw = torch.from_numpy(qw).to(d), torch.from_numpy(sw).to(d)
    rq.w4a4_gemm(tq, tsa, tqw, tsw, out)
    rq.w4a4_gemm_i32(tq, tqw, acc)
    torch.cuda.synchronize()
    assert rq.respin_device_status() == 0
    ref = O.w4a4_acc_fp64(got["q"], qw)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref)
    want = O.w4a4_epilogue_bits(ref, got["scale"], sw)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)
