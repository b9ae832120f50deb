"""Shared helpers for the GPU parity tests: run the CUDA path through the C
ABI and compare it with the oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
import rotation_post_quantization_b200 as rq
import workloads as W

# Acceptance (tolerances written here, used by every boundary test):
H_REL_TOL = 2e-3        # fp32 h' vs fp64 oracle, relative (floor 1e-3 * token rms)
CORR_REL_TOL = 2e-3     # correction term vs oracle, relative to its token norm
CODE_MISMATCH_FRAC = 1e-4
BF16_REL_TOL = 2.0 ** -8  # bf16 output: one ulp relative (same floor)


def bf16_keys(bits: np.ndarray) -> np.ndarray:
    """Order-preserving integer keys of bf16 bit patterns (adjacent = +-1)."""
    b = bits.astype(np.int32)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def run_boundary(fx: W.BoundaryFixture, *, f32: bool, residual=True,
                 h_out=True, device="cuda", qmax=7):
    """Run respin_boundary_forward on the fixture (INT4 codes, or INT3 codes
    for qmax = 3); returns numpy results."""
    D, N, r = fx.D, fx.N, fx.r
    flags = (rq.RESPIN_H_FP32_DEBUG if f32 else 0) | (rq.RESPIN_ACT_INT3 if qmax == 3 else 0)
    U32 = fx.U.astype(np.float32) if r else None
    V32 = fx.V.astype(np.float32) if r else None
    plan = rq.Plan(D, r, U32, V32, flags)
    x = fx.x.to(device)
    res = fx.residual.to(device) if residual else None
    h = None
    if h_out:
        h = torch.empty(N, D, device=device,
                        dtype=torch.float32 if f32 else torch.bfloat16)
    q = torch.full((N, D // 2), 0xAB, device=device, dtype=torch.uint8)
    s = torch.full((N,), -1.0, device=device, dtype=torch.float32)
    rq.respin_boundary_forward(plan, x, res, h, q, s)
    torch.cuda.synchronize()
    assert rq.respin_device_status() == 0
    plan.destroy()
    out = dict(q=q.cpu().numpy(), scale=s.cpu().numpy())
    if h is not None:
        out["h"] = (h.cpu().numpy() if f32 else
                    h.view(torch.int16).cpu().numpy().view(np.uint16))
    return out


def oracle_boundary(fx: W.BoundaryFixture, rows=None, residual=True, qmax=7):
    """Oracle for the fixture (optionally a row subset)."""
    x = fx.x.float().numpy()
    res = fx.residual.float().numpy() if residual else None
    if rows is not None:
        x = x[rows]
        res = res[rows] if res is not None else None
    U32 = fx.U.astype(np.float32)
    V32 = fx.V.astype(np.float32)
    return O.boundary_reference(x, res, U32, V32, qmax)


def check_h_f32(h_gpu: np.ndarray, h64: np.ndarray) -> float:
    rms = np.sqrt(np.mean(h64 ** 2, axis=1, keepdims=True))
    den = np.maximum(np.maximum(np.abs(h64), 1e-3 * rms), 1e-300)
    rel = np.abs(h_gpu.astype(np.float64) - h64) / den
    worst = float(np.max(rel))
    assert worst <= H_REL_TOL, f"fp32 h' max relative error {worst}"
    return worst


def check_corr(h_gpu, x, res, Uq, Vq):
    corr_ref = (res @ Uq) @ Vq.T
    corr_gpu = h_gpu.astype(np.float64) - res - x
    nrm = np.linalg.norm(corr_ref, axis=1)
    err = np.linalg.norm(corr_gpu - corr_ref, axis=1)
    ok = nrm > 0
    worst = float(np.max(err[ok] / nrm[ok])) if ok.any() else 0.0
    assert worst <= CORR_REL_TOL, f"correction relative error {worst}"
    return worst


def check_bf16_output(h_bits: np.ndarray, h64: np.ndarray) -> float:
    """bf16 h' vs the fp64 oracle.

    Rounding the output to bf16 costs up to 2^-9 relative by itself, so the
    elementwise bound for the bf16 output is one bf16 ulp (2^-8) relative,
    with the same token-rms floor as the fp32 check (elements where
    residual + x + correction cancels carry fp32 absolute error that can span
    a few ulps of the tiny result). Away from cancellation (|h| >= 1e-2 of
    the token rms) the fp32 error is far below half an ulp, so there the
    output must be bf16(oracle) or an adjacent value.
    """
    g = O.bf16_bits_to_f32(h_bits).astype(np.float64)
    rms = np.sqrt(np.mean(h64 ** 2, axis=1, keepdims=True))
    den = np.maximum(np.maximum(np.abs(h64), 1e-3 * rms), 1e-300)
    rel = np.abs(g - h64) / den
    worst = float(np.max(rel))
    assert worst <= BF16_REL_TOL, f"bf16 h' max relative error {worst}"
    d = np.abs(bf16_keys(h_bits) - bf16_keys(O.bf16_bits(h64)))
    away = np.abs(h64) >= 1e-2 * rms
    assert int(np.max(d[away], initial=0)) <= 1, \
        "bf16 h' more than one ulp from the oracle away from cancellation"
    return worst


def check_codes_on_own_h(h_bits, q_packed, scale, qmax=7):
    """Codes and scales bit-exact vs the oracle quantizer on the GPU's h'."""
    codes, sc = O.quantize_per_token(O.bf16_bits_to_f32(h_bits), qmax)
    assert np.array_equal(scale.view(np.uint32), sc.view(np.uint32)), \
        "scales differ"
    assert np.array_equal(q_packed, O.pack_int4(codes)), "codes differ"


def check_codes_end_to_end(q_packed, codes_ref):
    c = O.unpack_int4(q_packed).astype(np.int16)
    d = np.abs(c - codes_ref.astype(np.int16))
    assert int(d.max()) <= 1, "a code differs by more than 1"
    frac = float(np.mean(d != 0))
    assert frac <= CODE_MISMATCH_FRAC, f"code mismatch fraction {frac}"
    return frac


def subspace_of(fx: W.BoundaryFixture):
    """float32 (Q, R_sub) of the fixture's stored subspace form."""
    Qr, R = W.subspace_factors(fx.Q, fx.theta, fx.r)
    return Qr.astype(np.float32), R.astype(np.float32)


def run_boundary_subspace(fx: W.BoundaryFixture, *, f32: bool, residual=True,
                          h_out=True, device="cuda", qmax=7):
    """respin_boundary_forward with a plan made by respin_plan_create_subspace
    from the fixture's (Q, R_sub); returns numpy results."""
    D, N, r = fx.D, fx.N, fx.r
    flags = (rq.RESPIN_H_FP32_DEBUG if f32 else 0) | (rq.RESPIN_ACT_INT3 if qmax == 3 else 0)
    Q32, R32 = subspace_of(fx)
    plan = rq.SubspacePlan(D, r, Q32, R32, flags)
    x = fx.x.to(device)
    res = fx.residual.to(device) if residual else None
    h = None
    if h_out:
        h = torch.empty(N, D, device=device, dtype=torch.float32 if f32 else torch.bfloat16)
    q = torch.full((N, D // 2), 0xAB, device=device, dtype=torch.uint8)
    s = torch.full((N,), -1.0, device=device, dtype=torch.float32)
    rq.respin_boundary_forward(plan, x, res, h, q, s)
    torch.cuda.synchronize()
    assert rq.respin_device_status() == 0
    plan.destroy()
    out = dict(q=q.cpu().numpy(), scale=s.cpu().numpy())
    if h is not None:
        out["h"] = (h.cpu().numpy() if f32 else
                    h.view(torch.int16).cpu().numpy().view(np.uint16))
    return out


def oracle_boundary_subspace(fx: W.BoundaryFixture, rows=None, residual=True, qmax=7):
    """Oracle for a subspace plan of the fixture (optionally a row subset)."""
    x = fx.x.float().numpy()
    res = fx.residual.float().numpy() if residual else None
    if rows is not None:
        x = x[rows]
        res = res[rows] if res is not None else None
    Q32, R32 = subspace_of(fx)
    return O.boundary_reference_subspace(x, res, Q32, R32, qmax)


def subspace_corr_factors(fx: W.BoundaryFixture):
    """(U, V) with (res U) V^T equal to the subspace plan's correction term
    (U = bf16(Q), V = bf16(Q) M, float64)."""
    Q32, R32 = subspace_of(fx)
    Qq, M = O.subspace_plan_factors(Q32, R32)
    return Qq, Qq @ M
