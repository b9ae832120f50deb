"""Plain, slow CPU oracle for the ReSpinQuant block-boundary path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import or call this module. The
CUDA library shares no code with it and never calls it.

Sources: the five gist.science explainer pages of "ReSpinQuant: Efficient
Layer-Wise LLM Quantization via Subspace Residual Rotation Approximation"
(arXiv 2604.11080), cited below by language and section (zh, it, nl, es, fr).

What the pages fix, and how this module follows it:

* Basis-transition matrix ``T = R_out^T R_in`` between the rotation of a
  block's output and of its input (zh §2.1; nl §2B; es §2B; fr §2B. The it
  page §2B prints ``R_out R_in^T``; the four-to-one majority is followed).
* ``T`` is close to ``I`` and ``Delta T = T - I`` is low rank; a top-r SVD of
  ``Delta T`` gives the subspace (it §2C; nl §2C; es §2B; fr §2C).
* The subspace residual rotation for a column vector: ``y = Q^T x``,
  ``M = R_sub - I_r``, ``x_out = x + Q (M y)`` (zh §2.2, steps 1-3). The fr
  page §2C writes ``z = R_sub y, x_out = x + Q z``, which adds ``Q Q^T x``
  twice if read literally; it is read as the zh form.
* Row convention (every kernel and every function here): a token is a row
  ``h``, the boundary is ``h' = residual P + x`` with ``P = T`` and the rank-r
  form ``h' = residual + (residual U_r) V_r^T + x``. Column form ``Tc`` and row
  form ``P`` are related by ``P = Tc^T``; for the subspace form this gives
  ``U_r = Q`` and ``V_r = Q M``.
* 4-bit activations (W4A4, zh §3-§4). The pages give no quantizer; the
  reading used: per-token symmetric, no clipping, ``inv = 7 / amax`` and
  ``q = clamp(rint(g * inv), -8, 7)`` (ties to even), ``scale = amax / 7``,
  all in IEEE binary32, on the bfloat16-rounded boundary output ``g``. Tokens
  with ``amax < 2^-125`` get scale 0 and all-zero codes (below that
  ``7 / amax`` would overflow binary32).
* 3-bit activations (W3A3, named beside W4A4 in zh §3-§4, it §3-§4,
  nl §3-§4, es §3-§4 and fr §4; no quantizer given either). Reading: the same
  per-token symmetric form with bound 3 instead of 7: ``inv = 3 / amax``,
  ``q = clamp(rint(g * inv), -4, 3)``, ``scale = amax / 3``; codes stay in
  4-bit containers (the pages give no 3-bit packing), so the integer GEMM is
  the same for both widths.
* Packing: element ``2j`` in the low nibble of byte ``j``, element ``2j+1`` in
  the high nibble, two's complement.
* W4A4 GEMM: ``acc[n, o] = sum_k a[n, k] w[o, k]`` exactly in integers, then
  ``out = bf16((float(acc) * sa[n]) * sw[o])`` in binary32, round to nearest
  even at every step.

Parity pins (tests/test_oracle_pins.py): Hadamard vs scipy; orthogonality of
``T`` and ``T = I`` for equal rotations; SVD factors vs the closed-form
fixture; rank-r = dense product for exact-rank ``T`` and for ``r = D``;
Eckart-Young bound; norm preservation; brute-force loops at tiny sizes;
bfloat16 rounding vs torch; quantizer invariants; integer GEMM vs a naive loop
and a selection-matrix special case; the pages' printed parameter counts.
Parity unpinned: nothing in this module; the pages' 32.3M-MAC overhead figure
is internally inconsistent and is not reproduced.
"""
from __future__ import annotations

import math

import numpy as np
import scipy.linalg

ZERO_TOKEN_AMAX = np.float32(2.0 ** -125)
BF16_MAX = (2.0 - 2.0 ** -7) * 2.0 ** 127


# --------------------------------------------------------------------------
# Rotations and the basis-transition matrix
# --------------------------------------------------------------------------

def hadamard(D: int) -> np.ndarray:
    """Normalised Sylvester Hadamard matrix H_D / sqrt(D), float64.

    The learned rotations start from a Hadamard matrix (zh §2.1; it §2C).
    """
    if D < 1 or D & (D - 1):
        raise ValueError("Sylvester construction needs D a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < D:
        H = np.block([[H, H], [H, -H]])
    return H / math.sqrt(D)


def skew_from_planes(Q: np.ndarray, theta: np.ndarray) -> np.ndarray:
    """Dense skew matrix A = sum_j theta_j (q_a q_b^T - q_b q_a^T).

    Plane j is spanned by columns (2j, 2j+1) of Q.
    """
    D = Q.shape[0]
    A = np.zeros((D, D))
    for j, t in enumerate(theta):
        qa = Q[:, 2 * j]
        qb = Q[:, 2 * j + 1]
        A += t * (np.outer(qa, qb) - np.outer(qb, qa))
    return A


def rotation_pair(Q: np.ndarray, theta: np.ndarray):
    """(R_in, R_out) = (H expm(A), H) for the synthetic boundary."""
    D = Q.shape[0]
    H = hadamard(D)
    return H @ scipy.linalg.expm(skew_from_planes(Q, theta)), H


def transition_matrix(R_in: np.ndarray, R_out: np.ndarray) -> np.ndarray:
    """T = R_out^T R_in (zh §2.1; nl §2B; es §2B; fr §2B)."""
    return R_out.T @ R_in


def top_r_factors(P: np.ndarray, r: int):
    """Rank-r factors of P - I from a library SVD (it §2C; fr §2C).

    With P - I = W diag(s) Z^T, returns U = W[:, :r] and V = Z[:, :r] s[:r],
    so that h (P - I)_r = (h U) V^T for a row vector h, plus all of s.
    """
    D = P.shape[0]
    W, s, Zt = np.linalg.svd(P - np.eye(D))
    return W[:, :r].copy(), (Zt[:r].T * s[:r]).copy(), s


def subspace_basis(P: np.ndarray, r: int):
    """(Q, M) of the subspace form: Q = top-r left singular vectors of P - I,
    M = Q^T (P - I) Q (the r x r transform inside the subspace, zh §2.2)."""
    D = P.shape[0]
    W, _, _ = np.linalg.svd(P - np.eye(D))
    Q = W[:, :r].copy()
    return Q, Q.T @ (P - np.eye(D)) @ Q


def subspace_residual_rotation(x_col: np.ndarray, Q: np.ndarray,
                               R_sub: np.ndarray) -> np.ndarray:
    """Column form of zh §2.2: y = Q^T x; M = R_sub - I_r; x + Q (M y).

    ``x_col`` is [D] or [D, n] (n column vectors).
    """
    r = Q.shape[1]
    y = Q.T @ x_col                      # step 1: projection
    M = R_sub - np.eye(r)                # step 2: transform inside the subspace
    return x_col + Q @ (M @ y)           # step 3: re-projection and residual


# --------------------------------------------------------------------------
# The boundary fix (row convention)
# --------------------------------------------------------------------------

def boundary_fp64(x: np.ndarray, residual: np.ndarray | None,
                  U: np.ndarray, V: np.ndarray) -> np.ndarray:
    """h' = residual + (residual U) V^T + x, float64 [N, D].

    ``residual`` None means zero. The rank-r fix is applied to the skip path
    before the addition of the block output (fr §2B; zh §2.2).
    """
    h = np.asarray(x, np.float64).copy()
    if residual is not None:
        res = np.asarray(residual, np.float64)
        h += res
        if U.shape[1]:
            h += (res @ np.asarray(U, np.float64)) @ np.asarray(V, np.float64).T
    return h


def boundary_subspace_fp64(x: np.ndarray, residual: np.ndarray | None,
                           Q: np.ndarray, M: np.ndarray) -> np.ndarray:
    """Row form of the zh §2.2 subspace residual rotation, float64 [N, D]:
    y = residual Q (step 1, projection), z = y M^T (step 2, M = R_sub - I
    inside the subspace), h' = residual + x + z Q^T (step 3, re-projection
    and residual). A row h maps as h^T does in the column form."""
    h = np.asarray(x, np.float64).copy()
    if residual is not None:
        res = np.asarray(residual, np.float64)
        h += res
        if Q.shape[1]:
            y = res @ np.asarray(Q, np.float64)          # step 1
            z = y @ np.asarray(M, np.float64).T          # step 2
            h += z @ np.asarray(Q, np.float64).T         # step 3
    return h


def dense_boundary_fp64(x: np.ndarray, residual: np.ndarray,
                        P: np.ndarray) -> np.ndarray:
    """h' = residual P + x with the dense D x D operator, float64."""
    return np.asarray(residual, np.float64) @ P + np.asarray(x, np.float64)


# --------------------------------------------------------------------------
# bfloat16
# --------------------------------------------------------------------------

def round_to_bf16(a) -> np.ndarray:
    """Nearest bfloat16 value (ties to even) of each float64/float32 entry,
    returned as float64. Overflow gives +-inf, NaN stays NaN."""
    a = np.asarray(a, np.float64)
    out = np.array(a, copy=True)
    fin = np.isfinite(a) & (a != 0.0)
    v = a[fin]
    _, e = np.frexp(v)                   # |v| in [2^(e-1), 2^e)
    # 8 significant bits for normals, fixed quantum 2^-133 below 2^-126
    q_exp = np.maximum(e, -125) - 8
    scaled = np.ldexp(v, -q_exp)         # exact: power-of-two scaling
    r = np.ldexp(np.rint(scaled), q_exp) # rint rounds half to even
    r = np.where(np.abs(r) > BF16_MAX, np.copysign(np.inf, r), r)
    out[fin] = r
    return out


def bf16_bits(a) -> np.ndarray:
    """uint16 bit patterns of round_to_bf16(a)."""
    v = round_to_bf16(a).astype(np.float32)   # exact: bf16 values are floats
    return (v.view(np.uint32) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits) -> np.ndarray:
    """float32 values of bfloat16 bit patterns (exact widening)."""
    b = np.asarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32)


# --------------------------------------------------------------------------
# Per-token symmetric INT4 / INT3 quantizer (binary32)
# --------------------------------------------------------------------------

def quantize_per_token(g, qmax: int) -> tuple[np.ndarray, np.ndarray]:
    """(codes int8 [N, D], scale float32 [N]) for float32 [N, D] input ``g``
    with ``qmax`` = 7 (INT4) or 3 (INT3).

    Every operation is one IEEE binary32 operation with round to nearest even:
    amax = max |g|; inv = qmax / amax; q = clamp(rint(g * inv), -qmax-1, qmax);
    scale = amax / qmax. A token with amax < 2^-125 gets scale 0 and zero
    codes.
    """
    if qmax not in (7, 3):
        raise ValueError("qmax must be 7 (INT4) or 3 (INT3)")
    g = np.asarray(g, np.float32)
    N, D = g.shape
    codes = np.zeros((N, D), np.int8)
    scale = np.zeros(N, np.float32)
    qm = np.float32(qmax)
    for n in range(N):
        amax = np.float32(np.max(np.abs(g[n]))) if D else np.float32(0)
        if not amax >= ZERO_TOKEN_AMAX:
            continue
        inv = np.float32(qm / amax)
        t = (g[n] * inv).astype(np.float32)
        q = np.rint(t)
        codes[n] = np.clip(q, -qmax - 1, qmax).astype(np.int8)
        scale[n] = np.float32(amax / qm)
    return codes, scale


def quantize_int4_per_token(g) -> tuple[np.ndarray, np.ndarray]:
    """W4A4 activations: quantize_per_token with bound 7."""
    return quantize_per_token(g, 7)


def quantize_int3_per_token(g) -> tuple[np.ndarray, np.ndarray]:
    """W3A3 activations: quantize_per_token with bound 3."""
    return quantize_per_token(g, 3)


def pack_int4(codes) -> np.ndarray:
    """uint8 [..., D/2]: element 2j -> low nibble of byte j, 2j+1 -> high."""
    c = np.asarray(codes)
    if c.shape[-1] % 2:
        raise ValueError("odd number of codes")
    n = (c.astype(np.int16) & 0xF).astype(np.uint8)
    return (n[..., 0::2] | (n[..., 1::2] << 4)).astype(np.uint8)


def unpack_int4(packed) -> np.ndarray:
    """int8 [..., 2 * bytes]: inverse of pack_int4 (two's complement nibbles)."""
    p = np.asarray(packed, np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), np.int8)
    lo = (p & 0xF).astype(np.int16)
    hi = (p >> 4).astype(np.int16)
    out[..., 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[..., 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out


# --------------------------------------------------------------------------
# W4A4 GEMM
# --------------------------------------------------------------------------

def w4a4_acc(q_act_packed, q_w_packed) -> np.ndarray:
    """Exact int64 acc[n, o] = sum_k a[n, k] w[o, k]."""
    a = unpack_int4(q_act_packed).astype(np.int64)
    w = unpack_int4(q_w_packed).astype(np.int64)
    return a @ w.T


def w4a4_acc_fp64(q_act_packed, q_w_packed) -> np.ndarray:
    """The same integer sums through a float64 matrix product (fast).

    Exact: every product is an integer of magnitude <= 64 and every partial
    sum has magnitude <= 64 K < 2^53, so no float64 rounding occurs in any
    summation order.
    """
    a = unpack_int4(q_act_packed).astype(np.float64)
    w = unpack_int4(q_w_packed).astype(np.float64)
    if 64 * a.shape[1] >= 2 ** 53:
        raise ValueError("K too large for an exact float64 product")
    return (a @ w.T).astype(np.int64)


def w4a4_epilogue_bits(acc, scale_act, scale_w) -> np.ndarray:
    """bf16 bits of (float(acc) * sa[n]) * sw[o], binary32 throughout."""
    acc = np.asarray(acc, np.int64)
    if acc.size and np.max(np.abs(acc)) >= 2 ** 24:
        raise ValueError("accumulator not exactly representable in binary32")
    f = acc.astype(np.float32)
    t = (f * np.asarray(scale_act, np.float32)[:, None]).astype(np.float32)
    t = (t * np.asarray(scale_w, np.float32)[None, :]).astype(np.float32)
    return bf16_bits(t)


def w4a4_dequant_fp64(acc, scale_act, scale_w) -> np.ndarray:
    """sa[n] sw[o] acc[n, o] in float64 (target of the relative-Frobenius check)."""
    return (np.asarray(acc, np.float64) * np.asarray(scale_act, np.float64)[:, None]
            * np.asarray(scale_w, np.float64)[None, :])


# --------------------------------------------------------------------------
# Composite reference for one boundary call
# --------------------------------------------------------------------------

def plan_factors(U, V):
    """The factors as the plan holds them: float32 input rounded to bfloat16,
    returned as float64 values."""
    return (round_to_bf16(np.asarray(U, np.float32)),
            round_to_bf16(np.asarray(V, np.float32)))


def boundary_reference(x, residual, U32, V32, qmax: int = 7):
    """Full reference for one boundary call with float32 host factors.

    Returns (h64, h_bf16_bits, codes, scale): h64 is the float64 fix with the
    plan's bfloat16 factors, h_bf16_bits its bfloat16 rounding, and the codes /
    scales come from the quantizer (bound qmax) applied to that bfloat16
    output.
    """
    Uq, Vq = plan_factors(U32, V32)
    h64 = boundary_fp64(x, residual, Uq, Vq)
    hb = bf16_bits(h64)
    codes, scale = quantize_per_token(bf16_bits_to_f32(hb), qmax)
    return h64, hb, codes, scale


def subspace_plan_factors(Q, R_sub):
    """The stored subspace form as the plan holds it: the float32 basis Q
    rounded to bfloat16, and M = R_sub - I from the float32 rotation, the
    difference taken exactly and rounded once to binary32; both returned as
    float64 values."""
    R = np.asarray(R_sub, np.float32).astype(np.float64)
    M = (R - np.eye(R.shape[0])).astype(np.float32).astype(np.float64)
    return round_to_bf16(np.asarray(Q, np.float32)), M


def boundary_reference_subspace(x, residual, Q32, R32, qmax: int = 7):
    """boundary_reference for a plan made from the stored subspace form
    (float32 Q [D, r] and R_sub [r, r], zh §2.2)."""
    Qq, M = subspace_plan_factors(Q32, R32)
    h64 = boundary_subspace_fp64(x, residual, Qq, M)
    hb = bf16_bits(h64)
    codes, scale = quantize_per_token(bf16_bits_to_f32(hb), qmax)
    return h64, hb, codes, scale


# --------------------------------------------------------------------------
# Offline weight preparation (zh §2.2 offline weight merging; fr §2A)
# --------------------------------------------------------------------------

def fuse_weight_fp64(W, R_in, R_out=None) -> np.ndarray:
    """W~ = R_out^T W R_in (or W R_in), float64: for y = W x with x~ = R_in^T x,
    W~ x~ = R_out^T y."""
    Wf = np.asarray(W, np.float64) @ np.asarray(R_in, np.float64)
    if R_out is not None:
        Wf = np.asarray(R_out, np.float64).T @ Wf
    return Wf


def quantize_weight_rows(W32, qmax: int = 7):
    """Per-output-channel symmetric codes of float32 W [O, K]: the activation
    quantizer applied to each row (binary32), packed two per byte."""
    codes, scale = quantize_per_token(np.asarray(W32, np.float32), qmax)
    return pack_int4(codes), scale


# --------------------------------------------------------------------------
# Counts the pages print (zh §4; nl §4; es §4; fr §4)
# --------------------------------------------------------------------------

def online_factor_params(layers: int, D: int, r: int,
                         boundaries_per_layer: int = 2) -> int:
    """Online parameters of the subspace form: one D x r basis per boundary."""
    return layers * boundaries_per_layer * D * r


def training_rotation_params(layers: int, D: int,
                             boundaries_per_layer: int = 2) -> int:
    """Learnable entries of one full D x D rotation per boundary."""
    return layers * boundaries_per_layer * D * D
