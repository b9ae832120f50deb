"""Seeded synthetic inputs for the ReSpinQuant block-boundary path.

This module is shared by the tests, the benchmark and the CPU oracle's checks.
It draws random numbers and builds fixtures; it holds none of the boundary,
quantizer or GEMM arithmetic (those live, independently, in the CUDA library
and in the oracle).

Workload recipe (all draws seeded; ``seed`` 0 everywhere, distinct tensor ids):

* Activations ``x`` and ``residual``: i.i.d. N(0, 1) (or Student-t with 3
  degrees of freedom for the 70B-shaped workload), with a seeded set of outlier
  channels, shared by both tensors, multiplied by a fixed factor. The values are
  drawn in float64 and converted to bfloat16 by torch (round to nearest even).
* Basis change between two blocks: the pages say the learned rotations start from
  a Hadamard matrix and stay close to it, so that ``T = R_out^T R_in`` is close
  to the identity and ``T - I`` is low rank (ReSpinQuant explainers, zh page
  §2.1 and nl page §2C). The fixture takes ``R_out = H`` and
  ``R_in = H expm(A)`` with ``A`` a random skew matrix of rank ``k``:
  ``A = sum_j theta_j (q_a q_b^T - q_b q_a^T)`` over ``k/2`` planes spanned by
  a seeded orthonormal basis, so ``T = expm(A)``. The plane angles follow a
  1/j spectrum scaled so that the Frobenius norm of ``A`` equals ``nu``.
* Rank-r factors: ``expm(A)`` rotates plane j by ``theta_j`` and leaves the rest
  alone, so ``T - I`` restricted to plane j is the 2x2 block
  ``B_j = [[cos-1, sin], [-sin, cos-1]]`` whose two singular values are both
  ``2 |sin(theta_j / 2)|``. Because the angles decrease with j, the top-r
  singular subspace of ``T - I`` is the first ``r/2`` planes, and in the row
  convention ``h (T - I)_r = (h U_r) V_r^T`` with ``U_r = [q_a q_b ...]`` and
  ``V_r = U_r blockdiag(B_j)^T``. This is the closed form of the offline SVD
  step (zh page §2.2, nl page §2C); the oracle checks it against a library SVD
  of its own dense ``T``.
* INT4 weights: uniformly random bytes, i.e. two uniformly random two's
  complement nibbles in [-8, 7] per byte; per-output-channel fp32 scales
  ``U(0.5, 1.5) / (4.61 sqrt(K))``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

# Tensor ids keep every draw independent for a given seed.
TID_X = 1
TID_RESIDUAL = 2
TID_BASIS = 3
TID_OUTLIERS = 4
TID_WEIGHTS = 5
TID_WSCALE = 6
TID_ACODES = 7
TID_ASCALE = 8


@dataclass(frozen=True)
class Workload:
    """One synthetic workload shaped like the pages' models."""
    name: str
    D: int
    N: int
    r: int
    k: int
    nu: float
    n_outlier: int
    outlier_scale: float
    dist: str = "normal"          # "normal" or "student_t3"
    O: int | None = None          # GEMM output channels (None: no GEMM)
    extra: dict = field(default_factory=dict)


# The five workloads; names say what they are shaped like.
WORKLOADS = {
    "tiny": Workload("tiny", D=256, N=64, r=8, k=8, nu=0.05, n_outlier=2,
                     outlier_scale=20.0),
    "llama2_7b": Workload("llama2_7b", D=4096, N=2048, r=32, k=64, nu=0.1,
                          n_outlier=8, outlier_scale=50.0, O=11008),
    "decode": Workload("decode", D=4096, N=256, r=32, k=32, nu=0.05,
                       n_outlier=2, outlier_scale=20.0, O=4096,
                       extra={"Ns": (1, 8, 32, 64, 256)}),
    "llama3_8b_stack": Workload("llama3_8b_stack", D=4096, N=4096, r=32, k=64,
                                nu=0.1, n_outlier=8, outlier_scale=50.0,
                                O=14336, extra={"layers": 32, "mlp": 14336}),
    "llama2_70b": Workload("llama2_70b", D=8192, N=8192, r=32, k=128, nu=0.1,
                           n_outlier=16, outlier_scale=100.0,
                           dist="student_t3", O=28672,
                           extra={"ranks": (16, 32, 64, 128)}),
}


def rng(seed: int, tensor_id: int) -> np.random.Generator:
    """Independent deterministic stream for (seed, tensor id)."""
    return np.random.default_rng([int(seed), int(tensor_id)])


def outlier_channels(D: int, n: int, seed: int = 0) -> np.ndarray:
    """Seeded outlier channel indices, drawn without replacement."""
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    return np.sort(rng(seed, TID_OUTLIERS).choice(D, size=n, replace=False))


def activations_f64(N: int, D: int, *, n_outlier: int, outlier_scale: float,
                    dist: str = "normal", seed: int = 0, tensor_id: int = TID_X,
                    row0: int = 0) -> np.ndarray:
    """float64 [N, D] activations; rows ``row0 .. row0+N-1`` of the stream.

    Each row is drawn from its own sub-stream, so any row range of a large
    workload can be regenerated without drawing the rows before it.
    """
    out = np.empty((N, D), dtype=np.float64)
    idx = outlier_channels(D, n_outlier, seed)
    for i in range(N):
        g = np.random.default_rng([int(seed), int(tensor_id), int(row0 + i)])
        if dist == "normal":
            v = g.standard_normal(D)
        elif dist == "student_t3":
            z = g.standard_normal(D)
            w = g.standard_normal((3, D))
            v = z / np.sqrt((w * w).sum(axis=0) / 3.0)
            # outlier channels are N(0,1) times the factor
            v[idx] = z[idx]
        else:
            raise ValueError(dist)
        v[idx] *= outlier_scale
        out[i] = v
    return out


def activations_bf16(N: int, D: int, **kw) -> torch.Tensor:
    """bfloat16 [N, D] CPU tensor: float64 draw -> float32 -> bfloat16 (RNE)."""
    a = activations_f64(N, D, **kw)
    return torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)


def activations_bf16_fast(N: int, D: int, *, n_outlier: int,
                          outlier_scale: float, dist: str = "normal",
                          seed: int = 0, tensor_id: int = TID_X,
                          device: str = "cpu") -> torch.Tensor:
    """Large-size variant for the benchmark: one torch generator per tensor.

    Same distribution as :func:`activations_bf16`, different stream; used where
    only the statistics of the inputs matter (timing), never for stored values.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1000003 + int(tensor_id))
    if dist == "normal":
        v = torch.randn(N, D, generator=g, dtype=torch.float32)
    else:
        z = torch.randn(N, D, generator=g, dtype=torch.float32)
        w = torch.randn(3, N, D, generator=g, dtype=torch.float32)
        v = z / torch.sqrt((w * w).sum(0) / 3.0)
    idx = torch.from_numpy(outlier_channels(D, n_outlier, seed))
    if len(idx):
        v[:, idx] *= outlier_scale
    return v.to(torch.bfloat16).to(device)


def orthonormal_basis(D: int, k: int, seed: int = 0,
                      tensor_id: int = TID_BASIS) -> np.ndarray:
    """Seeded float64 [D, k] matrix with orthonormal columns (QR, sign-fixed)."""
    g = rng(seed, tensor_id)
    a = g.standard_normal((D, k))
    q, rr = np.linalg.qr(a)
    s = np.sign(np.diag(rr))
    s[s == 0] = 1.0
    return q * s


def plane_angles(k: int, nu: float) -> np.ndarray:
    """Angles theta_j = nu (1/j) / sqrt(2 sum_{i<=k/2} 1/i^2), j = 1..k/2.

    With this scaling the skew generator sum_j theta_j (q_a q_b^T - q_b q_a^T)
    has Frobenius norm nu. Angles are distinct and decreasing.
    """
    if k % 2:
        raise ValueError("k must be even (planes come in pairs of columns)")
    m = k // 2
    j = np.arange(1, m + 1, dtype=np.float64)
    return nu * (1.0 / j) / math.sqrt(2.0 * float(np.sum(1.0 / j ** 2)))


def lowrank_factors(Q: np.ndarray, theta: np.ndarray, r: int):
    """Closed-form rank-r factors (U_r, V_r), float64 [D, r] each.

    Plane j uses columns (2j, 2j+1) of Q; its 2x2 block is
    B_j = [[cos t - 1, sin t], [-sin t, cos t - 1]]. The first r/2 planes are
    kept (largest angles = largest singular values); requires r even and
    r/2 <= number of planes.
    """
    if r % 2:
        raise ValueError("r must be even so that no rotation plane is split")
    m = r // 2
    if m > len(theta):
        raise ValueError("r larger than the rank of T - I")
    D = Q.shape[0]
    U = np.ascontiguousarray(Q[:, :r])
    V = np.zeros((D, r), dtype=np.float64)
    for j in range(m):
        c, s = math.cos(theta[j]), math.sin(theta[j])
        B = np.array([[c - 1.0, s], [-s, c - 1.0]])
        V[:, 2 * j:2 * j + 2] = U[:, 2 * j:2 * j + 2] @ B.T
    return U, V


def subspace_factors(Q: np.ndarray, theta: np.ndarray, r: int):
    """The stored subspace form (basis, rotation) of the same rank-r fix,
    float64: ``Q_r`` = the first r columns of the plane basis and ``R_sub`` =
    blockdiag of the 2x2 plane rotations [[cos t, -sin t], [sin t, cos t]],
    so that ``R_sub - I`` = blockdiag(B_j)^T and ``Q_r (R_sub - I)`` equals
    the ``V_r`` of :func:`lowrank_factors` (zh page §2.2 stores one D x r
    basis and one r x r rotation per boundary)."""
    if r % 2:
        raise ValueError("r must be even so that no rotation plane is split")
    m = r // 2
    if m > len(theta):
        raise ValueError("r larger than the rank of T - I")
    R = np.eye(r)
    for j in range(m):
        c, s = math.cos(theta[j]), math.sin(theta[j])
        R[2 * j:2 * j + 2, 2 * j:2 * j + 2] = [[c, -s], [s, c]]
    return np.ascontiguousarray(Q[:, :r]), R


@dataclass
class BoundaryFixture:
    """Everything one boundary call needs, on the CPU."""
    D: int
    N: int
    r: int
    Q: np.ndarray          # float64 [D, k] plane basis
    theta: np.ndarray      # float64 [k/2]
    U: np.ndarray          # float64 [D, r]
    V: np.ndarray          # float64 [D, r]
    x: torch.Tensor        # bf16 [N, D]
    residual: torch.Tensor # bf16 [N, D]


def boundary_fixture(D: int, N: int, r: int, *, k: int, nu: float,
                     n_outlier: int, outlier_scale: float,
                     dist: str = "normal", seed: int = 0,
                     basis_id: int = TID_BASIS) -> BoundaryFixture:
    """Fixture for one block boundary (rank-r factors plus activations)."""
    Q = orthonormal_basis(D, k, seed, basis_id)
    theta = plane_angles(k, nu)
    U, V = lowrank_factors(Q, theta, r) if r > 0 else (
        np.zeros((D, 0)), np.zeros((D, 0)))
    kw = dict(n_outlier=n_outlier, outlier_scale=outlier_scale, dist=dist,
              seed=seed)
    x = activations_bf16(N, D, tensor_id=TID_X, **kw)
    res = activations_bf16(N, D, tensor_id=TID_RESIDUAL, **kw)
    return BoundaryFixture(D, N, r, Q, theta, U, V, x, res)


def workload_fixture(name: str, *, N: int | None = None, r: int | None = None,
                     nu: float | None = None, seed: int = 0) -> BoundaryFixture:
    """Boundary fixture of a named workload, optionally resized."""
    w = WORKLOADS[name]
    return boundary_fixture(w.D, w.N if N is None else N,
                            w.r if r is None else r, k=w.k,
                            nu=w.nu if nu is None else nu,
                            n_outlier=w.n_outlier,
                            outlier_scale=w.outlier_scale, dist=w.dist,
                            seed=seed)


def int4_packed_random(rows: int, K: int, seed: int = 0,
                       tensor_id: int = TID_WEIGHTS) -> np.ndarray:
    """uint8 [rows, K/2]: uniformly random bytes = two random int4 nibbles each."""
    if K % 2:
        raise ValueError("K must be even")
    return rng(seed, tensor_id).integers(0, 256, size=(rows, K // 2),
                                         dtype=np.uint8)


def int3_packed_random(rows: int, K: int, seed: int = 0,
                       tensor_id: int = TID_WEIGHTS) -> np.ndarray:
    """uint8 [rows, K/2]: two uniformly random 3-bit codes (-4..3) per byte,
    each in a two's-complement nibble (low nibble first)."""
    b = int4_packed_random(rows, K, seed, tensor_id)
    lo, hi = b & 7, (b >> 4) & 7
    # 3-bit two's complement -> 4-bit: copy bit 2 into bit 3
    lo = lo | ((lo & 4) << 1)
    hi = hi | ((hi & 4) << 1)
    return (lo | (hi << 4)).astype(np.uint8)


def weight_scales(O: int, K: int, seed: int = 0) -> np.ndarray:
    """float32 [O] per-output-channel scales U(0.5, 1.5) / (4.61 sqrt(K))."""
    u = rng(seed, TID_WSCALE).uniform(0.5, 1.5, size=O)
    return (u / (4.61 * math.sqrt(K))).astype(np.float32)


def activation_scales(N: int, seed: int = 0) -> np.ndarray:
    """float32 [N] positive per-token scales for GEMM-only cases."""
    return rng(seed, TID_ASCALE).uniform(0.5, 8.0, size=N).astype(np.float32)
