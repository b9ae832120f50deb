"""Host factor builders of the C library against the oracle (no GPU).

respin_factors_from_subspace: the zh §2.2 subspace form (Q, R_sub) turned
into the plan's row-form pair (U_r, V_r) = (Q, Q (R_sub - I)).
respin_factors_from_transition: the top-r SVD of Delta T = T - I (it §2C,
nl §2C, es §2B, fr §2C) by float64 subspace iteration in the library, checked
against the oracle's library SVD and the closed form of the synthetic T
(s_j = 2 |sin(theta_j / 2)|, each twice), with the gap refusal.
"""
import numpy as np
import pytest

import oracle as O
import rotation_post_quantization_b200 as rq
import workloads as W


def synthetic_T(D, k, nu, seed=0):
    Q = W.orthonormal_basis(D, k, seed)
    theta = W.plane_angles(k, nu)
    R_in, R_out = O.rotation_pair(Q, theta)
    return O.transition_matrix(R_in, R_out), theta


def test_subspace_form_matches_column_form():
    D, r = 256, 8
    Q = W.orthonormal_basis(D, r, 3)
    th = np.array([0.3, -0.2, 0.05, 0.7])
    R = np.zeros((r, r))
    for j, t in enumerate(th):
        c, s = np.cos(t), np.sin(t)
        R[2 * j:2 * j + 2, 2 * j:2 * j + 2] = [[c, -s], [s, c]]
    U, V = rq.respin_factors_from_subspace(Q.astype(np.float32), R.astype(np.float32))
    assert np.array_equal(U, Q.astype(np.float32))
    h = np.random.default_rng(1).standard_normal((5, D))
    got = h + (h @ U.astype(np.float64)) @ V.astype(np.float64).T
    Q32, R32 = Q.astype(np.float32).astype(np.float64), R.astype(np.float32).astype(np.float64)
    want = O.subspace_residual_rotation(h.T, Q32, R32).T
    assert np.max(np.abs(got - want)) <= 1e-6 * np.max(np.abs(want))


def test_transition_matches_library_svd_and_closed_form():
    D, k, r = 256, 16, 8
    T, theta = synthetic_T(D, k, 0.5)
    T32 = T.astype(np.float32)
    U, V, sig = rq.respin_factors_from_transition(T32, r)
    Uo, Vo, so = O.top_r_factors(T32.astype(np.float64), r)
    got = U.astype(np.float64) @ V.astype(np.float64).T
    want = Uo @ Vo.T
    assert np.max(np.abs(got - want)) <= 1e-5 * np.max(np.abs(want))
    assert np.max(np.abs(sig - so[:r + 1])) <= 1e-6
    closed = np.sort(np.repeat(2 * np.abs(np.sin(theta / 2)), 2))[::-1]
    assert np.max(np.abs(sig[:r + 1] - closed[:r + 1])) <= 1e-5
    # left factors orthonormal; V carries the singular values
    assert np.max(np.abs(U.T.astype(np.float64) @ U - np.eye(r))) <= 1e-5
    assert np.allclose(np.linalg.norm(V.astype(np.float64), axis=0), sig[:r], rtol=1e-5)


def test_transition_exact_rank_reproduces_delta_t():
    D, k = 128, 8
    T, _ = synthetic_T(D, k, 0.3, seed=2)
    T32 = T.astype(np.float32)
    U, V, sig = rq.respin_factors_from_transition(T32, k)
    dT = T32.astype(np.float64) - np.eye(D)
    err = np.linalg.norm(U.astype(np.float64) @ V.astype(np.float64).T - dT)
    assert err <= 1e-5 * np.linalg.norm(dT)
    assert sig[k] <= 1e-5 * sig[0]


def test_transition_refuses_a_split_pair():
    """Singular values come in equal pairs (one per rotation plane): a rank
    that splits a pair has no unique top-r subspace."""
    T, _ = synthetic_T(128, 8, 0.3, seed=2)
    with pytest.raises(rq.RespinError) as ei:
        rq.respin_factors_from_transition(T.astype(np.float32), 3)
    assert ei.value.status == rq.RESPIN_ERR_UNSUPPORTED
    assert "not unique" in ei.value.message


@pytest.mark.parametrize("r", [0, 128, 129])
def test_transition_bad_rank(r):
    T = np.eye(128, dtype=np.float32)
    with pytest.raises(rq.RespinError) as ei:
        rq.respin_factors_from_transition(T, r)
    assert ei.value.status == rq.RESPIN_ERR_INVALID_ARG


def test_transition_identity_has_no_gap():
    """T = I: Delta T = 0, nothing to truncate."""
    with pytest.raises(rq.RespinError) as ei:
        rq.respin_factors_from_transition(np.eye(64, dtype=np.float32), 4)
    assert ei.value.status == rq.RESPIN_ERR_UNSUPPORTED
    assert "not unique" in ei.value.message
