"""Offline weight preparation (host C ABI, no GPU): rotation fusion
W~ = R_out^T W R_in (zh §2.2 offline weight merging; fr §2A, W~ = W R) and
per-output-channel INT4 / INT3 weight codes, against the oracle and the
property that fixes the convention: W~ x~ = R_out^T W x with x~ = R_in^T x."""
import numpy as np
import pytest

import oracle as O
import rotation_post_quantization_b200 as rq


def orth(n, seed):
    q, r = np.linalg.qr(np.random.default_rng(seed).standard_normal((n, n)))
    return q * np.sign(np.diag(r))


@pytest.mark.parametrize("O_,K,with_out", [(40, 64, True), (33, 128, False), (256, 256, True)])
def test_fuse_weight_matches_oracle_and_rotates(O_, K, with_out):
    rs = np.random.default_rng(O_ + K)
    W = (rs.standard_normal((O_, K)) / np.sqrt(K)).astype(np.float32)
    Ri = orth(K, 1).astype(np.float32)
    Ro = orth(O_, 2).astype(np.float32) if with_out else None
    got = rq.respin_fuse_weight(W, Ri, Ro).astype(np.float64)
    ref = O.fuse_weight_fp64(W, Ri, Ro)
    # one float32 rounding of a float64 result (summation order may differ in
    # the last float64 bits)
    assert np.max(np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)) <= 2.0 ** -23
    # the defining property, in float64: W~ (R_in^T x) = R_out^T (W x), up to
    # the float32 rounding of the rotations (orthogonal to ~1e-7)
    x = rs.standard_normal((K, 5))
    lhs = ref @ (Ri.astype(np.float64).T @ x)
    rhs = W.astype(np.float64) @ x
    if with_out:
        rhs = Ro.astype(np.float64).T @ rhs
    np.testing.assert_allclose(lhs, rhs, atol=1e-5 * np.max(np.abs(rhs)))
    # the transposed input rotation is a different weight
    bad = W.astype(np.float64) @ Ri.astype(np.float64).T
    if with_out:
        bad = Ro.astype(np.float64).T @ bad
    assert not np.allclose(bad @ (Ri.astype(np.float64).T @ x), rhs, atol=1e-3)


def test_fuse_weight_identity_rotations():
    rs = np.random.default_rng(5)
    W = rs.standard_normal((24, 32)).astype(np.float32)
    got = rq.respin_fuse_weight(W, np.eye(32, dtype=np.float32), np.eye(24, dtype=np.float32))
    assert np.array_equal(got, W)


@pytest.mark.parametrize("qmax", [7, 3])
def test_quantize_weight_matches_oracle(qmax):
    rs = np.random.default_rng(qmax)
    W = (rs.standard_normal((37, 96)) * rs.uniform(0.01, 3, (37, 1))).astype(np.float32)
    W[3] = 0.0                         # an all-zero channel
    W[4, :] = 0.0
    W[4, 17] = -2.5                    # one nonzero entry
    q, sc = rq.respin_quantize_weight(W, qmax)
    qref, scref = O.quantize_weight_rows(W, qmax)
    assert np.array_equal(q, qref)
    assert np.array_equal(sc.view(np.uint32), scref.view(np.uint32))
    assert sc[3] == 0.0 and not q[3].any()
    c = O.unpack_int4(q)
    assert c.min() >= -qmax - 1 and c.max() <= qmax
    assert c[4, 17] == -qmax


def test_weight_tool_validation():
    fp = rq.ctypes.POINTER(rq.ctypes.c_float)
    buf = (rq.ctypes.c_float * 16)()
    p = rq.ctypes.cast(buf, fp)
    assert rq.lib.respin_fuse_weight(0, 4, p, p, None, p) == rq.RESPIN_ERR_INVALID_ARG
    assert rq.lib.respin_fuse_weight(2, 2, p, None, None, p) == rq.RESPIN_ERR_INVALID_ARG
    qb = (rq.ctypes.c_uint8 * 16)()
    assert rq.lib.respin_quantize_weight(2, 3, p, 7, qb, p) == rq.RESPIN_ERR_INVALID_ARG   # odd K
    assert rq.lib.respin_quantize_weight(2, 4, p, 5, qb, p) == rq.RESPIN_ERR_INVALID_ARG   # qmax
    assert rq.last_error()


def test_fuse_weight_permutation_permutes_columns():
    """A permutation as the input rotation only reorders W's columns."""
    rs = np.random.default_rng(9)
    W = rs.standard_normal((16, 64)).astype(np.float32)
    perm = rs.permutation(64)
    P = np.zeros((64, 64), np.float32)
    P[perm, np.arange(64)] = 1.0          # (W P)[:, j] = W[:, perm[j]]
    got = rq.respin_fuse_weight(W, P)
    assert np.array_equal(got, W[:, perm])


@pytest.mark.parametrize("qmax,bytes_", [(7, [0xC7, 0x02]), (3, [0xE3, 0x01])])
def test_quantize_weight_hand_worked_row(qmax, bytes_):
    """Row [2, -1, 0.5, 0]: inv = qmax/2; -1*inv = -qmax/2 is a tie that goes
    to the even integer (-4 for INT4, -2 for INT3); scale = 2/qmax."""
    W = np.array([[2.0, -1.0, 0.5, 0.0]], np.float32)
    q, sc = rq.respin_quantize_weight(W, qmax)
    assert list(q[0]) == bytes_
    assert sc[0] == np.float32(2.0) / np.float32(qmax)
    qo, so = O.quantize_weight_rows(W, qmax)
    assert list(qo[0]) == bytes_ and so[0] == sc[0]
