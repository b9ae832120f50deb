"""GPU parity of the W4A4 GEMM kernels (skinny kernel for N <= 128 tokens,
tensor-memory kernel above) against the exact-integer oracle.

W4A4 linear (ReSpinQuant explainers zh §3-§4, fr §4): int32 accumulators
must be bit-exact; the bf16 output of the binary32 scale epilogue must be
bit-exact given the same codes and scales, and within 1e-2 relative Frobenius
of the float64 dequantized product.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rotation_post_quantization_b200 as rq
import workloads as W

pytestmark = pytest.mark.gpu


def make(N, K, O_, seed=0):
    qa = W.int4_packed_random(N, K, seed, W.TID_ACODES)
    qw = W.int4_packed_random(O_, K, seed, W.TID_WEIGHTS)
    sa = W.activation_scales(N, seed)
    sw = W.weight_scales(O_, K, seed)
    return qa, qw, sa, sw


def run(qa, qw, sa, sw):
    d = "cuda"
    tqa, tqw = torch.from_numpy(qa).to(d), torch.from_numpy(qw).to(d)
    tsa, tsw = torch.from_numpy(sa).to(d), torch.from_numpy(sw).to(d)
    N, O_ = qa.shape[0], qw.shape[0]
    acc = torch.full((N, O_), 0x7eadbeef, dtype=torch.int32, device=d)
    out = torch.full((N, O_), 7.0, dtype=torch.bfloat16, device=d)
    rq.w4a4_gemm_i32(tqa, tqw, acc)
    rq.w4a4_gemm(tqa, tsa, tqw, tsw, out)
    torch.cuda.synchronize()
    assert rq.respin_device_status() == 0
    return (acc.cpu().numpy(),
            out.view(torch.int16).cpu().numpy().view(np.uint16))


def check(qa, qw, sa, sw, acc, outb, rows=None):
    if rows is not None:
        qa, sa, acc, outb = qa[rows], sa[rows], acc[rows], outb[rows]
    ref = O.w4a4_acc_fp64(qa, qw)
    assert np.array_equal(acc.astype(np.int64), ref), "int32 accumulators differ"
    want = O.w4a4_epilogue_bits(ref, sa, sw)
    assert np.array_equal(outb, want), "bf16 outputs differ"
    deq = O.w4a4_dequant_fp64(ref, sa, sw)
    got = O.bf16_bits_to_f32(outb).astype(np.float64)
    assert np.linalg.norm(got - deq) / np.linalg.norm(deq) <= 1e-2


@pytest.mark.parametrize("N,K,O_", [
    # tensor-memory kernel (more than 128 tokens; CTA pairs of 256 rows)
    (129, 128, 16),        # smallest K and O
    (133, 256, 48),        # ragged everything
    (256, 512, 256),       # exactly one pair tile
    (200, 1024, 272),      # ragged M and N tiles, several K blocks
    (300, 4096, 512),
    (129, 1024, 4096),     # one row past a single-CTA tile
    (200, 4096, 4112),     # last tile 16 channels wide, ragged rows
    (256, 2048, 272),      # exactly one pair tile of rows, ragged channels
    (300, 8192, 1040),     # 64 K blocks, two row tiles
])
def test_gemm_small(N, K, O_):
    qa, qw, sa, sw = make(N, K, O_)
    acc, outb = run(qa, qw, sa, sw)
    check(qa, qw, sa, sw, acc, outb)


@pytest.mark.parametrize("N,K,O_", [
    # skinny kernel (N <= 128): token tiles of 8 / 16 / 32 / 2 x 32 / 4 x 32
    (1, 128, 16),          # one chunk: 7 of 8 warps hold no K
    (7, 256, 32),
    (9, 1152, 48),         # 9 chunks over 8 warps
    (16, 4096, 11008),
    (17, 4096, 4096),
    (31, 14336, 4096),     # 112 chunks: 14 per warp, ragged last group
    (33, 2048, 16),
    (63, 4096, 272),
    (64, 14336, 4096),     # down-projection K (stack workload)
    (65, 8192, 1040),
    (100, 1024, 4096),
    (128, 2048, 272),
])
def test_gemm_skinny(N, K, O_):
    qa, qw, sa, sw = make(N, K, O_, seed=3)
    acc, outb = run(qa, qw, sa, sw)
    check(qa, qw, sa, sw, acc, outb)


def test_gemm_skinny_extremes_exact():
    """Skinny kernel at the largest K: all codes -8 gives acc = 64 K = 2^22
    (the MMA sums 2^30 before the shift back)."""
    N, K, O_ = 9, 65536, 16
    qa = np.full((N, K // 2), 0x88, np.uint8)
    qw = np.full((O_, K // 2), 0x88, np.uint8)
    acc, _ = run(qa, qw, np.ones(N, np.float32), np.ones(O_, np.float32))
    assert np.all(acc == 64 * K)
    qw2 = np.full((O_, K // 2), 0x77, np.uint8)
    acc2, _ = run(qa, qw2, np.ones(N, np.float32), np.ones(O_, np.float32))
    assert np.all(acc2 == -56 * K)


@pytest.mark.parametrize("N", [1, 8, 32, 64, 256])
def test_gemm_decode_4096(N):
    qa, qw, sa, sw = make(N, 4096, 4096, seed=1)
    acc, outb = run(qa, qw, sa, sw)
    check(qa, qw, sa, sw, acc, outb)


def test_gemm_full_size_llama2_7b():
    """2048 x 4096 -> 11008 (bench launch configuration; several tiles per
    persistent CTA), every output checked, twice in a row."""
    qa, qw, sa, sw = make(2048, 4096, 11008)
    for _ in range(2):
        acc, outb = run(qa, qw, sa, sw)
        check(qa, qw, sa, sw, acc, outb)


def test_gemm_full_size_llama3_8b_down_sampled():
    """4096 x 14336 -> 4096 (down projection of the stack workload), 128 rows."""
    qa, qw, sa, sw = make(4096, 14336, 4096, seed=2)
    acc, outb = run(qa, qw, sa, sw)
    rows = np.sort(np.random.default_rng(4).choice(4096, 128, replace=False))
    check(qa, qw, sa, sw, acc, outb, rows)


def test_gemm_extremes_exact():
    """All codes -8 (largest magnitude): acc = 64 K exactly (tensor-memory
    kernel)."""
    N, K, O_ = 130, 14336, 32
    qa = np.full((N, K // 2), 0x88, np.uint8)
    qw = np.full((O_, K // 2), 0x88, np.uint8)
    sa = np.ones(N, np.float32)
    sw = np.ones(O_, np.float32)
    acc, _ = run(qa, qw, sa, sw)
    assert np.all(acc == 64 * K)
    qw2 = np.full((O_, K // 2), 0x77, np.uint8)   # +7 * -8
    acc2, _ = run(qa, qw2, sa, sw)
    assert np.all(acc2 == -56 * K)


@pytest.mark.parametrize("N", [20, 70])
def test_gemm_selection_matrix(N):
    """One +1 per weight row: the GEMM gathers activation codes (skinny and
    tensor-memory kernels)."""
    K, O_ = 512, 64
    rs = np.random.default_rng(9)
    qa = W.int4_packed_random(N, K, 4, W.TID_ACODES)
    sel = rs.integers(0, K, O_)
    cw = np.zeros((O_, K), np.int8)
    cw[np.arange(O_), sel] = 1
    qw = O.pack_int4(cw)
    acc, _ = run(qa, qw, np.ones(N, np.float32), np.ones(O_, np.float32))
    assert np.array_equal(acc, O.unpack_int4(qa)[:, sel].astype(np.int32))
