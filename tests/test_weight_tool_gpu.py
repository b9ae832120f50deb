"""Rotation-fused INT4 weights feeding the W4A4 GEMM (Llama-2-7B-shaped
input width K = 4096). A linear y = W x runs on activations that arrive in
the rotated basis (x~ = R_in^T x, row form a~ = a R_in); with the weight
fused offline (W~ = W R_in, zh §2.2 offline weight merging; fr §2A) and both
operands quantized per token / per channel, the GEMM must reproduce the
oracle bit for bit on its codes and approximate a W^T within the INT4 error,
while the unfused weight does not."""
import numpy as np
import pytest
import torch

import oracle as O
import rotation_post_quantization_b200 as rq
import workloads as W

pytestmark = pytest.mark.gpu


def test_fused_int4_weights_feed_the_gemm():
    K, O_, N = 4096, 512, 200
    wl = W.WORKLOADS["llama2_7b"]
    Q = W.orthonormal_basis(K, wl.k, 0)
    R_in, _ = O.rotation_pair(Q, W.plane_angles(wl.k, wl.nu))       # H expm(A), dense
    rs = np.random.default_rng(11)
    Wt = (rs.standard_normal((O_, K)) / np.sqrt(K)).astype(np.float32)
    a = W.activations_bf16(N, K, n_outlier=wl.n_outlier, outlier_scale=wl.outlier_scale, seed=3)
    a64 = a.float().numpy().astype(np.float64)
    # activations in the rotated basis (the boundary's output), then per-token codes
    a_rot = torch.from_numpy((a64 @ R_in).astype(np.float32)).to(torch.bfloat16)
    plan = rq.Plan(K, 0)
    dev = "cuda"
    q = torch.empty(N, K // 2, dtype=torch.uint8, device=dev)
    sa = torch.empty(N, dtype=torch.float32, device=dev)
    rq.respin_boundary_forward(plan, a_rot.to(dev), None, None, q, sa)
    Wf = rq.respin_fuse_weight(Wt, R_in.astype(np.float32))
    results = {}
    for name, w in (("fused", Wf), ("unfused", Wt)):
        qw, sw = rq.respin_quantize_weight(w, 7)
        out = torch.empty(N, O_, dtype=torch.bfloat16, device=dev)
        rq.w4a4_gemm(q, sa, torch.from_numpy(qw).to(dev), torch.from_numpy(sw).to(dev), out)
        torch.cuda.synchronize()
        assert rq.respin_device_status() == 0
        bits = out.view(torch.int16).cpu().numpy().view(np.uint16)
        want = O.w4a4_epilogue_bits(O.w4a4_acc_fp64(q.cpu().numpy(), qw), sa.cpu().numpy(), sw)
        assert np.array_equal(bits, want)
        got = O.bf16_bits_to_f32(bits).astype(np.float64)
        ref = a64 @ Wt.astype(np.float64).T                 # the unrotated linear
        results[name] = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    plan.destroy()
    print("W4A4 relative error vs a W^T: fused %.3f, unfused %.3f" % (results["fused"], results["unfused"]))
    assert results["fused"] < 0.25
    assert results["unfused"] > 0.9
