"""CUDA-graph capture of the library calls: each boundary path (row tiles,
CTA pairs, clusters of 4, the three tensor-core passes with their dependent
launches) and the W4A4 GEMM, captured once and replayed, must give the eager
call's outputs bit for bit."""
import numpy as np
import pytest
import torch

import rotation_post_quantization_b200 as rq
import workloads as W

pytestmark = pytest.mark.gpu

CASES = [
    # (name, D, N, r, form)
    ("rowtile", 4096, 2048, 32, "factor"),
    ("pair", 4096, 2048, 32, "subspace"),
    ("quad", 4096, 64, 32, "subspace"),
    ("tc_r64", 8192, 512, 64, "factor"),
]


def _plan(D, r, form, k):
    Q = W.orthonormal_basis(D, k, 0)
    th = W.plane_angles(k, 0.1)
    if form == "subspace":
        Qr, R = W.subspace_factors(Q, th, r)
        return rq.SubspacePlan(D, r, Qr.astype(np.float32), R.astype(np.float32))
    U, V = W.lowrank_factors(Q, th, r)
    return rq.Plan(D, r, U.astype(np.float32), V.astype(np.float32))


def _graph(fn):
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()   # first call outside the capture (plan set-up is done by now)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        fn()
    return g


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_boundary_graph_replay_matches_eager(case):
    _, D, N, r, form = case
    plan = _plan(D, r, form, k=max(2 * r, 64))
    dev = "cuda"
    x = W.activations_bf16_fast(N, D, tensor_id=W.TID_X, n_outlier=8, outlier_scale=50.0, seed=1, device=dev)
    res = W.activations_bf16_fast(N, D, tensor_id=W.TID_RESIDUAL, n_outlier=8, outlier_scale=50.0, seed=2, device=dev)
    outs = []
    for mode in ("eager", "graph"):
        h = torch.full((N, D), 7.0, dtype=torch.bfloat16, device=dev)
        q = torch.full((N, D // 2), 0xAB, dtype=torch.uint8, device=dev)
        s = torch.full((N,), -1.0, dtype=torch.float32, device=dev)
        fn = lambda: rq.respin_boundary_forward(plan, x, res, h, q, s)
        if mode == "eager":
            fn()
        else:
            g = _graph(fn)
            h.fill_(7.0); q.fill_(0xAB); s.fill_(-1.0)
            g.replay()
            g.replay()
        torch.cuda.synchronize()
        assert rq.respin_device_status() == 0
        outs.append((h.view(torch.int16).cpu(), q.cpu(), s.view(torch.int32).cpu()))
    plan.destroy()
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_gemm_graph_replay_matches_eager():
    N, K, O = 2048, 4096, 1024
    g0 = torch.Generator(device="cuda")
    g0.manual_seed(3)
    qa = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device="cuda", generator=g0)
    sa = torch.rand(N, device="cuda", generator=g0) + 0.5
    qw = torch.randint(0, 256, (O, K // 2), dtype=torch.uint8, device="cuda", generator=g0)
    sw = (torch.rand(O, device="cuda", generator=g0) + 0.5) / 300
    outs = []
    for mode in ("eager", "graph"):
        out = torch.zeros(N, O, dtype=torch.bfloat16, device="cuda")
        fn = lambda: rq.w4a4_gemm(qa, sa, qw, sw, out)
        if mode == "eager":
            fn()
        else:
            g = _graph(fn)
            out.zero_()
            g.replay()
        torch.cuda.synchronize()
        assert rq.respin_device_status() == 0
        outs.append(out.view(torch.int16).cpu())
    assert torch.equal(outs[0], outs[1])
