"""W4A4 GEMM with per-token tile maxima of its output, and the per-token
quantization that uses them (the quant-only step between the up and down
projections, with its reduction moved into the GEMM epilogue): outputs equal
the plain GEMM bit for bit, the maxima equal max |out| per 256-channel tile,
and the codes and scales equal both the oracle quantizer on the GEMM's output
and the r = 0 boundary call on it."""
import numpy as np
import pytest
import torch

import oracle as O
import rotation_post_quantization_b200 as rq
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K,O_,qmax", [(300, 4096, 14336, 7), (4096, 4096, 14336, 7), (257, 1024, 1040, 3)])
def test_gemm_rowmax_and_quantize(N, K, O_, qmax):
    dev = "cuda"
    g = torch.Generator(device=dev)
    g.manual_seed(N + O_)
    qa = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g)
    sa = torch.rand(N, device=dev, generator=g) + 0.5
    qw = torch.from_numpy(W.int4_packed_random(O_, K, 0, W.TID_WEIGHTS)).to(dev)
    sw = torch.from_numpy(W.weight_scales(O_, K, 0)).to(dev)
    out_ref = torch.empty(N, O_, dtype=torch.bfloat16, device=dev)
    out = torch.empty(N, O_, dtype=torch.bfloat16, device=dev)
    parts = (O_ + 255) // 256
    rm = torch.full((N, parts), -1.0, dtype=torch.float32, device=dev)
    rq.w4a4_gemm(qa, sa, qw, sw, out_ref)
    rq.w4a4_gemm_rowmax(qa, sa, qw, sw, out, rm)
    torch.cuda.synchronize()
    assert rq.respin_device_status() == 0
    ob = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(ob, out_ref.view(torch.int16).cpu().numpy().view(np.uint16))
    u = np.abs(O.bf16_bits_to_f32(ob))
    pad = np.zeros((N, parts * 256), np.float32)
    pad[:, :O_] = u
    want = pad.reshape(N, parts, 256).max(axis=2)
    assert np.array_equal(rm.cpu().numpy(), want)
    if O_ % 256:
        return   # the code pass needs D % 256 == 0
    flags = rq.RESPIN_ACT_INT3 if qmax == 3 else 0
    q = torch.full((N, O_ // 2), 0xAB, dtype=torch.uint8, device=dev)
    s = torch.full((N,), -1.0, dtype=torch.float32, device=dev)
    rq.respin_quantize_rowmax(out, rm, q, s, flags)
    plan = rq.Plan(O_, 0, flags=flags)
    q2 = torch.empty_like(q)
    s2 = torch.empty_like(s)
    rq.respin_boundary_forward(plan, out, None, None, q2, s2)
    torch.cuda.synchronize()
    assert rq.respin_device_status() == 0
    plan.destroy()
    assert torch.equal(q, q2) and torch.equal(s.view(torch.int32), s2.view(torch.int32))
    codes, scale = O.quantize_per_token(O.bf16_bits_to_f32(ob), qmax)
    assert np.array_equal(q.cpu().numpy(), O.pack_int4(codes))
    assert np.array_equal(s.cpu().numpy().view(np.uint32), scale.view(np.uint32))
