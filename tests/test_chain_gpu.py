"""Llama-3-8B-shaped layer chain on the GPU (workload llama3_8b_stack, two
layers at a small token count), checked step by step.

Per layer: attention boundary (rank-32 fix + codes), W4A4 GEMM D -> 14336,
quant-only pass over the 14336-wide output, W4A4 GEMM 14336 -> D, MLP
boundary whose residual is the attention boundary's h' (the MLP nonlinearity
is omitted: the pages give no chain). Every step is re-anchored: the oracle
is fed the GPU's own inputs and must agree with the GPU's outputs (bf16 h'
within the bf16 tolerance, codes bit-exact on the GPU's h', GEMM outputs
bit-exact). The end-to-end drift of an oracle-only chain against the GPU
chain is reported and bounded.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rotation_post_quantization_b200 as rq
import workloads as W
from parity_util import check_bf16_output, check_codes_on_own_h

pytestmark = pytest.mark.gpu

D, MLP, N, LAYERS = 4096, 14336, 40, 2
WL = W.WORKLOADS["llama3_8b_stack"]


def factors(i):
    Q = W.orthonormal_basis(D, WL.k, seed=i)
    U, V = W.lowrank_factors(Q, W.plane_angles(WL.k, WL.nu), WL.r)
    return U.astype(np.float32), V.astype(np.float32)


def acts(seed, tid):
    return W.activations_bf16(N, D, n_outlier=WL.n_outlier, outlier_scale=WL.outlier_scale,
                              seed=seed, tensor_id=tid)


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def gemm_ref_bits(qa, sa, qw, sw):
    return O.w4a4_epilogue_bits(O.w4a4_acc_fp64(qa, qw), sa, sw)


def boundary(plan, x, res, dev):
    h = torch.empty(N, D, dtype=torch.bfloat16, device=dev)
    q = torch.empty(N, D // 2, dtype=torch.uint8, device=dev)
    s = torch.empty(N, dtype=torch.float32, device=dev)
    rq.respin_boundary_forward(plan, x, res, h, q, s)
    return h, q, s


def check_boundary(h, q, s, x, res, U, V):
    h64, _, _, _ = O.boundary_reference(x.float().cpu().numpy(), res.float().cpu().numpy(), U, V)
    check_bf16_output(bits(h), h64)
    check_codes_on_own_h(bits(h), q.cpu().numpy(), s.cpu().numpy())


def test_chain_two_layers_reanchored_and_drift():
    dev = "cuda"
    res = acts(99, W.TID_RESIDUAL).to(dev)
    res_oracle = res.float().cpu().numpy()
    qonly = rq.Plan(MLP, 0)
    for l in range(LAYERS):
        Ua, Va = factors(2 * l)
        Um, Vm = factors(2 * l + 1)
        pa, pm = rq.Plan(D, WL.r, Ua, Va), rq.Plan(D, WL.r, Um, Vm)
        wu, su = W.int4_packed_random(MLP, D, l, W.TID_WEIGHTS), W.weight_scales(MLP, D, l)
        wd, sd = W.int4_packed_random(D, MLP, 100 + l, W.TID_WEIGHTS), W.weight_scales(D, MLP, 100 + l)
        x_att = acts(100 + l, W.TID_X).to(dev)

        # attention boundary
        h1, q1, s1 = boundary(pa, x_att, res, dev)
        check_boundary(h1, q1, s1, x_att, res, Ua, Va)
        # up GEMM, bit-exact on the GPU's codes
        u = torch.empty(N, MLP, dtype=torch.bfloat16, device=dev)
        rq.w4a4_gemm(q1, s1, torch.from_numpy(wu).to(dev), torch.from_numpy(su).to(dev), u)
        assert np.array_equal(bits(u), gemm_ref_bits(q1.cpu().numpy(), s1.cpu().numpy(), wu, su))
        # quant-only pass, bit-exact on the GPU's GEMM output
        q2 = torch.empty(N, MLP // 2, dtype=torch.uint8, device=dev)
        s2 = torch.empty(N, dtype=torch.float32, device=dev)
        rq.respin_boundary_forward(qonly, u, None, None, q2, s2)
        check_codes_on_own_h(bits(u), q2.cpu().numpy(), s2.cpu().numpy())
        # down GEMM
        xm = torch.empty(N, D, dtype=torch.bfloat16, device=dev)
        rq.w4a4_gemm(q2, s2, torch.from_numpy(wd).to(dev), torch.from_numpy(sd).to(dev), xm)
        assert np.array_equal(bits(xm), gemm_ref_bits(q2.cpu().numpy(), s2.cpu().numpy(), wd, sd))
        # MLP boundary: residual = the attention boundary's h'
        h2, q3, s3 = boundary(pm, xm, h1, dev)
        check_boundary(h2, q3, s3, xm, h1, Um, Vm)
        assert rq.respin_device_status() == 0

        # oracle-only chain from the same starting point
        xa = x_att.float().cpu().numpy()
        _, hb1, c1, sc1 = O.boundary_reference(xa, res_oracle, Ua, Va)
        u_o = O.bf16_bits_to_f32(gemm_ref_bits(O.pack_int4(c1), sc1, wu, su))
        c2, sc2 = O.quantize_int4_per_token(u_o)
        xm_o = O.bf16_bits_to_f32(gemm_ref_bits(O.pack_int4(c2), sc2, wd, sd))
        _, hb2, _, _ = O.boundary_reference(xm_o, O.bf16_bits_to_f32(hb1), Um, Vm)
        res_oracle = O.bf16_bits_to_f32(hb2)
        res = h2
        pa.destroy()
        pm.destroy()

    gpu = res.float().cpu().numpy().astype(np.float64)
    ref = res_oracle.astype(np.float64)
    drift = np.linalg.norm(gpu - ref) / np.linalg.norm(ref)
    print("end-to-end drift after %d layers: %.3e (relative Frobenius)" % (LAYERS, drift))
    assert drift < 1e-2
