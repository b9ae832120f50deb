"""Parity at the full sizes the benchmark times (seeded row samples; every
token's result depends only on its own row, so a sampled row is checked
exactly).

* Llama-3-8B-shaped chain (4096 tokens, D = 4096, MLP 14336): two layers of
  attention boundary -> W4A4 GEMM 4096 -> 14336 -> quant-only pass -> W4A4
  GEMM 14336 -> 4096 -> MLP boundary, through the pair boundary kernel and
  the CTA-pair tensor-memory GEMM. Every step is re-anchored (the oracle gets
  the GPU's inputs of that step) on 192 seeded rows; the drift of an
  oracle-only chain over the same rows is reported and bounded.
* Llama-2-70B-shaped boundary (D = 8192, 8192 tokens, Student-t inputs) at
  r = 64 and r = 128, fp32 h' and bf16 h' on 256 seeded rows.
* The GEMMs 8192 x 8192 -> 28672 and 4096 x 4096 -> 14336 at their full
  token counts, accumulators and bf16 outputs bit-exact on seeded rows.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rotation_post_quantization_b200 as rq
import workloads as W
from parity_util import (check_bf16_output, check_codes_end_to_end, check_codes_on_own_h, check_corr,
                         check_h_f32)

pytestmark = pytest.mark.gpu


def bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def sample_rows(N, n, seed):
    return np.sort(np.random.default_rng([seed, 77]).choice(N, size=n, replace=False))


def gemm_bits(qa, sa, qw, sw):
    return O.w4a4_epilogue_bits(O.w4a4_acc_fp64(qa, qw), sa, sw)


# ---------------------------------------------------------------- chain

def test_llama3_8b_chain_full_tokens_reanchored():
    wl = W.WORKLOADS["llama3_8b_stack"]
    D, MLP, N, L = wl.D, wl.extra["mlp"], wl.N, 2
    dev = "cuda"
    rows = sample_rows(N, 192, 1)
    kw = dict(n_outlier=wl.n_outlier, outlier_scale=wl.outlier_scale)
    res = W.activations_bf16_fast(N, D, tensor_id=W.TID_RESIDUAL, seed=99, **kw)
    res_o = res.float().numpy()[rows]        # oracle-only chain over the sampled rows
    res = res.to(dev)
    qonly = rq.Plan(MLP, 0)
    worst = {}
    for l in range(L):
        plans, subs = [], []
        for i in (2 * l, 2 * l + 1):
            Qr, R = W.subspace_factors(W.orthonormal_basis(D, wl.k, seed=i), W.plane_angles(wl.k, wl.nu), wl.r)
            subs.append((Qr.astype(np.float32), R.astype(np.float32)))
            plans.append(rq.SubspacePlan(D, wl.r, *subs[-1]))
        wu, su = W.int4_packed_random(MLP, D, l, W.TID_WEIGHTS), W.weight_scales(MLP, D, l)
        wd, sd = W.int4_packed_random(D, MLP, 100 + l, W.TID_WEIGHTS), W.weight_scales(D, MLP, 100 + l)
        x_att = W.activations_bf16_fast(N, D, tensor_id=W.TID_X, seed=100 + l, **kw).to(dev)

        h1 = torch.empty(N, D, dtype=torch.bfloat16, device=dev)
        q1 = torch.empty(N, D // 2, dtype=torch.uint8, device=dev)
        s1 = torch.empty(N, dtype=torch.float32, device=dev)
        rq.respin_boundary_forward(plans[0], x_att, res, h1, q1, s1)
        u = torch.empty(N, MLP, dtype=torch.bfloat16, device=dev)
        rq.w4a4_gemm(q1, s1, torch.from_numpy(wu).to(dev), torch.from_numpy(su).to(dev), u)
        q2 = torch.empty(N, MLP // 2, dtype=torch.uint8, device=dev)
        s2 = torch.empty(N, dtype=torch.float32, device=dev)
        rq.respin_boundary_forward(qonly, u, None, None, q2, s2)
        xm = torch.empty(N, D, dtype=torch.bfloat16, device=dev)
        rq.w4a4_gemm(q2, s2, torch.from_numpy(wd).to(dev), torch.from_numpy(sd).to(dev), xm)
        h2 = torch.empty(N, D, dtype=torch.bfloat16, device=dev)
        q3 = torch.empty(N, D // 2, dtype=torch.uint8, device=dev)
        s3 = torch.empty(N, dtype=torch.float32, device=dev)
        rq.respin_boundary_forward(plans[1], xm, h1, h2, q3, s3)
        torch.cuda.synchronize()
        assert rq.respin_device_status() == 0

        rs_ = lambda t: t[rows]
        # attention boundary, re-anchored on the GPU's inputs
        h64, _, _, _ = O.boundary_reference_subspace(rs_(x_att).float().cpu().numpy(),
                                                     rs_(res).float().cpu().numpy(), *subs[0])
        worst[("attn", l)] = check_bf16_output(bits(rs_(h1)), h64)
        check_codes_on_own_h(bits(rs_(h1)), rs_(q1).cpu().numpy(), rs_(s1).cpu().numpy())
        # up GEMM on the GPU's codes
        assert np.array_equal(bits(rs_(u)), gemm_bits(rs_(q1).cpu().numpy(), rs_(s1).cpu().numpy(), wu, su))
        # quant-only on the GPU's GEMM output
        check_codes_on_own_h(bits(rs_(u)), rs_(q2).cpu().numpy(), rs_(s2).cpu().numpy())
        # down GEMM
        assert np.array_equal(bits(rs_(xm)), gemm_bits(rs_(q2).cpu().numpy(), rs_(s2).cpu().numpy(), wd, sd))
        # MLP boundary, residual = the GPU's attention h'
        h64, _, _, _ = O.boundary_reference_subspace(rs_(xm).float().cpu().numpy(),
                                                     rs_(h1).float().cpu().numpy(), *subs[1])
        worst[("mlp", l)] = check_bf16_output(bits(rs_(h2)), h64)
        check_codes_on_own_h(bits(rs_(h2)), rs_(q3).cpu().numpy(), rs_(s3).cpu().numpy())

        # oracle-only chain over the sampled rows
        _, hb1, c1, sc1 = O.boundary_reference_subspace(rs_(x_att).float().cpu().numpy(), res_o, *subs[0])
        u_o = O.bf16_bits_to_f32(gemm_bits(O.pack_int4(c1), sc1, wu, su))
        c2, sc2 = O.quantize_int4_per_token(u_o)
        xm_o = O.bf16_bits_to_f32(gemm_bits(O.pack_int4(c2), sc2, wd, sd))
        _, hb2, _, _ = O.boundary_reference_subspace(xm_o, O.bf16_bits_to_f32(hb1), *subs[1])
        res_o = O.bf16_bits_to_f32(hb2)
        res = h2
        for p in plans:
            p.destroy()
    gpu = res[rows].float().cpu().numpy().astype(np.float64)
    drift = np.linalg.norm(gpu - res_o) / np.linalg.norm(res_o)
    print("4096-token chain: worst bf16 relative error per step %s; oracle-only drift after %d layers "
          "on %d rows: %.3e" % ({k: "%.2e" % v for k, v in worst.items()}, L, len(rows), drift))
    assert drift < 1e-2


# ---------------------------------------------------------------- 70B boundary

@pytest.mark.parametrize("r", [64, 128])
def test_llama2_70b_boundary_full_tokens(r):
    wl = W.WORKLOADS["llama2_70b"]
    D, N = wl.D, wl.N
    dev = "cuda"
    Q = W.orthonormal_basis(D, wl.k, seed=0)
    U, V = W.lowrank_factors(Q, W.plane_angles(wl.k, wl.nu), r)
    U32, V32 = U.astype(np.float32), V.astype(np.float32)
    kw = dict(n_outlier=wl.n_outlier, outlier_scale=wl.outlier_scale, dist=wl.dist)
    x = W.activations_bf16_fast(N, D, tensor_id=W.TID_X, seed=5, **kw)
    res = W.activations_bf16_fast(N, D, tensor_id=W.TID_RESIDUAL, seed=5, **kw)
    rows = sample_rows(N, 256, r)
    xs, rs_ = x.float().numpy()[rows], res.float().numpy()[rows]
    h64, _, codes_ref, _ = O.boundary_reference(xs, rs_, U32, V32)
    for f32 in (True, False):
        plan = rq.Plan(D, r, U32, V32, rq.RESPIN_H_FP32_DEBUG if f32 else 0)
        h = torch.empty(N, D, dtype=torch.float32 if f32 else torch.bfloat16, device=dev)
        q = torch.empty(N, D // 2, dtype=torch.uint8, device=dev)
        s = torch.empty(N, dtype=torch.float32, device=dev)
        rq.respin_boundary_forward(plan, x.to(dev), res.to(dev), h, q, s)
        torch.cuda.synchronize()
        assert rq.respin_device_status() == 0
        plan.destroy()
        hs, qs, ss = h[rows].cpu().numpy() if f32 else bits(h[rows]), q[rows].cpu().numpy(), s[rows].cpu().numpy()
        if f32:
            check_h_f32(hs, h64)
            Uq, Vq = O.plan_factors(U32, V32)
            check_corr(hs, xs.astype(np.float64), rs_.astype(np.float64), Uq, Vq)
            check_codes_on_own_h(O.bf16_bits(hs), qs, ss)
        else:
            check_bf16_output(hs, h64)
            check_codes_on_own_h(hs, qs, ss)
        check_codes_end_to_end(qs, codes_ref)


# ---------------------------------------------------------------- GEMMs

@pytest.mark.parametrize("N,K,O_", [(8192, 8192, 28672), (4096, 4096, 14336), (4096, 14336, 4096)],
                         ids=["70b_8192x8192x28672", "8b_up_4096x4096x14336", "8b_down_4096x14336x4096"])
def test_gemm_full_tokens(N, K, O_):
    dev = "cuda"
    qa = W.int4_packed_random(N, K, 3, W.TID_ACODES)
    qw = W.int4_packed_random(O_, K, 3, W.TID_WEIGHTS)
    sa = W.activation_scales(N, 3)
    sw = W.weight_scales(O_, K, 3)
    tqa, tqw = torch.from_numpy(qa).to(dev), torch.from_numpy(qw).to(dev)
    out = torch.empty(N, O_, dtype=torch.bfloat16, device=dev)
    rq.w4a4_gemm(tqa, torch.from_numpy(sa).to(dev), tqw, torch.from_numpy(sw).to(dev), out)
    rows = sample_rows(N, 128, N + K + O_)
    torch.cuda.synchronize()
    outb = bits(out[rows])
    del out
    acc = torch.empty(N, O_, dtype=torch.int32, device=dev)
    rq.w4a4_gemm_i32(tqa, tqw, acc)
    torch.cuda.synchronize()
    assert rq.respin_device_status() == 0
    acc_s = acc[rows].cpu().numpy().astype(np.int64)
    del acc
    ref = O.w4a4_acc_fp64(qa[rows], qw)
    assert np.array_equal(acc_s, ref), "int32 accumulators differ"
    assert np.array_equal(outb, O.w4a4_epilogue_bits(ref, sa[rows], sw)), "bf16 outputs differ"
