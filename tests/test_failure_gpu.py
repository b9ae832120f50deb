"""Device-side failure detection on the GPU, tested without a fault.

Every wait inside the kernels is bounded: after its limit it records a site
code in the device status word, skips the stores it guarded and lets the
kernel finish. Here a wait that nothing completes (a one-thread self-test
kernel with a 1 ms limit) gives up; the host reads the code and clears the
word. The word is sticky until read, and a stale code must not change what
later launches compute: the boundary kernels and the GEMM run correctly while
it is set.
"""
import numpy as np
import pytest
import torch

import oracle as O
import rotation_post_quantization_b200 as rq
import workloads as W
from parity_util import check_bf16_output, check_codes_on_own_h, oracle_boundary

pytestmark = pytest.mark.gpu

SITE_SELFTEST = 901


def test_bounded_wait_gives_up_and_reports_its_site():
    assert rq.respin_device_status() == 0
    rq.respin_selftest_wait_limit(1000)          # 1 ms, nothing arrives
    assert rq.respin_device_status() == SITE_SELFTEST
    assert rq.respin_device_status() == 0        # reading cleared it


def test_first_failure_is_kept_until_read():
    rq.respin_selftest_wait_limit(1000)
    rq.respin_selftest_wait_limit(1000)
    assert rq.respin_device_status() == SITE_SELFTEST
    assert rq.respin_device_status() == 0


@pytest.mark.parametrize("N", [40, 1301], ids=["cluster_kernel", "rowtile_kernel"])
def test_stale_status_does_not_change_later_launches(N):
    rq.respin_selftest_wait_limit(1000)
    torch.cuda.synchronize()
    fx = W.workload_fixture("llama2_7b", N=N)
    dev = "cuda"
    plan = rq.Plan(fx.D, fx.r, fx.U.astype(np.float32), fx.V.astype(np.float32))
    h = torch.empty(N, fx.D, dtype=torch.bfloat16, device=dev)
    q = torch.full((N, fx.D // 2), 0xAB, dtype=torch.uint8, device=dev)
    sc = torch.full((N,), -1.0, dtype=torch.float32, device=dev)
    rq.respin_boundary_forward(plan, fx.x.to(dev), fx.residual.to(dev), h, q, sc)
    O_ = 512
    qw = W.int4_packed_random(O_, fx.D, 0, W.TID_WEIGHTS)
    sw = W.weight_scales(O_, fx.D, 0)
    out = torch.empty(N, O_, dtype=torch.bfloat16, device=dev)
    rq.w4a4_gemm(q, sc, torch.from_numpy(qw).to(dev), torch.from_numpy(sw).to(dev), out)
    torch.cuda.synchronize()
    # the launches succeeded and left the earlier code in place
    assert rq.respin_device_status() == SITE_SELFTEST
    plan.destroy()
    hb = h.view(torch.int16).cpu().numpy().view(np.uint16)
    h64, _, _, _ = oracle_boundary(fx)
    check_bf16_output(hb, h64)
    check_codes_on_own_h(hb, q.cpu().numpy(), sc.cpu().numpy())
    want = O.w4a4_epilogue_bits(O.w4a4_acc_fp64(q.cpu().numpy(), qw), sc.cpu().numpy(), sw)
    assert np.array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)
    assert rq.respin_device_status() == 0
