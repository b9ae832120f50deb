#!/usr/bin/env python
"""Benchmark of the ReSpinQuant block-boundary hot path on B200.

One step = the whole path on one batch of tokens: the fused boundary kernel
(rank-r basis fix + per-token INT4 quantization, ReSpinQuant explainers zh
§2.2 and §3-§4) followed by the tcgen05 W4A4 GEMM that consumes its codes.
Workload: Llama-2-7B-shaped, D = 4096, 2048 tokens per GPU, r = 32 (rank-64
skew deviation, norm 0.1, 8 outlier channels x50), GEMM 4096 -> 11008 with
INT4 weights uniform in [-8, 7]. Synthetic, seeded inputs. The boundary plan
is built from the stored subspace form (basis Q and rotation R_sub, zh §2.2)
or from the factor pair (U_r, V_r), --boundary-form. --workload
llama2_7b_w3a3 runs the same step with 3-bit activation and weight codes
(W3A3); the other --workload names print the remaining configurations, which
the default run also reports in its `workloads` object.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--boundary-form subspace|factor]

Under torchrun each rank processes its own 2048 tokens (weak scaling, no
data-path collective); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "tokens/s fused ΔT-lowrank+INT4 quant (D=4096,r=32); W4A4 GEMM TOPS"
WORKLOAD = "llama2_7b"
# The headline step in its two quantization settings: activation (and weight)
# code width per --workload name.
STEP_BITS = {"llama2_7b": 4, "llama2_7b_w3a3": 3}


def metric(bits: int) -> str:
    return METRIC if bits == 4 else METRIC.replace("INT4", "INT3").replace("W4A4", "W3A3")
NSETS = 4            # rotating input sets: 4 x 56 MB > 126 MB L2
DEFAULT_FORM = "factor"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 / 2.25 PFLOP/s)


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-workloads", action="store_true",
                   help="skip the other workload configurations in the default run")
    p.add_argument("--boundary-form", choices=["subspace", "factor"], default=DEFAULT_FORM,
                   help="boundary plan of the headline step: the stored subspace form "
                        "(basis Q, rotation R_sub) or the factor pair (U_r, V_r)")
    p.add_argument("--repeat", type=int, default=10,
                   help="extra timed blocks of --steps steps after the timed region, "
                        "reported as their median (supplementary steadiness figure)")
    p.add_argument("--profile-launch", choices=["boundary", "gemm"],
                   help="profiling aid: warm up, then launch one kernel once "
                        "(for ncu captures); prints no bench line")
    p.add_argument("--tokens", type=int, default=None,
                   help="tokens for --profile-launch (default: the workload's)")
    p.add_argument("--rank", type=int, default=None,
                   help="rank for --profile-launch (default: the workload's; "
                        "with --workload llama2_70b the factor plan of that rank)")
    p.add_argument("--workload", default="llama2_7b",
                   choices=["llama2_7b", "llama2_7b_w3a3", "tiny", "decode", "llama2_70b",
                            "llama3_8b_stack"],
                   help="llama2_7b (default): the headline step; llama2_7b_w3a3: the "
                        "same step with 3-bit activation and weight codes. The others "
                        "print one JSON line each for the remaining workload "
                        "configurations (1 GPU)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            m = json.load(fh)
        return float(m["hbm_gbs"]), float(m["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# ---------------------------------------------------------------- clocks

REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting",
           0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x10: "sync_boost",
           0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
           0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler(threading.Thread):
    """Polls NVML (read only) for SM clock, throttle reasons and power."""

    def __init__(self, torch_device: int, period_s: float = 0.005):
        super().__init__(daemon=True)
        self.period = period_s
        self.samples = []
        self.stop_evt = threading.Event()
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            pr = torch.cuda.get_device_properties(torch_device)
            bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id,
                                        pr.pci_device_id)
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(
                self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)

    def run(self):
        if not self.ok:
            return
        nv = self.nv
        while not self.stop_evt.is_set():
            try:
                t = time.time()
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((t, mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def wait_first(self, limit_s: float = 2.0):
        """Block until the thread has taken its first sample (the first NVML
        query can take longer than a short timed region), at most limit_s."""
        t_end = time.time() + limit_s
        while self.ok and not self.samples and time.time() < t_end:
            time.sleep(0.005)

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [],
                    "samples": 0, "note": getattr(self, "err", "nvml")}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        if not win:   # region shorter than the poll period: nearest samples
            win = sorted(self.samples, key=lambda s: abs(s[0] - t1))[:2]
        mhz = sorted(s[1] for s in win)
        mask = 0
        for s in win:
            mask |= s[2]
        reasons = [n for b, n in REASONS.items() if mask & b and b != 0x1]
        return {"sm_mhz": mhz[len(mhz) // 2] if mhz else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(win)}


# ---------------------------------------------------------------- oracle legs
#
# The CPU baseline is the C++ oracle as it stands (plain single-threaded
# loops, -O2, no fast-math), with the calling thread pinned to one core;
# every figure is the median of 5 runs of a bounded sample of the workload,
# boundary tokens/s and GEMM GOPS reported separately.

ORACLE_REPS = 5


def host_cpu() -> str:
    """CPU model of the host (the oracle's machine) and its logical core count."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return "%s, %d logical cores" % (model, os.cpu_count() or 0)


def _pinned(fn):
    """fn() with the calling thread pinned to one CPU; returns (result, cpu)."""
    prev = cpu = None
    try:
        prev = os.sched_getaffinity(0)
        cpu = min(prev)
        os.sched_setaffinity(0, {cpu})
    except (AttributeError, OSError):
        prev = None
    try:
        return fn(), cpu
    finally:
        if prev is not None:
            os.sched_setaffinity(0, prev)


def _median_s(fn, reps: int = ORACLE_REPS) -> float:
    ts = []
    for _ in range(reps):
        t0 = time.perf_counter()
        fn()
        ts.append(time.perf_counter() - t0)
    return sorted(ts)[len(ts) // 2]


def _bits(t):
    import numpy as np
    import torch
    return t.view(torch.int16).numpy().view(np.uint16)


def oracle_boundary_tps(x, res, factors, form: str, qmax: int = 7) -> float:
    """Oracle boundary tokens/s on the rows of x / res (bf16 CPU tensors);
    factors = (U, V) for the factor form, (Q, R_sub) for the subspace form."""
    import numpy as np
    from oracle import native
    native.lib()
    xb, rb = _bits(x), _bits(res) if res is not None else None
    A, B = (np.ascontiguousarray(f, np.float32) for f in factors)
    call = native.boundary_reference_subspace if form == "subspace" else native.boundary_reference
    t = _median_s(lambda: call(xb, rb, A, B, qmax, want_h64=False))
    return x.shape[0] / t


def oracle_gemm_gops(qa, sa, qw, sw) -> float:
    """Oracle W4A4 GEMM GOPS (2 ops per multiply-add) on the rows of qa."""
    from oracle import native
    native.lib()
    t = _median_s(lambda: native.w4a4_gemm(qa, sa, qw, sw))
    return 2.0 * qa.shape[0] * 2 * qa.shape[1] * qw.shape[0] / t / 1e9


def step_cpu_baseline(fx, qw, sw, form: str, bits: int, n_boundary: int, n_gemm: int) -> dict:
    """The headline step on the oracle: boundary on n_boundary tokens and the
    GEMM on n_gemm rows; tokens/s of the whole step per token."""
    import numpy as np
    from oracle import native

    def run():
        factors = subspace_of(fx) if form == "subspace" else (fx.U, fx.V)
        b = oracle_boundary_tps(fx.x[:n_boundary], fx.residual[:n_boundary], factors, form, 7 if bits == 4 else 3)
        _, _, codes, scale = native.boundary_reference(_bits(fx.x[:n_gemm]), _bits(fx.residual[:n_gemm]),
                                                       fx.U.astype(np.float32), fx.V.astype(np.float32),
                                                       7 if bits == 4 else 3, want_h64=False)
        gops = oracle_gemm_gops(native.pack(codes), scale, qw, sw)
        return b, gops
    (b, gops), cpu = _pinned(run)
    K, O_ = fx.D, qw.shape[0]
    per_tok = 1.0 / b + 2.0 * K * O_ / (gops * 1e9)
    return {"value": 1.0 / per_tok, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "boundary_tokens_per_s": b, "gemm_gops": gops, "cpu": host_cpu(), "pinned_cpu": cpu,
            "sample": "C++ oracle (plain loops, -O2, one thread pinned to one core), median of %d: "
                      "boundary (fp64 fix, %s form, + binary32 INT%d quantizer) on %d tokens, "
                      "W%dA%d GEMM (exact int64 + binary32 epilogue) on %d rows x %d channels; "
                      "step tokens/s = 1 / (boundary s/token + GEMM s/token)"
                      % (ORACLE_REPS, form, bits, n_boundary, bits, bits, n_gemm, O_)}


def subspace_of(fx):
    """(Q, R_sub) of a fixture's stored subspace form (float64)."""
    import workloads as W
    return W.subspace_factors(fx.Q, fx.theta, fx.r)


def weight_codes(W, bits: int, rows: int, K: int, seed: int):
    return (W.int4_packed_random if bits == 4 else W.int3_packed_random)(rows, K, seed, W.TID_WEIGHTS)


def workload_inputs(device: str | None, bits: int = 4):
    import numpy as np
    import workloads as W
    w = W.WORKLOADS[WORKLOAD]
    fx = W.workload_fixture(WORKLOAD)
    K = w.D
    qw = weight_codes(W, bits, w.O, K, 0)
    sw = W.weight_scales(w.O, K, 0)
    return w, fx, qw, sw


def run_reference(args, rank: int):
    """The reference arm: the CPU oracle, timed on the host cores. One step is
    a bounded sample of the headline step (boundary on 256 tokens, GEMM on 16
    rows); ms_per_step is that sample's measured time, value the oracle's
    tokens/s of the whole step (per-token costs of both parts)."""
    if rank != 0:
        return
    import numpy as np
    from oracle import native
    bits = STEP_BITS.get(args.workload, 4)
    form = args.boundary_form
    w, fx, qw, sw = workload_inputs(None, bits)
    qmax = 7 if bits == 4 else 3
    nb, ng = 256, 16
    factors = subspace_of(fx) if form == "subspace" else (fx.U, fx.V)
    A, B = (np.ascontiguousarray(f, np.float32) for f in factors)
    call = native.boundary_reference_subspace if form == "subspace" else native.boundary_reference
    xb, rb = _bits(fx.x[:nb]), _bits(fx.residual[:nb])
    _, _, codes, scale = native.boundary_reference(_bits(fx.x[:ng]), _bits(fx.residual[:ng]),
                                                   fx.U.astype(np.float32), fx.V.astype(np.float32),
                                                   qmax, want_h64=False)
    qa = native.pack(codes)

    def one_step():
        t0 = time.perf_counter()
        call(xb, rb, A, B, qmax, want_h64=False)
        t1 = time.perf_counter()
        native.w4a4_gemm(qa, scale, qw, sw)
        t2 = time.perf_counter()
        return t1 - t0, t2 - t1

    def run():
        for _ in range(max(0, args.warmup)):
            one_step()
        return [one_step() for _ in range(args.steps)]
    samples, cpu = _pinned(run)
    tb = sum(s[0] for s in samples) / len(samples)
    tg = sum(s[1] for s in samples) / len(samples)
    per_tok = tb / nb + tg / ng
    value = 1.0 / per_tok
    line = {
        "impl": "reference", "metric": metric(bits), "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": (tb + tg) * 1e3,
        "ms_per_step_is": "the timed sample step: boundary on %d tokens + GEMM on %d rows "
                          "(value = the oracle's per-token cost of the whole step)" % (nb, ng),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64+f32+int64", "data": "synthetic",
        "config": config_block(w, args.gpus, bits, form),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "pinned_cpu": cpu,
                         "kind": "oracle", "cpu": host_cpu(),
                         "boundary_tokens_per_s": nb / tb,
                         "gemm_gops": 2.0 * ng * w.D * w.O / tg / 1e9,
                         "sample": "each step: C++ oracle, boundary (%s form) on %d tokens + "
                                   "GEMM on %d rows x %d channels, one thread pinned to one core"
                                   % (form, nb, ng, w.O)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_block(w, n_gpus, bits: int = 4, form: str = "subspace"):
    return {"workload": "Llama-2-7B-shaped boundary + W%dA%d GEMM: D=4096, "
                        "2048 tokens/GPU, r=32, GEMM 4096->11008" % (bits, bits),
            "boundary_plan": "stored subspace form (Q, R_sub)" if form == "subspace"
                             else "factor pair (U_r, V_r)",
            "act_bits": bits, "weight_bits": bits,
            "D": w.D, "tokens_per_gpu": w.N, "r": w.r, "gemm_out": w.O,
            "global_batch": w.N * n_gpus, "parallelism": "dp%d" % n_gpus,
            "l2": "inputs larger than L2: %d rotating input sets of %.0f MB"
                  % (NSETS, (2 * w.N * w.D * 2 + w.O * w.D // 2) / 1e6)}


def traffic_for(kernel_file: str, name: str):
    """ncu DRAM bytes per launch recorded for this exact kernel source, or
    None when the kernel changed since the capture."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    src = os.path.join(ROOT, "rotation_post_quantization_b200", "csrc",
                       kernel_file)
    try:
        with open(path) as fh:
            rec = json.load(fh).get(name)
        with open(src, "rb") as fh:
            sha = hashlib.sha256(fh.read()).hexdigest()
        if rec and rec.get("source_sha256") == sha:
            return rec["bytes_per_launch"]
    except Exception:
        pass
    return None


# ---------------------------------------------------------------- ranks

def rank_env():
    """(rank, world size, local rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(backend: str, device=None, timeout_s: float = 120.0):
    """Process group for the barrier and the max-over-ranks reduction; a short
    timeout so that ranks waiting for a dead peer end with an error."""
    import datetime
    import torch.distributed as dist
    kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)
    return dist


def max_over_ranks(values, dist, device=None):
    """Element-wise maximum of per-rank timings (every rank gets the result);
    the identity without a process group."""
    import torch
    if dist is None:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tokens_per_s(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job throughput under weak scaling: every rank processes its own
    tokens_per_rank tokens per step, the step lasts the slowest rank's time."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def rank_seed(rank: int, i: int) -> int:
    """Seed of input set i on a rank: ranks hold different tokens (shards of
    the batch), set i of rank 0 is the workload's own fixture."""
    return 1000 * rank + i


# ---------------------------------------------------------------- our arm

def boundary_bytes(N: int, D: int, r: int, form: str) -> float:
    """Algorithmic HBM bytes of one boundary launch: x, residual and h' (bf16),
    codes (D/2 bytes), scale (4 bytes) per token, plus the plan's factors once
    (the basis Q for a subspace plan, U_r and V_r for a factor plan)."""
    return N * (6.5 * D + 4) + (1 if form == "subspace" else 2) * D * r * 2


def boundary_kernel_of(form: str, N: int):
    """(kernel name, source file) that serves a headline-shaped boundary call."""
    if form == "subspace":
        return "boundary_pair_kernel", "boundary_pair.cuh"
    return ("boundary_rowtile_kernel", "boundary_rowtile.cuh") if N > 1280 else \
        ("boundary_cluster_rf_kernel", "boundary_kernels.cuh")


def run_ours(args, rank: int, world: int, local_rank: int):
    import numpy as np
    import torch
    import rotation_post_quantization_b200 as rq
    import workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = init_dist("nccl", dev) if world > 1 else None

    bits = STEP_BITS[args.workload]
    form = args.boundary_form
    w, fx, qw_np, sw_np = workload_inputs("cuda", bits)
    D, N, r, O_ = w.D, w.N, w.r, w.O
    K = D
    pflags = rq.RESPIN_ACT_INT3 if bits == 3 else 0
    if form == "subspace":
        Qs, Rs = subspace_of(fx)
        plan = rq.SubspacePlan(D, r, Qs.astype(np.float32), Rs.astype(np.float32), pflags)
    else:
        plan = rq.Plan(D, r, fx.U.astype(np.float32), fx.V.astype(np.float32), pflags)

    sets = []
    for i in range(NSETS):
        kw = dict(n_outlier=w.n_outlier, outlier_scale=w.outlier_scale,
                  dist=w.dist, seed=rank_seed(rank, i))
        x = W.activations_bf16_fast(N, D, tensor_id=W.TID_X, device=str(dev), **kw)
        res = W.activations_bf16_fast(N, D, tensor_id=W.TID_RESIDUAL,
                                      device=str(dev), **kw)
        if i == 0 and rank == 0:
            x.copy_(fx.x.to(dev))
            res.copy_(fx.residual.to(dev))
        qw = torch.from_numpy(weight_codes(W, bits, O_, K, i)).to(dev)
        sw = torch.from_numpy(W.weight_scales(O_, K, i)).to(dev)
        sets.append((x, res, qw, sw))
    h = torch.empty(N, D, dtype=torch.bfloat16, device=dev)
    q = torch.empty(N, D // 2, dtype=torch.uint8, device=dev)
    sc = torch.empty(N, dtype=torch.float32, device=dev)
    out = torch.empty(N, O_, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream

    def step(i):
        x, res, qw, sw = sets[i % NSETS]
        rq.respin_boundary_forward(plan, x, res, h, q, sc, sptr)
        rq.w4a4_gemm(q, sc, qw, sw, out, sptr)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    if rq.respin_device_status() != 0:
        raise RuntimeError("a kernel reported a device-side failure in warm-up")

    sampler = ClockSampler(local_rank)
    sampler.start()
    sampler.wait_first()

    Ksteps = args.steps
    # per-kernel events on every EVERY-th step of the timed region (events
    # between two launches leave a gap of a few microseconds on the stream,
    # so they sample the kernels instead of sitting in every step)
    EVERY = 8
    sampled = list(range(0, Ksteps, EVERY))
    ev = {i: [torch.cuda.Event(enable_timing=True) for _ in range(3)] for i in sampled}
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    t_start.record(stream)
    for i in range(Ksteps):
        x, res, qw, sw = sets[i % NSETS]
        e = ev.get(i)
        if e: e[0].record(stream)
        rq.respin_boundary_forward(plan, x, res, h, q, sc, sptr)
        if e: e[1].record(stream)
        rq.w4a4_gemm(q, sc, qw, sw, out, sptr)
        if e: e[2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    if dist:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    b_ms = sum(e[0].elapsed_time(e[1]) for e in ev.values()) / len(ev)
    g_ms = sum(e[1].elapsed_time(e[2]) for e in ev.values()) / len(ev)
    clocks = sampler.summary(wall0, wall1)
    if rq.respin_device_status() != 0:
        raise RuntimeError("a kernel reported a device-side failure")

    # ---- supplementary: the same K-step block repeated, median per-step time
    # (the official figure above is the single timed region)
    blocks = []
    for rep_i in range(max(0, args.repeat)):
        b0e = torch.cuda.Event(enable_timing=True)
        b1e = torch.cuda.Event(enable_timing=True)
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        b0e.record(stream)
        for i in range(Ksteps):
            x, res, qw, sw = sets[i % NSETS]
            rq.respin_boundary_forward(plan, x, res, h, q, sc, sptr)
            rq.w4a4_gemm(q, sc, qw, sw, out, sptr)
        b1e.record(stream)
        torch.cuda.synchronize()
        blocks.append(b0e.elapsed_time(b1e) / Ksteps)
    blocks = max_over_ranks(blocks, dist, dev) if blocks else []

    # ---- supplementary: the same step with the boundary plan made from the
    # other form of the same fix (device time of its boundary launches)
    other = "factor" if form == "subspace" else "subspace"
    if other == "subspace":
        Qs, Rs = subspace_of(fx)
        oplan = rq.SubspacePlan(D, r, Qs.astype(np.float32), Rs.astype(np.float32), pflags)
    else:
        oplan = rq.Plan(D, r, fx.U.astype(np.float32), fx.V.astype(np.float32), pflags)
    Ko = max(3, min(Ksteps, 100))
    evo = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(Ko)]
    for i in range(3):
        x, res, qw, sw = sets[i % NSETS]
        rq.respin_boundary_forward(oplan, x, res, h, q, sc, sptr)
        rq.w4a4_gemm(q, sc, qw, sw, out, sptr)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(Ko):
        x, res, qw, sw = sets[i % NSETS]
        evo[i][0].record(stream)
        rq.respin_boundary_forward(oplan, x, res, h, q, sc, sptr)
        evo[i][1].record(stream)
        rq.w4a4_gemm(q, sc, qw, sw, out, sptr)
        evo[i][2].record(stream)
    torch.cuda.synchronize()
    ob_ms = sum(e[0].elapsed_time(e[1]) for e in evo) / Ko
    ost_ms = sum(e[0].elapsed_time(e[2]) for e in evo) / Ko
    oplan.destroy()
    if rq.respin_device_status() != 0:
        raise RuntimeError("a kernel reported a device-side failure")
    ob_ms, ost_ms = max_over_ranks([ob_ms, ost_ms], dist, dev)

    # ---- end to end through the public API with pinned host buffers. Three
    # streams and two device buffer sets, as a user would pipeline it: the
    # results of step i go back to the host (one copy engine) while the inputs
    # of step i+1 arrive (the other) and its kernels run; every step moves
    # all of its bytes (x and residual in, GEMM output and h' out).
    x_h = fx.x.pin_memory() if rank == 0 else sets[0][0].cpu().pin_memory()
    r_h = fx.residual.pin_memory() if rank == 0 else sets[0][1].cpu().pin_memory()
    out_h = torch.empty(N, O_, dtype=torch.bfloat16).pin_memory()
    h_h = torch.empty(N, D, dtype=torch.bfloat16).pin_memory()
    bufs = [dict(x=torch.empty_like(sets[0][0]), r=torch.empty_like(sets[0][1]), h=torch.empty_like(h),
                 q=torch.empty_like(q), sc=torch.empty_like(sc), out=torch.empty_like(out))
            for _ in range(2)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    Ke = max(3, min(Ksteps, 50))

    def e2e_step(i):
        k = i % 2
        b = bufs[k]
        _, _, qw, sw = sets[i % NSETS]
        s_in.wait_event(ev_cmp[k])        # the kernels that read this set's inputs are done
        with torch.cuda.stream(s_in):
            b["x"].copy_(x_h, non_blocking=True)
            b["r"].copy_(r_h, non_blocking=True)
        ev_in[k].record(s_in)
        s_cmp.wait_event(ev_in[k])
        s_cmp.wait_event(ev_out[k])       # this set's previous results are on the host
        rq.respin_boundary_forward(plan, b["x"], b["r"], b["h"], b["q"], b["sc"], s_cmp.cuda_stream)
        rq.w4a4_gemm(b["q"], b["sc"], qw, sw, b["out"], s_cmp.cuda_stream)
        ev_cmp[k].record(s_cmp)
        s_out.wait_event(ev_cmp[k])
        with torch.cuda.stream(s_out):
            out_h.copy_(b["out"], non_blocking=True)
            h_h.copy_(b["h"], non_blocking=True)
        ev_out[k].record(s_out)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(s_in)
    for i in range(Ke):
        e2e_step(i)
    e1.record(s_out)                      # after the last step's results reached the host
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e2e_ms = e0.elapsed_time(e1) / Ke
    if rq.respin_device_status() != 0:
        raise RuntimeError("a kernel reported a device-side failure")
    sampler.stop_evt.set()

    total_ms, e2e_ms, b_ms, g_ms = max_over_ranks([total_ms, e2e_ms, b_ms, g_ms],
                                                  dist, dev)
    ms_step = total_ms / Ksteps

    if rank == 0:
        hbm_gbs, bf16_tf, src = peaks()
        int8_tops = bf16_tf * INT8_OVER_BF16
        gemm_ops = 2.0 * N * K * O_
        gemm_tops = gemm_ops / (g_ms * 1e-3) / 1e12
        b_bytes = boundary_bytes(N, D, r, form)
        b_gbs = b_bytes / (b_ms * 1e-3) / 1e9
        bkern, bfile = boundary_kernel_of(form, N)
        line = {
            "metric": metric(bits),
            "value": job_tokens_per_s(world, N, ms_step),
            "unit": "tokens/s",
            "n_gpus": world, "steps": Ksteps, "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16+int%d" % bits, "data": "synthetic",
            "config": config_block(w, world, bits, form),
            "metric_components": {
                "boundary_tokens_per_s": job_tokens_per_s(world, N, b_ms),
                "gemm_tops": gemm_tops * world,
                "note": "the metric names two figures: tokens/s of the fused boundary kernel "
                        "and TOPS of the W4A4 GEMM; value is tokens/s of the whole step "
                        "(boundary + GEMM per batch of tokens)"},
            "boundary_tokens_per_s": job_tokens_per_s(world, N, b_ms),
            "boundary_us": b_ms * 1e3,
            "gemm_tops": gemm_tops * world,
            "gemm_us": g_ms * 1e3,
            "kernel_timing": "CUDA events around the boundary and GEMM launches of every %dth step "
                             "of the timed region (%d of %d steps)" % (EVERY, len(ev), Ksteps),
            "roofline": {
                "kernel": "w4a4_gemm_ta_kernel", "bound": "tensor",
                "achieved": gemm_tops, "peak": int8_tops, "unit": "TFLOP/s",
                "frac": gemm_tops / int8_tops,
                "traffic": traffic_for("w4a4_gemm_kernels.cuh", "w4a4_gemm_ta_kernel"),
                "peak_source": "%s bf16 burst %.1f TFLOP/s x %.0f (nominal "
                               "int8/bf16 dense ratio); integer ops counted "
                               "as 2 per multiply-add" % (src, bf16_tf,
                                                          INT8_OVER_BF16)},
            "roofline_boundary": {
                "kernel": bkern, "bound": "hbm",
                "achieved": b_gbs, "peak": hbm_gbs, "unit": "GB/s",
                "frac": b_gbs / hbm_gbs,
                "traffic": traffic_for(bfile, bkern),
                "algorithmic_bytes": b_bytes,
                "peak_source": "%s HBM copy bandwidth" % src},
            "other_boundary_form": {
                "boundary_plan": config_block(w, world, bits, other)["boundary_plan"],
                "kernel": boundary_kernel_of(other, N)[0],
                "boundary_us": ob_ms * 1e3,
                "boundary_frac_of_hbm": boundary_bytes(N, D, r, other) / (ob_ms * 1e-3) / 1e9 / hbm_gbs,
                "step_us": ost_ms * 1e3, "steps": Ko,
                "note": "supplementary: the same step with the plan built from the other form of "
                        "the same fix, timed after the timed region"},
            "steady": {"blocks": len(blocks), "steps_per_block": Ksteps,
                       "ms_per_step_median": (sorted(blocks)[len(blocks) // 2] if blocks else None),
                       "ms_per_step_min": (min(blocks) if blocks else None),
                       "note": "supplementary: the timed K-step block repeated after the timed "
                               "region; value above is the single timed region"},
            "e2e": {"value": job_tokens_per_s(world, N, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": 2 * N * D * 2,
                    "d2h_bytes_per_step": N * O_ * 2 + N * D * 2,
                    "pipelining": "pinned host buffers; copies in, kernels and copies out on "
                                  "three streams with two device buffer sets"},
            "gpu_launches": 2 * Ksteps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = step_cpu_baseline(fx, qw_np, sw_np, form, bits, w.N, 16)
        if world == 1 and not args.no_workloads:
            line["workloads"] = all_workloads(args, form, cpu=not args.no_cpu_baseline)
        print(json.dumps(line), flush=True)
    plan.destroy()
    if dist:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------- other workloads

def _events_ms(torch, fn, iters: int, stream) -> float:
    """Mean device time of fn() over iters launches (CUDA events on `stream`)."""
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(iters):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def _graph_ms(torch, fn, iters: int) -> float:
    """Mean device time per call of fn(i) captured `iters` times in one CUDA
    graph and replayed (no host launch overhead between the calls)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for i in range(3):
            fn(i)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        for i in range(iters):
            fn(i)
    graph.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    graph.replay()
    e1.record()
    torch.cuda.synchronize()
    del graph
    return e0.elapsed_time(e1) / iters


def _plan_for(rq, W, D, r, k, nu, seed=0, form="factor"):
    import numpy as np
    Q = W.orthonormal_basis(D, k, seed)
    th = W.plane_angles(k, nu)
    if form == "subspace":
        Qr, R = W.subspace_factors(Q, th, r)
        return rq.SubspacePlan(D, r, Qr.astype(np.float32), R.astype(np.float32))
    U, V = W.lowrank_factors(Q, th, r)
    return rq.Plan(D, r, U.astype(np.float32), V.astype(np.float32))


def _line(workload: str, args, extra: dict) -> dict:
    hbm_gbs, bf16_tf, src = peaks()
    line = {"metric": METRIC, "workload": workload, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "dtype": "bf16+int4", "data": "synthetic",
            "peaks": {"hbm_gbs": hbm_gbs, "int8_tops": bf16_tf * INT8_OVER_BF16, "source": src}}
    line.update(extra)
    return line


class _Env:
    """Device, stream and helpers shared by the workload configurations."""

    def __init__(self, args):
        import torch
        self.torch = torch
        self.dev = torch.device("cuda", 0)
        torch.cuda.set_device(self.dev)
        self.stream = torch.cuda.current_stream(self.dev)
        self.sptr = self.stream.cuda_stream
        self.iters = max(3, min(args.steps, 50))
        self.warmup = max(3, args.warmup)
        self.g = torch.Generator(device=self.dev)
        self.g.manual_seed(0)
        hbm, bf16_tf, _ = peaks()
        self.hbm_gbs = hbm
        self.int8_tops = bf16_tf * INT8_OVER_BF16

    def codes(self, rows, K):
        return self.torch.randint(0, 256, (rows, K // 2), generator=self.g, device=self.dev,
                                  dtype=self.torch.uint8)

    def wscales(self, rows):
        return self.torch.rand(rows, generator=self.g, device=self.dev) * 1e-3 + 1e-3

    def acts(self, N, D, w, seed, tid):
        import workloads as W
        return W.activations_bf16_fast(N, D, n_outlier=w.n_outlier, outlier_scale=w.outlier_scale,
                                       dist=w.dist, seed=seed, tensor_id=tid, device=str(self.dev))

    def outs(self, N, D, O_=None):
        t = self.torch
        h = t.empty(N, D, dtype=t.bfloat16, device=self.dev)
        q = t.empty(N, D // 2, dtype=t.uint8, device=self.dev)
        sc = t.empty(N, dtype=t.float32, device=self.dev)
        out = t.empty(N, O_, dtype=t.bfloat16, device=self.dev) if O_ else None
        return h, q, sc, out


def _cpu_codes(x, res, U, V):
    """Packed codes and scales of some rows, from the oracle (CPU GEMM inputs)."""
    import numpy as np
    from oracle import native
    _, _, c, s = native.boundary_reference(_bits(x), _bits(res) if res is not None else None,
                                           np.asarray(U, np.float32), np.asarray(V, np.float32), 7,
                                           want_h64=False)
    return native.pack(c), s


def wl_tiny(args, env, cpu: bool) -> dict:
    import rotation_post_quantization_b200 as rq
    import workloads as W
    w = W.WORKLOADS["tiny"]
    fx = W.workload_fixture("tiny")
    plan = _plan_for(rq, W, w.D, w.r, w.k, w.nu)
    x, res = fx.x.to(env.dev), fx.residual.to(env.dev)
    h, q, sc, _ = env.outs(w.N, w.D)
    # no explicit stream: the call goes to torch's current stream, which is
    # the capturing stream inside _graph_ms
    f = lambda i: rq.respin_boundary_forward(plan, x, res, h, q, sc)
    for i in range(env.warmup):
        f(i)
    us = _events_ms(env.torch, f, env.iters, env.stream) * 1e3
    gus = _graph_ms(env.torch, f, env.iters) * 1e3
    plan.destroy()
    b_bytes = boundary_bytes(w.N, w.D, w.r, "factor")
    out = {"config": {"D": w.D, "N": w.N, "r": w.r, "plan": "factor pair (D=256 is below the pair "
                                                             "kernel's sizes)"},
           "boundary_us": gus, "eager_boundary_us": us,
           "boundary_frac_of_hbm": b_bytes / env.hbm_gbs / 1e3 / gus,
           "note": "CUDA-graph replay (device time per call); inputs L2-resident"}
    if cpu:
        (b,), pc = _pinned(lambda: (oracle_boundary_tps(fx.x, fx.residual, (fx.U, fx.V), "factor"),))
        out["cpu_baseline"] = {"boundary_tokens_per_s": b, "cores": 1, "pinned_cpu": pc, "kind": "oracle",
                               "sample": "all 64 tokens, median of %d" % ORACLE_REPS}
    return out


def wl_decode(args, env, form: str, cpu: bool) -> dict:
    import numpy as np
    import rotation_post_quantization_b200 as rq
    import workloads as W
    w = W.WORKLOADS["decode"]
    plans = {"subspace": _plan_for(rq, W, w.D, w.r, w.k, w.nu, form="subspace"),
             "factor": _plan_for(rq, W, w.D, w.r, w.k, w.nu, form="factor")}
    NW = 16   # rotating weight sets: 16 x 8.4 MB > L2
    wsets = [(env.codes(w.O, w.D), env.wscales(w.O)) for _ in range(NW)]
    rows = []
    for N in w.extra["Ns"]:
        x, res = env.acts(N, w.D, w, 1, W.TID_X), env.acts(N, w.D, w, 2, W.TID_RESIDUAL)
        h, q, sc, out = env.outs(N, w.D, w.O)
        row = {"N": N}
        for name, plan in plans.items():
            fb = lambda i, plan=plan: rq.respin_boundary_forward(plan, x, res, h, q, sc)
            for i in range(env.warmup):
                fb(i)
            b_us = _graph_ms(env.torch, fb, env.iters) * 1e3
            row["boundary_us_" + name] = b_us
            row["boundary_frac_of_hbm_" + name] = boundary_bytes(N, w.D, w.r, name) / env.hbm_gbs / 1e3 / b_us
        fg = lambda i: rq.w4a4_gemm(q, sc, wsets[i % NW][0], wsets[i % NW][1], out)
        for i in range(env.warmup):
            fg(i)
        g_us = _graph_ms(env.torch, fg, env.iters) * 1e3
        g_bytes = w.O * w.D / 2 + N * w.D / 2 + N * w.O * 2 + 4 * (N + w.O)
        row.update({"gemm_us": g_us, "gemm_frac_of_hbm": g_bytes / env.hbm_gbs / 1e3 / g_us,
                    "gemm_tops": 2.0 * N * w.D * w.O / g_us / 1e6})
        rows.append(row)
    for p in plans.values():
        p.destroy()
    out = {"config": {"D": w.D, "r": w.r, "gemm": "%d -> %d" % (w.D, w.O),
                      "weights": "16 rotating sets (134 MB > L2)"},
           "rows": rows,
           "note": "CUDA-graph replay, device time per call; boundary for both plan forms; "
                   "fractions: algorithmic bytes / HBM bandwidth / time"}
    if cpu:
        fx = W.workload_fixture("decode", N=256)
        qw = W.int4_packed_random(w.O, w.D, 0, W.TID_WEIGHTS)
        sw = W.weight_scales(w.O, w.D, 0)
        Qs, Rs = subspace_of(fx)

        def run():
            res_ = []
            for N in w.extra["Ns"]:
                b = oracle_boundary_tps(fx.x[:N], fx.residual[:N], (Qs, Rs) if form == "subspace" else (fx.U, fx.V),
                                        form)
                ng = min(N, 16)
                qa, sa = _cpu_codes(fx.x[:ng], fx.residual[:ng], fx.U, fx.V)
                res_.append({"N": N, "boundary_tokens_per_s": b, "gemm_gops": oracle_gemm_gops(qa, sa, qw, sw)})
            return res_
        r_, pc = _pinned(run)
        out["cpu_baseline"] = {"rows": r_, "cores": 1, "pinned_cpu": pc, "kind": "oracle",
                               "sample": "boundary (%s form) on all N tokens, GEMM 4096 -> 4096 on min(N, 16) "
                                         "rows; median of %d" % (form, ORACLE_REPS)}
    return out


def wl_70b(args, env, cpu: bool) -> dict:
    import numpy as np
    import rotation_post_quantization_b200 as rq
    import workloads as W
    w = W.WORKLOADS["llama2_70b"]
    N, D = w.N, w.D
    sets = [(env.acts(N, D, w, 2 * i + 1, W.TID_X), env.acts(N, D, w, 2 * i + 2, W.TID_RESIDUAL)) for i in range(2)]
    h, q, sc, _ = env.outs(N, D)
    rows = []
    for r in w.extra["ranks"]:
        try:
            plan = _plan_for(rq, W, D, r, w.k, w.nu)
        except rq.RespinError as e:
            rows.append({"r": r, "unsupported": str(e)})
            continue
        fb = lambda i: rq.respin_boundary_forward(plan, *sets[i % 2], h, q, sc, env.sptr)
        for i in range(env.warmup):
            fb(i)
        b_us = _events_ms(env.torch, fb, env.iters, env.stream) * 1e3
        rows.append({"r": r, "boundary_us": b_us, "tokens_per_s": N / b_us * 1e6,
                     "frac_of_hbm": boundary_bytes(N, D, r, "factor") / env.hbm_gbs / 1e3 / b_us})
        plan.destroy()
    qw = env.codes(w.O, D)
    sw = env.wscales(w.O)
    out_t = env.torch.empty(N, w.O, dtype=env.torch.bfloat16, device=env.dev)
    fg = lambda i: rq.w4a4_gemm(q, sc, qw, sw, out_t, env.sptr)
    for i in range(env.warmup):
        fg(i)
    g_us = _events_ms(env.torch, fg, env.iters, env.stream) * 1e3
    tops = 2.0 * N * D * w.O / g_us / 1e6
    del sets, out_t
    out = {"config": {"D": D, "N": N, "gemm": "%d -> %d" % (D, w.O), "dist": w.dist,
                      "plan": "factor pair (the pair kernel serves D = 2048, 4096)"},
           "boundary_rank_sweep": rows, "gemm_us": g_us, "gemm_tops": tops,
           "gemm_frac_of_peak": tops / env.int8_tops}
    if cpu:
        fx_rows = 128

        def run():
            x = W.activations_bf16(fx_rows, D, n_outlier=w.n_outlier, outlier_scale=w.outlier_scale,
                                   dist=w.dist, tensor_id=W.TID_X)
            res = W.activations_bf16(fx_rows, D, n_outlier=w.n_outlier, outlier_scale=w.outlier_scale,
                                     dist=w.dist, tensor_id=W.TID_RESIDUAL)
            Q = W.orthonormal_basis(D, w.k, 0)
            sweep = []
            for r in w.extra["ranks"]:
                U, V = W.lowrank_factors(Q, W.plane_angles(w.k, w.nu), r)
                sweep.append({"r": r, "boundary_tokens_per_s": oracle_boundary_tps(x, res, (U, V), "factor")})
            U, V = W.lowrank_factors(Q, W.plane_angles(w.k, w.nu), w.r)
            qa, sa = _cpu_codes(x[:4], res[:4], U, V)
            qw_np = W.int4_packed_random(w.O, D, 0, W.TID_WEIGHTS)
            sw_np = W.weight_scales(w.O, D, 0)
            return sweep, oracle_gemm_gops(qa, sa, qw_np, sw_np)
        (sweep, gops), pc = _pinned(run)
        out["cpu_baseline"] = {"boundary_rank_sweep": sweep, "gemm_gops": gops, "cores": 1, "pinned_cpu": pc,
                               "kind": "oracle",
                               "sample": "boundary on %d tokens per rank, GEMM 8192 -> 28672 on 4 rows; "
                                         "median of %d" % (fx_rows, ORACLE_REPS)}
    return out


def wl_stack(args, env, form: str, cpu: bool) -> dict:
    import numpy as np
    import rotation_post_quantization_b200 as rq
    import workloads as W
    w = W.WORKLOADS["llama3_8b_stack"]
    torch = env.torch
    N, D, M, L = w.N, w.D, w.extra["mlp"], w.extra["layers"]
    plans = [_plan_for(rq, W, D, w.r, w.k, w.nu, seed=i, form=form) for i in range(2 * L)]
    wup = [(env.codes(M, D), env.wscales(M)) for _ in range(L)]
    wdn = [(env.codes(D, M), env.wscales(D)) for _ in range(L)]
    xatt = [env.acts(N, D, w, 100 + i, W.TID_X) for i in range(4)]
    res0 = env.acts(N, D, w, 99, W.TID_RESIDUAL)
    resid = [torch.empty(N, D, dtype=torch.bfloat16, device=env.dev) for _ in range(2)]
    _, q1, s1, _ = env.outs(N, D)
    u = torch.empty(N, M, dtype=torch.bfloat16, device=env.dev)
    q2 = torch.empty(N, M // 2, dtype=torch.uint8, device=env.dev)
    s2 = torch.empty(N, dtype=torch.float32, device=env.dev)
    xm = torch.empty(N, D, dtype=torch.bfloat16, device=env.dev)
    _, q3, s3, _ = env.outs(N, D)
    qonly = rq.Plan(M, 0)
    rowmax = torch.empty(N, M // 256, dtype=torch.float32, device=env.dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5 * L + 1)]
    sp = env.sptr

    # The up projection's GEMM also writes the per-token maxima of its output
    # per 256-channel tile, so the quant-only step before the down projection
    # is a pure streaming pass (no reduction of its own).
    def stack(record):
        cur = res0
        for l in range(L):
            h1 = resid[0]
            if record: ev[5 * l].record(env.stream)
            rq.respin_boundary_forward(plans[2 * l], xatt[l % 4], cur, h1, q1, s1, sp)
            if record: ev[5 * l + 1].record(env.stream)
            rq.w4a4_gemm_rowmax(q1, s1, wup[l][0], wup[l][1], u, rowmax, sp)
            if record: ev[5 * l + 2].record(env.stream)
            rq.respin_quantize_rowmax(u, rowmax, q2, s2, 0, sp)
            if record: ev[5 * l + 3].record(env.stream)
            rq.w4a4_gemm(q2, s2, wdn[l][0], wdn[l][1], xm, sp)
            if record: ev[5 * l + 4].record(env.stream)
            rq.respin_boundary_forward(plans[2 * l + 1], xm, h1, resid[1], q3, s3, sp)
            cur = resid[1]
        if record: ev[5 * L].record(env.stream)

    stack(False)
    torch.cuda.synchronize()
    reps = 3
    parts = np.zeros(5)
    total = 0.0
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    for _ in range(reps):   # the stack alone (no events between its kernels)
        t0.record(env.stream)
        stack(False)
        t1.record(env.stream)
        torch.cuda.synchronize()
        total += t0.elapsed_time(t1)
    # the quant-only step as a row-wise pass with its own reduction, for comparison
    for _ in range(3):
        rq.respin_boundary_forward(qonly, u, None, None, q2, s2, sp)
    qo_rowwise_us = _events_ms(torch, lambda i: rq.respin_boundary_forward(qonly, u, None, None, q2, s2, sp),
                               10, env.stream) * 1e3
    for _ in range(reps):   # per-part device times (events between the kernels)
        stack(True)
        torch.cuda.synchronize()
        for l in range(L):
            for j in range(5):
                parts[j] += ev[5 * l + j].elapsed_time(ev[5 * l + j + 1])
    if rq.respin_device_status() != 0:
        raise RuntimeError("a kernel reported a device-side failure")
    for p in plans:
        p.destroy()
    qonly.destroy()
    ms = total / reps
    parts = parts / reps / L * 1e3
    ops = L * 2.0 * N * D * M * 2
    bb = boundary_bytes(N, D, w.r, form)
    out = {"config": {"D": D, "N": N, "layers": L, "mlp": M, "r": w.r,
                      "plan": "stored subspace form" if form == "subspace" else "factor pair",
                      "chain": "attn boundary, GEMM D->mlp (with per-token tile maxima of its output), "
                               "quant-only mlp from those maxima, GEMM mlp->D, mlp boundary "
                               "(nonlinearity omitted)"},
           "tokens_per_s": N / (ms * 1e-3), "ms_per_stack": ms,
           "per_layer_us": {"attn_boundary": parts[0], "gemm_up": parts[1], "quant_only": parts[2],
                            "gemm_down": parts[3], "mlp_boundary": parts[4]},
           "quant_only_rowwise_us": qo_rowwise_us,
           "note": "ms_per_stack: the stack with no events between its kernels; per_layer_us: "
                   "the same stack with events around every kernel; quant_only_rowwise_us: the "
                   "quant-only step as a row-wise pass with its own reduction, for comparison",
           "gemm_tops": ops / ((parts[1] + parts[3]) * L * 1e-6) / 1e12,
           "boundary_frac_of_hbm": bb / env.hbm_gbs / 1e3 / ((parts[0] + parts[4]) / 2),
           "quant_only_frac_of_hbm": (N * (2 * M + M / 2 + 4)) / env.hbm_gbs / 1e3 / parts[2]}
    del wup, wdn
    if cpu:
        nb, ng = 256, 8

        def run():
            fx = W.workload_fixture("llama3_8b_stack", N=nb)
            Qs, Rs = subspace_of(fx)
            b = oracle_boundary_tps(fx.x, fx.residual, (Qs, Rs) if form == "subspace" else (fx.U, fx.V), form)
            u_rows = W.activations_bf16(nb, M, n_outlier=w.n_outlier, outlier_scale=w.outlier_scale,
                                        tensor_id=W.TID_X, seed=7)
            qo = oracle_boundary_tps(u_rows, None, (np.zeros((M, 0)), np.zeros((M, 0))), "factor")
            qa, sa = _cpu_codes(fx.x[:ng], fx.residual[:ng], fx.U, fx.V)
            g_up = oracle_gemm_gops(qa, sa, W.int4_packed_random(M, D, 0, W.TID_WEIGHTS), W.weight_scales(M, D, 0))
            qa2, sa2 = _cpu_codes(u_rows[:ng], None, np.zeros((M, 0)), np.zeros((M, 0)))
            g_dn = oracle_gemm_gops(qa2, sa2, W.int4_packed_random(D, M, 0, W.TID_WEIGHTS), W.weight_scales(D, M, 0))
            return b, qo, g_up, g_dn
        (b, qo, g_up, g_dn), pc = _pinned(run)
        per_tok_layer = 2.0 / b + 1.0 / qo + 2.0 * D * M / (g_up * 1e9) + 2.0 * M * D / (g_dn * 1e9)
        out["cpu_baseline"] = {"tokens_per_s": 1.0 / (L * per_tok_layer), "boundary_tokens_per_s": b,
                               "quant_only_tokens_per_s": qo, "gemm_up_gops": g_up, "gemm_down_gops": g_dn,
                               "cores": 1, "pinned_cpu": pc, "kind": "oracle",
                               "sample": "one layer's parts on %d tokens (boundaries, quant-only) and %d rows "
                                         "(GEMMs), median of %d; tokens/s through %d layers"
                                         % (nb, ng, ORACLE_REPS, L)}
    return out


def all_workloads(args, form: str, cpu: bool) -> dict:
    """Configurations 1, 3, 4, 5 (compact), appended to the headline line."""
    env = _Env(args)
    res = {}
    for name, fn in (("tiny", lambda: wl_tiny(args, env, cpu)),
                     ("decode", lambda: wl_decode(args, env, form, cpu)),
                     ("llama3_8b_stack", lambda: wl_stack(args, env, form, cpu)),
                     ("llama2_70b", lambda: wl_70b(args, env, cpu))):
        try:
            res[name] = fn()
        except Exception as e:   # one configuration failing must not hide the others
            res[name] = {"error": repr(e)}
        env.torch.cuda.empty_cache()
    return res


def run_workload(args):
    """Workload configurations besides the headline step, one JSON line each."""
    env = _Env(args)
    name = args.workload
    form = args.boundary_form
    cpu = not args.no_cpu_baseline
    fn = {"tiny": lambda: wl_tiny(args, env, cpu), "decode": lambda: wl_decode(args, env, form, cpu),
          "llama2_70b": lambda: wl_70b(args, env, cpu),
          "llama3_8b_stack": lambda: wl_stack(args, env, form, cpu)}[name]
    line = _line(name, args, fn())
    import rotation_post_quantization_b200 as rq
    if rq.respin_device_status() != 0:
        raise RuntimeError("a kernel reported a device-side failure")
    print(json.dumps(line), flush=True)


def run_profile_launch(args):
    """Warm-up launches, then exactly one more launch of the chosen kernel."""
    import numpy as np
    import torch
    import rotation_post_quantization_b200 as rq
    import workloads as W

    name = "llama2_70b" if args.workload == "llama2_70b" else WORKLOAD
    w = W.WORKLOADS[name]
    N = args.tokens or w.N
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if name == "llama2_70b":
        plan = _plan_for(rq, W, w.D, args.rank or w.r, w.k, w.nu)
    else:
        fx = W.workload_fixture(WORKLOAD, N=16)
        if args.boundary_form == "subspace":
            Qs, Rs = subspace_of(fx)
            plan = rq.SubspacePlan(w.D, w.r, Qs.astype(np.float32), Rs.astype(np.float32))
        else:
            plan = rq.Plan(w.D, w.r, fx.U.astype(np.float32), fx.V.astype(np.float32))
    kw = dict(n_outlier=w.n_outlier, outlier_scale=w.outlier_scale, dist=w.dist)
    x = W.activations_bf16_fast(N, w.D, tensor_id=W.TID_X, device="cuda", **kw)
    res = W.activations_bf16_fast(N, w.D, tensor_id=W.TID_RESIDUAL, device="cuda", **kw)
    h = torch.empty(N, w.D, dtype=torch.bfloat16, device=dev)
    q = torch.empty(N, w.D // 2, dtype=torch.uint8, device=dev)
    sc = torch.empty(N, dtype=torch.float32, device=dev)
    qw = torch.from_numpy(W.int4_packed_random(w.O, w.D, 0, W.TID_WEIGHTS)).to(dev)
    sw = torch.from_numpy(W.weight_scales(w.O, w.D, 0)).to(dev)
    out = torch.empty(N, w.O, dtype=torch.bfloat16, device=dev)
    rq.respin_boundary_forward(plan, x, res, h, q, sc)
    for _ in range(args.warmup + 1):
        if args.profile_launch == "boundary":
            rq.respin_boundary_forward(plan, x, res, h, q, sc)
        else:
            rq.w4a4_gemm(q, sc, qw, sw, out)
    torch.cuda.synchronize()
    assert rq.respin_device_status() == 0
    plan.destroy()
    print("profile launch done: %s, %d tokens" % (args.profile_launch, N))


def main():
    args = parse_args()
    if args.profile_launch:
        run_profile_launch(args)
        return
    rank, world, local_rank = rank_env()
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.workload not in STEP_BITS:
        run_workload(args)
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
