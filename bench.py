#!/usr/bin/env python
"""Benchmark of the ReSpinQuant block-boundary hot path on B200.

One step = the whole path on one batch of tokens: the fused boundary kernel
(rank-r basis fix + per-token INT4 quantization, ReSpinQuant explainers zh
§2.2 and §3-§4) followed by the tcgen05 W4A4 GEMM that consumes its codes.
Workload: Llama-2-7B-shaped, D = 4096, 2048 tokens per GPU, r = 32 (rank-64
skew deviation, norm 0.1, 8 outlier channels x50), GEMM 4096 -> 11008 with
INT4 weights uniform in [-8, 7]. Synthetic, seeded inputs. --workload
llama2_7b_w3a3 runs the same step with 3-bit activation and weight codes
(W3A3); the other --workload names print the remaining configurations.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

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
    p.add_argument("--profile-launch", choices=["boundary", "gemm"],
                   help="profiling aid: warm up, then launch one kernel once "
                        "(for ncu captures); prints no bench line")
    p.add_argument("--tokens", type=int, default=None,
                   help="tokens for --profile-launch (default 2048)")
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

def oracle_sample_rate(fx, qw, sw, n_boundary: int, n_gemm: int, bits: int = 4):
    """Time the C++ oracle (as it stands: plain single-threaded loops) on a
    bounded sample; tokens/s of the whole path per token =
    1 / (t_boundary/token + t_gemm/token)."""
    import numpy as np
    import torch

    from oracle import native
    native.lib()   # built before the clock starts
    xb = fx.x[:n_boundary].view(torch.int16).numpy().view(np.uint16)
    rb = fx.residual[:n_boundary].view(torch.int16).numpy().view(np.uint16)
    U32, V32 = fx.U.astype(np.float32), fx.V.astype(np.float32)
    t0 = time.perf_counter()
    _, _, codes, scale = native.boundary_reference(xb, rb, U32, V32, 7 if bits == 4 else 3, want_h64=False)
    t1 = time.perf_counter()
    qa = native.pack(codes[:n_gemm])
    native.w4a4_gemm(qa, scale[:n_gemm], qw, sw)
    t2 = time.perf_counter()
    per_tok = (t1 - t0) / n_boundary + (t2 - t1) / n_gemm
    return 1.0 / per_tok, (t2 - t0)


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


def cpu_baseline_block(fx, qw, sw, bits: int = 4):
    rate, secs = oracle_sample_rate(fx, qw, sw, 2048, 400, bits)
    return {"value": rate, "unit": "tokens/s", "cores": 1, "kind": "oracle", "cpu": host_cpu(),
            "sample": "C++ oracle (plain loops, -O2, one thread): boundary (fp64 fix + "
                      "binary32 INT%d quantizer) on all 2048 tokens, W%dA%d GEMM (exact "
                      "int64 + binary32 epilogue) on 400 of the 2048 rows x 11008 "
                      "channels; per-token times summed; %.1f s of CPU work"
                      % (bits, bits, bits, secs)}


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
    """The reference arm: the CPU oracle, timed on the host cores."""
    if rank != 0:
        return
    bits = STEP_BITS.get(args.workload, 4)
    w, fx, qw, sw = workload_inputs(None, bits)
    nb, ng = 256, 16
    for _ in range(max(0, args.warmup)):
        oracle_sample_rate(fx, qw, sw, nb, ng, bits)
    t = 0.0
    rates = []
    for _ in range(args.steps):
        r, s = oracle_sample_rate(fx, qw, sw, nb, ng, bits)
        rates.append(r)
        t += s
    # per step: the full 2048-token batch at the sampled per-token cost
    per_tok = sum(1.0 / r for r in rates) / len(rates)
    value = 1.0 / per_tok
    line = {
        "impl": "reference", "metric": metric(bits), "value": value,
        "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": per_tok * w.N * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64+f32+int64", "data": "synthetic",
        "config": config_block(w, args.gpus, bits),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1,
                         "kind": "oracle", "cpu": host_cpu(),
                         "sample": "each step: C++ oracle, boundary on 256 tokens "
                                   "+ GEMM on 16 rows, 1 thread; "
                                   "%.1f s total" % t},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_block(w, n_gpus, bits: int = 4):
    return {"workload": "Llama-2-7B-shaped boundary + W%dA%d GEMM: D=4096, "
                        "2048 tokens/GPU, r=32, GEMM 4096->11008" % (bits, bits),
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

def run_ours(args, rank: int, world: int, local_rank: int):
    import numpy as np
    import torch
    import rotation_post_quantization_b200 as rq
    import workloads as W

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = init_dist("nccl", dev) if world > 1 else None

    bits = STEP_BITS[args.workload]
    w, fx, qw_np, sw_np = workload_inputs("cuda", bits)
    D, N, r, O_ = w.D, w.N, w.r, w.O
    K = D
    plan = rq.Plan(D, r, fx.U.astype(np.float32), fx.V.astype(np.float32),
                   rq.RESPIN_ACT_INT3 if bits == 3 else 0)

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
    time.sleep(0.05)

    Ksteps = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
          for _ in range(Ksteps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    t_start.record(stream)
    for i in range(Ksteps):
        x, res, qw, sw = sets[i % NSETS]
        ev[i][0].record(stream)
        rq.respin_boundary_forward(plan, x, res, h, q, sc, sptr)
        ev[i][1].record(stream)
        rq.w4a4_gemm(q, sc, qw, sw, out, sptr)
        ev[i][2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    if dist:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    b_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / Ksteps
    g_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / Ksteps
    clocks = sampler.summary(wall0, wall1)
    if rq.respin_device_status() != 0:
        raise RuntimeError("a kernel reported a device-side failure")

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
        b_bytes = N * (6.5 * D + 4) + 2 * D * 32 * 2
        b_gbs = b_bytes / (b_ms * 1e-3) / 1e9
        line = {
            "metric": metric(bits),
            "value": job_tokens_per_s(world, N, ms_step),
            "unit": "tokens/s",
            "n_gpus": world, "steps": Ksteps, "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16+int%d" % bits, "data": "synthetic",
            "config": config_block(w, world, bits),
            "boundary_tokens_per_s": job_tokens_per_s(world, N, b_ms),
            "boundary_us": b_ms * 1e3,
            "gemm_tops": gemm_tops * world,
            "gemm_us": g_ms * 1e3,
            "roofline": {
                "kernel": "w4a4_gemm_kernel", "bound": "tensor",
                "achieved": gemm_tops, "peak": int8_tops, "unit": "TFLOP/s",
                "frac": gemm_tops / int8_tops,
                "traffic": traffic_for("w4a4_gemm_kernels.cuh", "w4a4_gemm_kernel"),
                "peak_source": "%s bf16 burst %.1f TFLOP/s x %.0f (nominal "
                               "int8/bf16 dense ratio); integer ops counted "
                               "as 2 per multiply-add" % (src, bf16_tf,
                                                          INT8_OVER_BF16)},
            "roofline_boundary": {
                "kernel": "boundary_rowtile_kernel", "bound": "hbm",
                "achieved": b_gbs, "peak": hbm_gbs, "unit": "GB/s",
                "frac": b_gbs / hbm_gbs,
                "traffic": traffic_for("boundary_rowtile.cuh",
                                       "boundary_rowtile_kernel"),
                "peak_source": "%s HBM copy bandwidth" % src},
            "e2e": {"value": job_tokens_per_s(world, N, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": 2 * N * D * 2,
                    "d2h_bytes_per_step": N * O_ * 2 + N * D * 2,
                    "pipelining": "pinned host buffers; copies in, kernels and copies out on "
                                  "three streams with two device buffer sets"},
            "gpu_launches": 2 * Ksteps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_block(fx, qw_np, sw_np, bits)
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


def _plan_for(rq, W, D, r, k, nu, seed=0):
    import numpy as np
    Q = W.orthonormal_basis(D, k, seed)
    U, V = W.lowrank_factors(Q, W.plane_angles(k, nu), r)
    return rq.Plan(D, r, U.astype(np.float32), V.astype(np.float32))


def _line(workload: str, args, extra: dict) -> dict:
    hbm_gbs, bf16_tf, src = peaks()
    line = {"metric": METRIC, "workload": workload, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "dtype": "bf16+int4", "data": "synthetic",
            "peaks": {"hbm_gbs": hbm_gbs, "int8_tops": bf16_tf * INT8_OVER_BF16, "source": src}}
    line.update(extra)
    return line


def run_workload(args):
    """Workload configurations besides the headline step, one JSON line each."""
    import numpy as np
    import torch
    import rotation_post_quantization_b200 as rq
    import workloads as W

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream
    hbm_gbs, bf16_tf, _ = peaks()
    int8_tops = bf16_tf * INT8_OVER_BF16
    iters = max(3, args.steps)
    g = torch.Generator(device=dev)
    g.manual_seed(0)

    def rand_codes(rows, K):
        return torch.randint(0, 256, (rows, K // 2), generator=g, device=dev, dtype=torch.uint8)

    def acts(N, D, w, seed):
        return W.activations_bf16_fast(N, D, n_outlier=w.n_outlier, outlier_scale=w.outlier_scale,
                                       dist=w.dist, seed=seed, device=str(dev))

    name = args.workload
    w = W.WORKLOADS[name]
    if name == "tiny":
        plan = _plan_for(rq, W, w.D, w.r, w.k, w.nu)
        fx = W.workload_fixture(name)
        x, res = fx.x.to(dev), fx.residual.to(dev)
        h = torch.empty_like(x)
        q = torch.empty(w.N, w.D // 2, dtype=torch.uint8, device=dev)
        sc = torch.empty(w.N, dtype=torch.float32, device=dev)
        f = lambda i: rq.respin_boundary_forward(plan, x, res, h, q, sc, sptr)
        for i in range(args.warmup):
            f(i)
        us = _events_ms(torch, f, iters, stream) * 1e3
        line = _line(name, args, {"config": {"D": w.D, "N": w.N, "r": w.r},
                                  "boundary_us": us, "unit": "us", "value": us,
                                  "higher_is_better": False,
                                  "note": "latency of one boundary call (inputs L2-resident)"})
    elif name == "decode":
        plan = _plan_for(rq, W, w.D, w.r, w.k, w.nu)
        NW = 16   # rotating weight sets: 16 x 8.4 MB > L2
        wsets = [(rand_codes(w.O, w.D), torch.rand(w.O, generator=g, device=dev) * 1e-3 + 1e-3)
                 for _ in range(NW)]
        rows = []
        for N in w.extra["Ns"]:
            x, res = acts(N, w.D, w, 1), acts(N, w.D, w, 2)
            h = torch.empty_like(x)
            q = torch.empty(N, w.D // 2, dtype=torch.uint8, device=dev)
            sc = torch.empty(N, dtype=torch.float32, device=dev)
            out = torch.empty(N, w.O, dtype=torch.bfloat16, device=dev)
            # the current stream: the graph's capture stream inside _graph_ms
            fb = lambda i: rq.respin_boundary_forward(plan, x, res, h, q, sc)
            fg = lambda i: rq.w4a4_gemm(q, sc, wsets[i % NW][0], wsets[i % NW][1], out)
            for i in range(args.warmup):
                fb(i)
                fg(i)
            eb_us = _events_ms(torch, fb, iters, stream) * 1e3
            eg_us = _events_ms(torch, fg, iters, stream) * 1e3
            b_us = _graph_ms(torch, fb, iters) * 1e3
            g_us = _graph_ms(torch, fg, iters) * 1e3
            b_bytes = N * (6.5 * w.D + 4) + 2 * w.D * w.r * 2
            g_bytes = w.O * w.D / 2 + N * w.D / 2 + N * w.O * 2 + 4 * (N + w.O)
            rows.append({"N": N, "boundary_us": b_us, "gemm_us": g_us,
                         "eager_boundary_us": eb_us, "eager_gemm_us": eg_us,
                         "boundary_frac_of_hbm": b_bytes / hbm_gbs / 1e3 / b_us,
                         "gemm_frac_of_hbm": g_bytes / hbm_gbs / 1e3 / g_us,
                         "gemm_tops": 2.0 * N * w.D * w.O / g_us / 1e6})
        line = _line(name, args, {"config": {"D": w.D, "r": w.r, "gemm": "%d -> %d" % (w.D, w.O),
                                             "weights": "16 rotating sets (134 MB > L2)"},
                                  "rows": rows, "unit": "us", "higher_is_better": False,
                                  "note": "times: CUDA-graph replay (device time per call); eager_*: "
                                          "back-to-back calls from Python (host-bound at these sizes). "
                                          "fractions: algorithmic bytes / HBM bandwidth / graph time"})
    elif name == "llama2_70b":
        N, D = w.N, w.D
        sets = [(acts(N, D, w, 2 * i + 1), acts(N, D, w, 2 * i + 2)) for i in range(2)]
        h = torch.empty(N, D, dtype=torch.bfloat16, device=dev)
        q = torch.empty(N, D // 2, dtype=torch.uint8, device=dev)
        sc = torch.empty(N, dtype=torch.float32, device=dev)
        rows = []
        for r in w.extra["ranks"]:
            try:
                plan = _plan_for(rq, W, D, r, w.k, w.nu)
            except rq.RespinError as e:
                rows.append({"r": r, "unsupported": str(e)})
                continue
            fb = lambda i: rq.respin_boundary_forward(plan, *sets[i % 2], h, q, sc, sptr)
            for i in range(args.warmup):
                fb(i)
            b_us = _events_ms(torch, fb, iters, stream) * 1e3
            b_bytes = N * (6.5 * D + 4) + 2 * D * r * 2
            rows.append({"r": r, "boundary_us": b_us, "tokens_per_s": N / b_us * 1e6,
                         "frac_of_hbm": b_bytes / hbm_gbs / 1e3 / b_us})
            plan.destroy()
        qw = rand_codes(w.O, D)
        sw = torch.rand(w.O, generator=g, device=dev) * 1e-3 + 1e-3
        out = torch.empty(N, w.O, dtype=torch.bfloat16, device=dev)
        fg = lambda i: rq.w4a4_gemm(q, sc, qw, sw, out, sptr)
        for i in range(args.warmup):
            fg(i)
        g_us = _events_ms(torch, fg, iters, stream) * 1e3
        tops = 2.0 * N * D * w.O / g_us / 1e6
        line = _line(name, args, {"config": {"D": D, "N": N, "gemm": "%d -> %d" % (D, w.O),
                                             "dist": w.dist},
                                  "boundary_rank_sweep": rows, "gemm_us": g_us, "gemm_tops": tops,
                                  "gemm_frac_of_peak": tops / int8_tops,
                                  "unit": "tokens/s", "higher_is_better": True})
    else:   # llama3_8b_stack
        N, D, M, L = w.N, w.D, w.extra["mlp"], w.extra["layers"]
        plans = [_plan_for(rq, W, D, w.r, w.k, w.nu, seed=i) for i in range(2 * L)]
        wup = [(rand_codes(M, D), torch.rand(M, generator=g, device=dev) * 1e-3 + 1e-3) for _ in range(L)]
        wdn = [(rand_codes(D, M), torch.rand(D, generator=g, device=dev) * 1e-3 + 1e-3) for _ in range(L)]
        xatt = [acts(N, D, w, 100 + i) for i in range(4)]
        res0 = acts(N, D, w, 99)
        resid = [torch.empty(N, D, dtype=torch.bfloat16, device=dev) for _ in range(2)]
        q1 = torch.empty(N, D // 2, dtype=torch.uint8, device=dev)
        s1 = torch.empty(N, dtype=torch.float32, device=dev)
        u = torch.empty(N, M, dtype=torch.bfloat16, device=dev)
        q2 = torch.empty(N, M // 2, dtype=torch.uint8, device=dev)
        s2 = torch.empty(N, dtype=torch.float32, device=dev)
        xm = torch.empty(N, D, dtype=torch.bfloat16, device=dev)
        q3 = torch.empty(N, D // 2, dtype=torch.uint8, device=dev)
        s3 = torch.empty(N, dtype=torch.float32, device=dev)
        qonly = rq.Plan(M, 0)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(5 * L + 1)]

        def stack(record):
            # h1 -> resid[0], h2 -> resid[1]; the next layer reads resid[1]
            cur = res0
            for l in range(L):
                h1 = resid[0]
                if record: ev[5 * l].record(stream)
                rq.respin_boundary_forward(plans[2 * l], xatt[l % 4], cur, h1, q1, s1, sptr)
                if record: ev[5 * l + 1].record(stream)
                rq.w4a4_gemm(q1, s1, wup[l][0], wup[l][1], u, sptr)
                if record: ev[5 * l + 2].record(stream)
                rq.respin_boundary_forward(qonly, u, None, None, q2, s2, sptr)
                if record: ev[5 * l + 3].record(stream)
                rq.w4a4_gemm(q2, s2, wdn[l][0], wdn[l][1], xm, sptr)
                if record: ev[5 * l + 4].record(stream)
                rq.respin_boundary_forward(plans[2 * l + 1], xm, h1, resid[1], q3, s3, sptr)
                cur = resid[1]
            if record: ev[5 * L].record(stream)

        for _ in range(max(1, args.warmup // 5)):
            stack(False)
        torch.cuda.synchronize()
        reps = max(1, min(args.steps, 5))
        parts = np.zeros(5)
        total = 0.0
        for _ in range(reps):
            stack(True)
            torch.cuda.synchronize()
            total += ev[0].elapsed_time(ev[5 * L])
            for l in range(L):
                for j in range(5):
                    parts[j] += ev[5 * l + j].elapsed_time(ev[5 * l + j + 1])
        ms = total / reps
        parts = parts / reps / L * 1e3
        ops = L * 2.0 * N * D * M * 2
        line = _line(name, args, {"config": {"D": D, "N": N, "layers": L, "mlp": M, "r": w.r,
                                             "chain": "attn boundary, GEMM D->mlp, quant-only mlp, "
                                                      "GEMM mlp->D, mlp boundary (nonlinearity omitted)"},
                                  "value": N / (ms * 1e-3), "unit": "tokens/s", "higher_is_better": True,
                                  "ms_per_stack": ms,
                                  "per_layer_us": {"attn_boundary": parts[0], "gemm_up": parts[1],
                                                   "quant_only": parts[2], "gemm_down": parts[3],
                                                   "mlp_boundary": parts[4]},
                                  "gemm_tops": ops / ((parts[1] + parts[3]) * L * 1e-6) / 1e12,
                                  "boundary_tokens_per_s": N / ((parts[0] + parts[4]) / 2 * 1e-6)})
    if rq.respin_device_status() != 0:
        raise RuntimeError("a kernel reported a device-side failure")
    print(json.dumps(line), flush=True)


def run_profile_launch(args):
    """Warm-up launches, then exactly one more launch of the chosen kernel."""
    import numpy as np
    import torch
    import rotation_post_quantization_b200 as rq
    import workloads as W

    w = W.WORKLOADS[WORKLOAD]
    N = args.tokens or w.N
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    fx = W.workload_fixture(WORKLOAD, N=16)
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
