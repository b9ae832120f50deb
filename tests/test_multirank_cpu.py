"""Multi-rank host logic of bench.py on CPU: world size 2 over gloo.

The timed path shards the batch across ranks with no data-path collective
(weak scaling); the only collectives are the barriers around the timed region
and the max-over-ranks reduction of the timings, which these tests run with
two gloo ranks. The reference arm runs under torchrun on rank 0 alone.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    r, w, lr = bench.rank_env()
    assert (r, w, lr) == (rank, world, rank)
    dist = bench.init_dist("gloo", timeout_s=60)
    try:
        dist.barrier()
        # rank-dependent timings: total, e2e, boundary, gemm (ms)
        mine = [1.0 + rank, 5.0 - rank, 0.25 * (rank + 1), 0.75]
        got = bench.max_over_ranks(mine, dist)
        dist.barrier()
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as fh:
            json.dump(got, fh)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks(tmp_path):
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = [json.load(open(tmp_path / ("rank%d.json" % r))) for r in range(world)]
    assert got[0] == got[1] == [2.0, 5.0, 0.5, 0.75]


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks([3.0, 1.0], None) == [3.0, 1.0]


def test_job_throughput_is_weak_scaling():
    # 2048 tokens per rank per step, slowest rank 0.1 ms per step
    assert bench.job_tokens_per_s(1, 2048, 0.1) == pytest.approx(2.048e7)
    assert bench.job_tokens_per_s(8, 2048, 0.1) == pytest.approx(8 * 2.048e7)


def test_ranks_hold_different_inputs():
    seeds = {bench.rank_seed(r, i) for r in range(8) for i in range(bench.NSETS)}
    assert len(seeds) == 8 * bench.NSETS
    assert bench.rank_seed(0, 0) == 0


@pytest.mark.parametrize("workload,bits", [("llama2_7b", 4), ("llama2_7b_w3a3", 3)])
def test_reference_arm_under_torchrun_two_ranks(workload, bits):
    port = free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--workload", workload]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, res.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
    assert line["config"]["act_bits"] == bits and ("INT%d" % bits) in line["metric"]
