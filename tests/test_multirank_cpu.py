"""Multi-rank host logic of bench.py, on CPU with the gloo backend.

The forward pass shards by (b, h): every head is independent, K mean and V
scales included, so N GPUs run N independent batches with no collective on
the data path (weak scaling).  What is multi-rank is the measurement: every
rank times its own steps, the job's time is the maximum over ranks, and the
job's throughput is the work of all ranks over that time.  These tests run
that logic as two gloo ranks, plus the reference arm's rank handling.
"""

import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from quantized_attention_quant_b200.workloads import WORKLOADS, make_qkv  # noqa: E402


def _rank_main(rank, world, port, result_q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # rank-dependent timings: rank 1 is the slow one for the step, rank 0 for e2e
        mine = [1.0 + rank, 0.5 + 0.25 * rank, 9.0 - rank]
        got = bench.max_over_ranks(mine, world, torch.device("cpu"))
        w = bench.rank_workload(WORKLOADS["tiny"], rank)
        q, _, _ = make_qkv(w, heads=[(0, 0)])
        # each rank's first input value, gathered to compare across ranks
        first = torch.tensor([float(q.flatten()[0])], dtype=torch.float64)
        allf = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(allf, first)
        result_q.put((rank, got, w.seed, [float(t) for t in allf]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_take_the_max_and_draw_distinct_batches():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, got, seed, firsts = q.get(timeout=120)
        res[rank] = (got, seed, firsts)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the same maxima
    assert res[0][0] == res[1][0] == [2.0, 0.75, 9.0]
    # weak scaling: distinct seeds, distinct inputs
    assert res[0][1] != res[1][1]
    assert res[0][2][0] != res[0][2][1]


def test_job_throughput_counts_all_ranks_over_the_slowest():
    w = WORKLOADS["llm"]
    one = bench.job_throughput(w.ops, 1, 0.3)
    assert bench.job_throughput(w.ops, 4, 0.3) == pytest.approx(4 * one)
    assert one == pytest.approx(w.ops / 0.3e-3 / 1e12)
    cfg = bench.config_of(w, 8)
    assert cfg["global_batch_heads"] == 8 * w.B * w.H and cfg["parallelism"].startswith("dp8")


def _run_reference(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "tiny", "--steps", "1", "--warmup", "3"],
                          capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_rank0_prints_one_line_other_ranks_exit_quietly():
    r0 = _run_reference({"RANK": "0", "WORLD_SIZE": "2", "LOCAL_RANK": "0"})
    assert r0.returncode == 0, r0.stderr[-2000:]
    lines = [ln for ln in r0.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["unit"] == "TOPS" and out["value"] > 0
    assert out["config"] == bench.config_of(WORKLOADS["tiny"], 2)
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["cpu_baseline"]["kind"] == "oracle"
    r1 = _run_reference({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r1.returncode == 0 and r1.stdout.strip() == ""
