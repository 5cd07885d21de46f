"""Multi-rank host logic on CPU with the gloo backend (world size 2): per-rank
seeding, max-over-ranks timing, whole-job aggregation, and the reference arm
under torchrun (rank 0 prints one line, the other rank exits without work)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank measures different times; the job's time is the slowest rank's
        times = [10.0 + rank, 5.0 * (world - rank), 1.0]
        got = bench.reduce_max(times)
        from online_softmax_12_b200 import inputs

        sh = inputs.SMALL_FWD["bf16_causal_gqa_h8_kv2_n1100_d128"]
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(inputs.SEED_BASE + sh.seed_index, rank))
        q = inputs.make_fwd_inputs(sh, seed=bench.rank_seed(inputs.SEED_BASE + sh.seed_index, rank))["q"]
        sums = [None] * world
        dist.all_gather_object(sums, float(q.float().sum()))
        out_q.put((rank, got, seeds, sums))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_distinct_rank_inputs():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, seeds, sums in res:
        assert got == [11.0, 10.0, 1.0]
        assert len(set(seeds)) == world          # independent problem instances
        assert sums[0] != sums[1]


def test_aggregate_is_whole_job_throughput():
    tflops, gbs = bench.aggregate(world=4, steps=10, flops_per_step=2e12, bytes_per_step=1e9,
                                  prefill_ms_max=20.0, decode_ms_max=2.0)
    assert tflops == pytest.approx(4 * 10 * 2e12 / 0.02 / 1e12)
    assert gbs == pytest.approx(4 * 10 * 1e9 / 0.002 / 1e9)


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3", "--small"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "TFLOP/s" and rec["value"] > 0
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["cpu_baseline"]["kind"] == "oracle"
