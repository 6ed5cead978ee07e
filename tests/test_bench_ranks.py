"""The multi-rank host logic of bench.py, on CPU with two gloo ranks.

The path shards into independent problems (each rank its own batch of heads, no
data exchange), so the only collective is the timing reduction: every rank takes
the slowest rank's time and the job's rate is the units of all ranks over it.
The reference arm, launched like the other arm under torchrun, runs on rank 0
alone and the other ranks leave without work.
"""
import datetime
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
from exact_io_aware_54_b200 import synth  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, times):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        ms_max = bench.max_over_ranks(times[rank], world, "cpu")
        rate = bench.whole_job_rate(world, 3.0e9, ms_max, scale=1e9)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms_max": ms_max, "rate": rate}, f)
    finally:
        torch.distributed.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_count_all_units(tmp_path):
    times = [2.0, 5.0]
    mp.spawn(_rank_main, args=(2, _free_port(), str(tmp_path), times), nprocs=2, join=True)
    got = [json.loads((tmp_path / f"rank{r}.json").read_text()) for r in range(2)]
    assert got[0] == got[1]
    assert got[0]["ms_max"] == 5.0
    # 2 ranks x 3e9 units in 5 ms = 1200e9 units/s
    assert got[0]["rate"] == pytest.approx(1200.0)


def test_one_rank_needs_no_process_group():
    assert not torch.distributed.is_initialized()
    assert bench.max_over_ranks(4.0, 1, "cpu") == 4.0
    assert bench.whole_job_rate(1, 2.0e12, 4.0) == pytest.approx(500.0)


def test_each_rank_draws_its_own_shard():
    base = synth.SEEDS["gpt2m"]
    seeds = [bench.shard_seed(base, r) for r in range(8)]
    assert len(set(seeds)) == 8 and seeds[0] == base
    q0 = synth.prefill_inputs(seeds[0], 1, 8, 8, 2, 64)[0]
    q1 = synth.prefill_inputs(seeds[1], 1, 8, 8, 2, 64)[0]
    assert not torch.equal(q0, q1)


def test_reference_arm_other_ranks_do_no_work():
    class Args:
        steps, warmup = 1, 3

    assert bench.run_reference(Args(), rank=1, world=2) is None


def test_reference_arm_under_torchrun_prints_one_line():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2", "--master-addr",
           "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
