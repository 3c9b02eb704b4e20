"""Host-side checks of bench.py (no GPU): the multi-rank timing reduction
and throughput aggregation over a world-size-2 gloo process group, the
reference arm's JSON line, and the seeds that keep ranks independent."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 20.0][rank]  # the second rank is slower
        ms = bench.max_over_ranks(local_ms, world)
        value = bench.throughput(1000, world, ms)
        out[rank] = (ms, value, bench.rank_seed(0, rank))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_time_and_whole_job_throughput():
    port = 29500 + (os.getpid() % 1000)
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    for rank in (0, 1):
        ms, value, seed = res[rank]
        assert ms == 20.0                      # max over ranks, on every rank
        assert value == pytest.approx(2 * 1000 / 0.020)  # all ranks' units / slowest time
    assert res[0][2] != res[1][2]              # independent batches per rank


def test_single_rank_passthrough():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.throughput(100, 1, 50.0) == pytest.approx(2000.0)


def test_algorithmic_counts():
    # chunk form at C=64, d=128: 2C(3dk+2dv) + 6 dk dv
    assert bench.chunk_flops_per_token_head(64, 128, 128) == 180224
    from linear_recurrence_sequence_chunked_b200.workloads import WORKLOADS
    assert bench.fwd_bytes_per_token_head(WORKLOADS["pgdn_bf16_4k"]) == 1032
    assert bench.decode_bytes_per_token_head(WORKLOADS["pgdn_decode_256"]) == 133128


def test_reference_arm_json_line():
    """--impl reference times the fp64 oracle on the host (the only
    reference this path has) and prints one JSON line with impl=reference."""
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "pdn_f32_small", "--steps", "1", "--warmup", "0",
                        "--cpu-seconds", "0.5"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "pdn_f32_small", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""
