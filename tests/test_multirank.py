"""The N > 1 path of bench.py on CPU: two gloo ranks, replicas of the same
step, the device-timed region reduced to its maximum over ranks, and the
reference arm doing no work on ranks other than 0."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 20.0][rank]  # this rank's device-timed region
        job_ms = bench.max_over_ranks(ms, world, torch.device("cpu"))
        value = bench.job_throughput(10**12, 4, world, job_ms)
        out[rank] = (job_ms, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_is_the_max_and_value_counts_all_ranks():
    world = 2
    manager = mp.get_context("spawn").Manager()  # no fork of a process that may hold a CUDA context
    out = manager.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1]
    job_ms, value = out[0]
    assert job_ms == 20.0
    # 2 ranks x 4 steps x 1e12 ops in 20 ms
    assert value == pytest.approx(2 * 4 * 1e12 / 0.020 / 1e12)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(7.0, 1, torch.device("cpu")) == 7.0


def test_reference_arm_on_a_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert res.returncode == 0
    assert res.stdout.strip() == ""


def test_reference_arm_prints_one_contract_line():
    """rank 0 of the reference arm: the oracle on a bounded sample of the layer
    step, one JSON line with the keys the bench contract asks for."""
    import json

    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["value"] > 0 and d["higher_is_better"] is True and d["unit"] == "TOPS"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "llama70b_layer_fwd_bwd"
