"""Host logic of bench.py's multi-process path, on CPU with gloo: the job's
time is the slowest rank's, the rate counts every rank's units, and the
reference arm runs on rank 0 alone."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        ms = [1.25, 3.5][rank]                       # rank 1 is the slow replica
        slowest = bench.max_over_ranks(ms, world)
        rate = bench.job_rate(1024, world, slowest)
        ref_ran = None
        if rank != 0:
            # the reference arm returns at once on every rank but 0
            class A:
                config, steps, warmup, cpu_sample_tokens = "tiny", 1, 1, 1
            ref_ran = bench.run_reference(A(), rank, world)
        out[rank] = (slowest, rate, ref_ran)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_rate():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        slowest, rate, ref_ran = out[rank]
        assert slowest == 3.5
        assert rate == pytest.approx(world * 1024 / 3.5e-3)
    assert out[1][2] is None


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(2.0, 1) == 2.0
    assert bench.job_rate(10, 1, 1.0) == pytest.approx(10000.0)


def test_reference_arm_line_matches_the_cuda_arm_contract():
    """The reference arm (the oracle on host cores) prints one JSON line with the
    CUDA arm's metric, unit, direction and workload keys, plus its own
    cpu_baseline and a zero-copy e2e."""
    import json
    import subprocess
    import bench
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--config", "tiny", "--steps", "1", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, check=True).stdout
    lines = [json.loads(l) for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = lines[0]
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC
    assert line["unit"] == "routed pairs/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 1 and line["warmup"] == 1
    cfg = bench.wl.config("tiny")
    expect = bench.workload_config(cfg, cfg.modes[0], *bench.routed_pairs_and_active(cfg))
    for k, v in expect.items():
        assert line["config"][k] == v, k
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
