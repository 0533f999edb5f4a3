"""The bench's multi-process path on the CPU: two gloo ranks, max-over-ranks timing and the whole-job rate.

Each rank is an independent replica (the path has no exchange step on one node), so the only collective is
the element-wise max of the ranks' timings; rank 0 reports B * world queries over the slowest rank's time.
"""

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
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r's step / e2e / stage times (ms): rank 1 is slower on the step, rank 0 on one stage
        mine = torch.tensor([0.10 + 0.02 * rank, 0.30 - 0.05 * rank, 0.04 + 0.01 * (1 - rank), 0.03], dtype=torch.float64)
        got = bench.max_over_ranks(mine, world)
        out[rank] = got.tolist()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_gloo_two_ranks():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    want = [0.12, 0.30, 0.05, 0.03]
    for r in range(world):
        assert out[r] == pytest.approx(want)


def test_job_rate_counts_every_rank():
    import bench

    assert bench.job_rate(16, 1, 0.1) == pytest.approx(160000.0)
    assert bench.job_rate(16, 8, 0.1) == pytest.approx(8 * 160000.0)


def test_reference_arm_runs_on_rank_zero_only():
    import bench

    class Args:
        steps, warmup = 1, 3

    assert bench.run_reference(Args(), rank=1, world=2) is None


@pytest.mark.timeout(300)
def test_reference_arm_line_on_rank_zero():
    """The oracle arm's JSON line carries the contract keys, with its own value repeated in cpu_baseline and e2e."""
    import bench

    class Args:
        steps, warmup = 1, 3

    res = bench.run_reference(Args(), rank=0, world=1)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in res, key
    assert res["impl"] == "reference" and res["value"] > 0 and res["steps"] == 1
    assert res["cpu_baseline"]["value"] == res["value"] and res["cpu_baseline"]["kind"] == "oracle"
    assert res["e2e"]["value"] == res["value"] and res["e2e"]["h2d_bytes_per_step"] == 0
    assert res["metric"] == "sparse decode queries/s @L=128K,K=2048"
