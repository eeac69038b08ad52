"""The multi-process plumbing of bench.py on CPU: two ranks over gloo (the
GPU path uses the same calls over NCCL).  The decode path itself has no
collective: every (batch, head) unit is independent, so each rank decodes its
own batch and only the step time is reduced (max over ranks)."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench
    ws, r, local = bench.dist_env()
    dist = bench.init_dist(ws, backend="gloo")
    try:
        # every rank reports its own step time; all must see the slowest
        mine = 10.0 + 7.5 * r
        slowest = bench.max_over_ranks(mine, dist, "cpu")
        # a second reduction in the same order on every rank
        second = bench.max_over_ranks(-float(r), dist, "cpu")
        dist.barrier()
        res = {"rank": r, "ws": ws, "local": local, "slowest": slowest, "second": second,
               "value": bench.job_tokens_per_s(ws, 16, slowest)}
        with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_job_throughput(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, d in enumerate(res):
        assert d["rank"] == r and d["ws"] == world and d["local"] == r
        assert d["slowest"] == 17.5          # max over ranks, not the rank's own
        assert d["second"] == 0.0
        # weak scaling: the job decodes world * batch tokens per slowest step
        assert d["value"] == pytest.approx(world * 16 * 1e3 / 17.5)


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.init_dist(1) is None
    assert bench.max_over_ranks(3.25, None, "cpu") == 3.25
    assert bench.job_tokens_per_s(1, 16, 20.0) == pytest.approx(800.0)


def test_reference_arm_runs_on_rank_zero_only():
    """Under torchrun the reference arm (the CPU oracle) runs on rank 0; the
    other ranks exit 0 without work or output."""
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    args = argparse.Namespace(gpus=2, steps=1, warmup=0, impl="reference")
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.run_reference(args, rank=1) == 0
    assert buf.getvalue() == ""
