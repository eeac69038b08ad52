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


def _partition_rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import numpy as np
    import bench
    import residual_bit_kv_b200.synth as synth
    from rq_harness import oracle_decode
    ws, r, _ = bench.dist_env()
    dist = bench.init_dist(ws, backend="gloo")
    try:
        per_rank = synth.WORKLOADS["ouro_layer"].replace(batch=2, heads=2, tokens=40)
        mine = bench.rank_share(per_rank, r, ws)
        lens = synth.seq_lens_ragged(mine)
        outs = [oracle_decode(mine, 0, loop, range(mine.batch), range(mine.heads), lens)
                for loop in range(mine.loops)]
        gathered = [None] * ws
        dist.all_gather_object(gathered, (mine.batch0, mine.batch, np.stack(outs)))
        if r == 0:
            np.save(os.path.join(out_dir, "gathered.npy"),
                    np.concatenate([g[2] for g in sorted(gathered, key=lambda g: g[0])], axis=1))
            with open(os.path.join(out_dir, "slices.json"), "w") as f:
                json.dump([[g[0], g[1]] for g in gathered], f)
    finally:
        dist.destroy_process_group()


def test_two_rank_batch_partition_matches_one_rank(tmp_path):
    """Multi-GPU runs split one global batch: rank r takes batch rows
    [rB/N, (r+1)B/N) of a workload of N times the per-rank batch.  Two gloo
    ranks each decode their rows with the oracle; their outputs, put side by
    side, equal the one-process oracle decode of the whole batch."""
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import numpy as np
    import residual_bit_kv_b200.synth as synth
    from rq_harness import oracle_decode
    world = 2
    mp.start_processes(_partition_rank_main, args=(world, _free_port(), str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    assert json.load(open(tmp_path / "slices.json")) == [[0, 2], [2, 2]]
    whole = synth.WORKLOADS["ouro_layer"].replace(batch=4, heads=2, tokens=40)
    lens = synth.seq_lens_ragged(whole)
    want = np.stack([oracle_decode(whole, 0, loop, range(4), range(2), lens)
                     for loop in range(whole.loops)])
    np.testing.assert_array_equal(np.load(tmp_path / "gathered.npy"), want)


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
