"""The multi-GPU bench path's host logic on CPU: two gloo ranks.

bench.py runs N independent replicas (rows are independent, weights are
replicated; there is no data-path exchange), so its only cross-rank logic is
the barrier, the max over ranks of the timed region, the whole-job aggregate
and the per-rank token batches.  This runs them with world_size 2 over gloo.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import lmoe_inputs as li
        dist.barrier()
        per_rank_ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        job_ms = bench.max_over_ranks(per_rank_ms, "cpu")
        w = li.WORKLOADS["tiny_fp32"]
        x = li.tokens(w, 8, seed=bench.replica_seed(w, rank))
        gathered = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(gathered, x)
        out[rank] = (job_ms, bench.job_tokens_per_s(world, w.T, job_ms), not torch.equal(gathered[0], gathered[1]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_distinct_batches():
    world = 2
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out[0] == out[1]
    job_ms, tok_s, distinct = out[0]
    assert job_ms == 15.0                                   # max over ranks
    assert tok_s == pytest.approx(world * 256 / 0.015)      # both ranks' tokens / slowest time
    assert distinct                                         # replicas draw different batches


def test_single_process_needs_no_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5


def test_bench_gpus_flag_starts_the_ranks_itself():
    """`bench.py --gpus 2` run as a plain script (no WORLD_SIZE) starts two
    ranks through torch.distributed.run; with --launch-check each rank times a
    trivial CPU step over gloo, and rank 0's line reports both ranks, the max
    over ranks (rank 1 adds 5 ms) and the whole-job aggregate."""
    import json
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--launch-check",
                        "--steps", "3", "--warmup", "3"], capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(s) for s in r.stdout.splitlines() if s.startswith("{")]
    assert len(lines) == 1, r.stdout                 # rank 0 alone prints
    line = lines[0]
    assert line["launch_check"] and line["n_gpus"] == 2
    assert line["job_ms"] >= line["rank_ms"]                  # the max over ranks
    assert line["value"] == pytest.approx(2 * 1024 / (line["job_ms"] / 3 / 1e3))
