"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The forward shards across GPUs by work item (batch element / head) with no
data-path collective; the only cross-rank steps are the timing and FLOP
reductions and the per-rank input sharding, which these tests exercise.
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import numpy as np
    import torch.distributed as dist

    import bench
    from synth import WORKLOADS, fourier_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    wl = WORKLOADS["tiny"]
    q, k, v = bench.rank_inputs(wl, rank)
    res = {
        "max": bench.max_over_ranks(float(rank + 1), dist),
        "sum": bench.sum_over_ranks(float(10 * (rank + 1)), dist),
        "shape": list(q.shape),
        "q_sum": int(q.astype(np.int64).sum()),
    }
    # the rank's slice is batch element `rank` of a batch of `world` copies
    import dataclasses
    big = dataclasses.replace(wl, B=world)
    qq, _, _ = fourier_inputs(big)
    res["matches_global"] = bool(np.array_equal(qq[rank:rank + 1], q))
    with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_reductions_and_sharding(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(world)]
    for x in r:
        assert x["max"] == 2.0          # slowest rank's time
        assert x["sum"] == 30.0         # FLOPs of all ranks
        assert x["shape"] == [1, 1, 1024, 64]
        assert x["matches_global"]
    assert r[0]["q_sum"] != r[1]["q_sum"]   # each rank works on its own batch element
