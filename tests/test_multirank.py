"""The N>1 bench path on CPU: two gloo ranks, independent replicas, max-over-ranks time.

The layer is token-parallel, so ranks exchange nothing on the data path. The only
cross-rank steps are the barriers and the MAX reduction of the timed duration.
"""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import bench
    import qe_inputs as qi
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    mine = 10.0 * (rank + 1)          # each rank's own timed duration
    got = bench.max_over_ranks(mine, dist)
    seeds = [bench.replica_x_seed(rank, p) for p in range(5)]
    cfg = qi.CONFIGS["tiny"]
    x = qi.outlier_activations(8, 256, bench.replica_x_seed(rank, 0), cfg.outlier_spec(256))
    dist.barrier()
    out[rank] = (got, seeds, float(x.sum()))
    dist.destroy_process_group()


def test_two_rank_replicas_take_max_time_and_distinct_batches():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 20.0
    assert set(res[0][1]).isdisjoint(res[1][1])    # replicas draw different token batches
    assert res[0][2] != res[1][2]


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(3.5, None) == 3.5
