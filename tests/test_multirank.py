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


def test_gpus_flag_launches_that_many_ranks():
    # `bench.py --gpus 2` outside torchrun starts two ranks itself (torch.distributed.run on
    # 127.0.0.1). The reference arm runs on CPU: rank 0 times the oracle and prints the line,
    # rank 1 exits without work, and n_gpus reports the launched world size.
    import json
    import subprocess
    env = dict(os.environ)
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(k, None)
    env["OMP_NUM_THREADS"] = "2"
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0", "--cpu-seconds", "0.3", "--workload", "qwen2vl2b"],
                       capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2


def test_gpus_flag_must_match_the_launcher():
    import subprocess
    env = dict(os.environ, WORLD_SIZE="3", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert r.returncode != 0 and "launcher started 3 ranks" in r.stderr
