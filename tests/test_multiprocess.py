"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

bench.py runs one process per GPU; every rank prunes its own draw of the
workload (no collective on the data path) and the step times are reduced with
MAX over ranks.  These tests run that host logic with the gloo backend."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    vals = bench.max_over_ranks([rank + 1.0, 10.0 - rank, -float(rank), 0.5 * rank])
    wl = bench.rank_workload(1, rank)
    desc = wl.describe()
    # the reference arm runs on rank 0 only; the other ranks return without work
    out = io.StringIO()
    if rank != 0:
        with redirect_stdout(out):
            bench.run_reference(type("A", (), dict(workload=1, steps=1, warmup=3, gpus=world,
                                                   ref_seconds=0.1))())
    dist.barrier()
    dist.destroy_process_group()
    queue.put((rank, vals, wl.seed, json.dumps(desc, sort_keys=True), out.getvalue()))


def test_max_over_ranks_and_per_rank_workloads():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=180) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    (r0, v0, s0, d0, o0), (r1, v1, s1, d1, o1) = res
    assert v0 == v1 == [2.0, 10.0, 0.0, 0.5]  # element-wise max, seen by every rank
    assert s0 != s1                           # each rank draws its own cache
    assert d0 == d1                           # of the same shapes
    assert o1 == ""                           # rank 1 printed no reference line


def test_single_process_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, -1.0]) == [3.0, -1.0]
    assert bench.rank_workload(1, 0).seed == 1
