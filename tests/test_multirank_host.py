"""The bench's multi-process host logic on CPU: two gloo ranks.

bench.py runs one process per GPU under torch.distributed.run and reports
the slowest rank's time, so its rank plumbing (environment parsing, the
element-wise max / sum over ranks, the barrier, and the reference arm that
only rank 0 runs) is checked here with world_size 2 on the gloo backend.
No GPU is touched.
"""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        env = bench.dist_env()
        mx = bench.reduce_over_ranks([rank + 1.0, 10.0 - rank, 0.5 * rank], "max")
        sm = bench.reduce_over_ranks([rank + 1.0], "sum")
        bench.barrier()
        # the reference arm: rank 0 alone does the work and returns its line
        ref_is_none = None
        if rank != 0:
            ref_is_none = bench.run_reference(None, rank) is None
        bench.barrier()
        dist.destroy_process_group()
        q.put((rank, env, mx, sm, ref_is_none, None))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, None, None, None, None, repr(e)))


def test_two_gloo_ranks_reduce_and_barrier():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    try:
        for _ in range(world):
            rank, env, mx, sm, ref_is_none, err = q.get(timeout=120)
            out[rank] = (env, mx, sm, ref_is_none, err)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    for rank in range(world):
        env, mx, sm, ref_is_none, err = out[rank]
        assert err is None, err
        assert env == (rank, world, rank)
        assert mx == [2.0, 10.0, 0.5]  # element-wise max over ranks
        assert sm == [3.0]
        if rank != 0:
            assert ref_is_none  # only rank 0 prints the reference line
    for p in procs:
        assert p.exitcode == 0


def test_single_process_reduce_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks([1.5, 2.5], "max") == [1.5, 2.5]
    bench.barrier()  # no process group: a no-op
