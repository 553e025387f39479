"""Expert parallelism across GPUs: the multi-rank host logic on CPU, two gloo
ranks (no GPU is touched).

Each rank is one GPU of the group and one source of its own tokens.  It
dispatches its tokens (here with the oracle, standing in for the GPU's
moe_dispatch), gathers every rank's per-instance counts with
ep.gather_counts, and passes ep.group_barrier.  The test then checks the
layout the group's kernels build from those counts -- copy (i, k) of rank
g of instance e lands at global row
    (rows of instances < e, all ranks) + (rows of e from ranks < g)
    + (its position among rank g's copies of e)
-- against the oracle's dispatch of all ranks' tokens on one device
(aclnnMoeDistributeDispatchV2, 计算公式: the AllToAllV over the EP ranks):
the group's rows must be exactly the single-device rows.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
G, BS, H, E, K, WS = 2, 48, 1024, 16, 4, 4


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload():
    from combine_moe_update_b200 import inputs as gen
    rng = np.random.Generator(np.random.PCG64(91))
    return (gen.bf16_bits(rng.standard_normal((G * BS, H), np.float32)), gen.topk_uniform(rng, G * BS, E, K),
            gen.identity_table(E, WS))


def _worker(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    try:
        import torch
        import torch.distributed as dist

        from combine_moe_update_b200 import ep
        from oracle import oracle as orc
        dist.init_process_group("gloo", rank=rank, world_size=G, timeout=datetime.timedelta(seconds=60))
        x, ids, table = _workload()
        mine = slice(rank * BS, (rank + 1) * BS)
        bal, bm, _ = orc.update_expert(ids[mine], table, WS)
        d = orc.dispatch(x[mine], bal, E, 0, mask=bm)
        counts_all = torch.empty((G, E), dtype=torch.int32)
        ep.gather_counts(torch.from_numpy(d["counts"]), counts_all)
        ep.group_barrier(torch.zeros(1))
        dist.destroy_process_group()
        q.put((rank, counts_all.numpy().copy(), d["expand_idx"], d["offsets"], bal, None))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, None, None, None, None, repr(e)))


def test_two_gloo_ranks_build_the_one_device_layout():
    from combine_moe_update_b200 import build
    build.build()  # the ranks import the library's binding
    from oracle import oracle as orc
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(G)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(G):
        r = q.get(timeout=180)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
    for r in res.values():
        assert r[5] is None, r[5]

    x, ids, table = _workload()
    bal, bm, _ = orc.update_expert(ids, table, WS)
    od = orc.dispatch(x, bal, E, 0, mask=bm)
    counts_all = np.stack([res[g][3][1:] - res[g][3][:-1] for g in range(G)])
    for g in range(G):
        np.testing.assert_array_equal(res[g][1], counts_all)  # every rank gathered every rank's counts
    tot = counts_all.sum(0)
    excl = np.concatenate([[0], np.cumsum(tot)[:-1]])
    for g in range(G):
        _, _, idx, off, bal_g, _ = res[g]
        before = counts_all[:g].sum(0)
        glob = np.where(idx >= 0, excl[bal_g] + before[bal_g] + (idx - off[bal_g]), -1)
        np.testing.assert_array_equal(glob, od["expand_idx"][g * BS:(g + 1) * BS])
    # each rank's instances own a contiguous stretch of the one-device rows
    El = E // G
    for qd in range(G):
        assert od["offsets"][(qd + 1) * El] - od["offsets"][qd * El] == tot[qd * El:(qd + 1) * El].sum()
