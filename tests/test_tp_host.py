"""The TP pair across two GPUs: the host logic on CPU, two gloo ranks (no GPU
is touched).

Rank t is GPU t of the pair, holding TP domain t's tokens.  Each rank
gathers the pair's token arrays with tp.gather_tp_major and dispatches all
of them (here with the oracle, standing in for the GPU's moe_dispatch).  The
gathered arrays must be the pair's arrays in TP-major order on both ranks
(domain 0's tokens first), and both ranks' rows must then be the one-device
rows of the 2 * ws sources, the oracle's AllToAllV per domain followed by
the AllGatherV (aclnnMoeDistributeDispatchV2, 计算公式): the same receive
buffer on both GPUs of the pair.
"""
import datetime
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
WS, BS, H, K = 4, 12, 1024, 3
E, S = WS, 2 * WS
T, TH = S * BS, WS * BS


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload():
    from combine_moe_update_b200 import inputs as gen
    rng = np.random.Generator(np.random.PCG64(93))
    return (gen.bf16_bits(rng.standard_normal((T, H), np.float32)), gen.topk_uniform(rng, T, E, K),
            gen.softmax_scales(rng, T, K), gen.identity_table(E, WS))


def _worker(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    try:
        import torch
        import torch.distributed as dist

        from combine_moe_update_b200 import tp
        from oracle import oracle as orc
        dist.init_process_group("gloo", rank=rank, world_size=2, timeout=datetime.timedelta(seconds=60))
        x, ids, sc, table = _workload()
        mine = slice(rank * TH, (rank + 1) * TH)
        # bf16 bits as pairs in int32 (gloo has no 16-bit integer type)
        gx = tp.gather_tp_major(torch.from_numpy(x[mine].view(np.int32))).numpy().view(np.uint16)
        gi = tp.gather_tp_major(torch.from_numpy(ids[mine])).numpy()
        gs = tp.gather_tp_major(torch.from_numpy(sc[mine])).numpy()
        bal, bm, _ = orc.update_expert(gi, table, WS, expert_scales=gs, prune_threshold=0.1)
        d = orc.dispatch_tp(gx, bal, E, 2, WS, BS, mask=bm)
        dist.destroy_process_group()
        q.put((rank, gx, gi, gs, d["expand_idx"], d["expand_x"], d["dyn_scales"], d["tp_counts"], None))
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank,) + (None,) * 7 + (repr(e),))


def test_two_gloo_ranks_gather_the_pair_and_hold_the_same_rows():
    from combine_moe_update_b200 import build
    build.build()  # the ranks import the library's binding
    from oracle import oracle as orc
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r = q.get(timeout=180)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
    for r in res.values():
        assert r[-1] is None, r[-1]

    x, ids, sc, table = _workload()
    bal, bm, _ = orc.update_expert(ids, table, WS, expert_scales=sc, prune_threshold=0.1)
    od = orc.dispatch_tp(x, bal, E, 2, WS, BS, mask=bm)
    n = od["n"]
    for t in (0, 1):
        _, gx, gi, gs, idx, ex, ds, tpc, _ = res[t]
        np.testing.assert_array_equal(gx, x)  # TP-major: domain 0's tokens, then domain 1's
        np.testing.assert_array_equal(gi, ids)
        np.testing.assert_array_equal(gs, sc)
        np.testing.assert_array_equal(idx, od["expand_idx"])
        np.testing.assert_array_equal(ex[:n], od["expand_x"][:n])
        np.testing.assert_array_equal(ds[:n], od["dyn_scales"][:n])
        np.testing.assert_array_equal(tpc, od["tp_counts"])
    assert od["tp_counts"][:, 0].sum() > 0 and od["tp_counts"][:, 1].sum() > 0  # both domains sent rows
