"""The TP domain of two ranks on one GPU (reading R26): the dispatch of all
2 * ws source devices' tokens (TP-major) with one instance per EP rank, the
per-(rank, domain) counts, and the combine whose gathered rows are the bf16
sums of the TP pair's two partial expert outputs (ReduceScatterV), against
the oracle's separate AllToAllV per domain + AllGatherV and its
ReduceScatterV (aclnnMoeDistributeDispatchV2 and
aclnnMoeDistributeCombineAddRmsNorm, 计算公式)."""
import numpy as np
import pytest
import torch

from combine_moe_update_b200 import inputs as gen
from oracle import oracle as orc

from gpu_harness import assert_close_bf16, dev, dev_bf16, host, poison_

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_moe_update_b200 import binding
    return binding


def _bytes(a, lo, hi):
    a = np.ascontiguousarray(a)
    return a.view(np.uint8).reshape(a.shape[0], -1)[lo:hi]


@pytest.mark.parametrize("ws,bs,K,H,mode,smooth,prune", [
    (4, 16, 4, 1024, 0, False, 0.0),     # 512 copies: the self-routing scatter
    (8, 64, 6, 2048, 2, True, 0.0),      # 6144 copies: the route kernel
    (8, 48, 8, 1040, 3, False, 0.1),     # ragged tile, pruning
    (4, 32, 4, 1024, 4, False, 0.0),     # mxfp8
    (16, 256, 4, 1024, 2, False, 0.05),  # 32768 copies: the three-pass route
])
def test_tp_dispatch_counts_and_combine(B, ws, bs, K, H, mode, smooth, prune):
    S, E = 2 * ws, ws
    T = S * bs
    rng = np.random.Generator(np.random.PCG64([126, ws, bs, mode]))
    x = gen.bf16_bits(rng.standard_normal((T, H), np.float32))
    ids = gen.topk_uniform(rng, T, E, K)
    sc = gen.softmax_scales(rng, T, K)
    table = gen.identity_table(E, ws)
    sm = rng.uniform(0.5, 2.0, size=(E, H)).astype(np.float32) if smooth else None
    sl = 0 if sm is None else sm.size
    wsp = B.new_workspace(nbytes=B.dispatch_workspace_bytes(bs, H, K, ws, E, mode, sl, S))
    bal = poison_(torch.empty((T, K), dtype=torch.int32, device="cuda"))
    bm = poison_(torch.empty((T, K), dtype=torch.uint8, device="cuda"))
    B.update_expert(dev(ids), dev(table), ws, expert_scales=dev(sc), prune_threshold=prune, workspace=wsp,
                    out=(bal, bm), sources=S)
    d = B.alloc_dispatch_outputs(T, H, K, E, mode)
    for t in d.values():
        if t is not None:
            poison_(t)
    B.dispatch(dev_bf16(x), bal, E, ws, mode, mask=bm, smooth=None if sm is None else dev(sm), workspace=wsp,
               out=d, sources=S)
    tpc = poison_(torch.empty((E, 2), dtype=torch.int32, device="cuda"))
    B.dispatch_tp_counts(d, bs, H, K, ws, mode, scales_len=sl, workspace=wsp, out=tpc)
    torch.cuda.synchronize()
    assert B.read_device_error(wsp) == 0

    bal_o, bm_o, e1 = orc.update_expert(ids, table, ws, expert_scales=sc, prune_threshold=prune)
    assert e1 == 0
    od = orc.dispatch_tp(x, bal_o, E, mode, ws, bs, mask=bm_o, smooth=sm)
    assert od["err"] == 0
    n = od["n"]
    np.testing.assert_array_equal(host(d["expand_idx"]), od["expand_idx"])
    np.testing.assert_array_equal(host(d["counts"]), od["counts"])
    np.testing.assert_array_equal(host(d["offsets"]), od["offsets"])
    np.testing.assert_array_equal(host(d["src_of_row"])[:n], od["src_of_row"])
    np.testing.assert_array_equal(_bytes(host(d["expand_x"]), 0, n), _bytes(od["expand_x"], 0, n))
    if od["dyn_scales"] is not None:
        np.testing.assert_array_equal(_bytes(host(d["dyn_scales"]), 0, n), _bytes(od["dyn_scales"], 0, n))
    np.testing.assert_array_equal(host(tpc), od["tp_counts"])

    # the TP pair's partial expert outputs of every row, then the combine with the ReduceScatterV
    rows = T * K
    p0 = gen.bf16_bits(rng.standard_normal((rows, H), np.float32))
    p1 = gen.bf16_bits(rng.standard_normal((rows, H), np.float32))
    res = gen.bf16_bits(rng.standard_normal((T, H), np.float32))
    sh = gen.bf16_bits(rng.standard_normal((T, H), np.float32))
    g = gen.bf16_bits(rng.uniform(0.5, 1.5, size=H).astype(np.float32))
    out = B.combine_add_rmsnorm_tp2(dev_bf16(p0), dev_bf16(p1), d["expand_idx"], dev(sc), dev_bf16(res),
                                    dev_bf16(g), 1e-6, shared_x=dev_bf16(sh), want_x_out=True, workspace=wsp,
                                    sources=S)
    torch.cuda.synchronize()
    assert B.read_device_error(wsp) == 0
    oc = orc.combine_add_rmsnorm_tp(p0, p1, od["expand_idx"], sc, res, g, 1e-6, shared_x=sh)
    assert_close_bf16(host(out["y"]), oc["y_f64"], what="y")
    assert_close_bf16(host(out["x_out"]), oc["x_f64"], what="x_out")


@pytest.mark.parametrize("K,shared", [(2, False), (8, True), (16, False)])
def test_tp_combine_reduces_exactly(B, K, shared):
    """With the second partial zero the TP combine is, bit for bit, the
    one-rank combine of the first; with two equal partials, that of the
    doubled rows (exact in bf16); and swapping the partials changes no bit.
    320 tokens: more than two per SM, so the one-rank combine also runs one
    block per token and sums x^2 in the same order (two half-row blocks per
    token would add the halves' sums, which may differ in the last bit)."""
    rng = np.random.default_rng(1000 + K)
    bs, H = 320, 7168
    rows = bs * K
    p0 = gen.bf16_bits(rng.standard_normal((rows, H), np.float32))
    idx = rng.permutation(rows).reshape(bs, K).astype(np.int32)
    idx[::5, 0] = -1
    sc = gen.softmax_scales(rng, bs, K)
    res = gen.bf16_bits(rng.standard_normal((bs, H), np.float32))
    sh = gen.bf16_bits(rng.standard_normal((bs, H), np.float32)) if shared else None
    g = gen.bf16_bits(rng.uniform(0.5, 1.5, size=H).astype(np.float32))
    D = lambda a: None if a is None else dev_bf16(a)
    zero = np.zeros_like(p0)
    twice = gen.bf16_bits(gen.bf16_to_f32(p0) * 2.0)
    a = B.combine_add_rmsnorm_tp2(D(p0), D(zero), dev(idx), dev(sc), D(res), D(g), 1e-6, shared_x=D(sh))
    b = B.combine_add_rmsnorm(D(p0), dev(idx), dev(sc), D(res), D(g), 1e-6, shared_x=D(sh))
    c = B.combine_add_rmsnorm_tp2(D(p0), D(p0), dev(idx), dev(sc), D(res), D(g), 1e-6, shared_x=D(sh))
    dd = B.combine_add_rmsnorm(D(twice), dev(idx), dev(sc), D(res), D(g), 1e-6, shared_x=D(sh))
    p1 = gen.bf16_bits(rng.standard_normal((rows, H), np.float32))
    e = B.combine_add_rmsnorm_tp2(D(p0), D(p1), dev(idx), dev(sc), D(res), D(g), 1e-6, shared_x=D(sh))
    f = B.combine_add_rmsnorm_tp2(D(p1), D(p0), dev(idx), dev(sc), D(res), D(g), 1e-6, shared_x=D(sh))
    torch.cuda.synchronize()
    assert torch.cuda.get_device_properties(0).multi_processor_count * 2 <= bs
    np.testing.assert_array_equal(host(a["y"]), host(b["y"]))
    np.testing.assert_array_equal(host(c["y"]), host(dd["y"]))
    np.testing.assert_array_equal(host(e["y"]), host(f["y"]))
    oc = orc.combine_add_rmsnorm_tp(p0, p1, idx, sc, res, g, 1e-6, shared_x=sh)
    assert_close_bf16(host(e["y"]), oc["y_f64"], what="y")


def test_tp_counts_refuses_other_layouts(B):
    """The TP counts need one instance per rank and 2 * ws sources."""
    ws, bs, K, H = 4, 8, 2, 1024
    d = B.alloc_dispatch_outputs(2 * ws * bs, H, K, ws, 0)
    with pytest.raises(B.MoeError):  # sources = 2 * ws, but 2 instances per rank
        p = B.DispatchParams(bs, H, K, ws, 2 * ws, 0, 0, 2 * ws)
        rc = B.lib.moe_dispatch_tp_counts(
            __import__("ctypes").byref(p), d["src_of_row"].data_ptr(), d["offsets"].data_ptr(),
            torch.empty((ws, 2), dtype=torch.int32, device="cuda").data_ptr(),
            B.new_workspace().data_ptr(), B.WORKSPACE_BYTES, None)
        B._check("moe_dispatch_tp_counts", rc)


@pytest.mark.parametrize("ws,bs,K,H,mode,smooth,prune,by_address", [
    (4, 8, 4, 1024, 0, False, 0.0, False),   # 256 copies: the self-routing scatter
    (8, 32, 6, 2048, 2, True, 0.05, True),   # 3072 copies: the route kernel; the peer's partial by address
    (8, 24, 8, 1040, 3, False, 0.1, True),   # ragged tile, pruning
])
def test_tp_pair_across_two_gpus_emulated(B, ws, bs, K, H, mode, smooth, prune, by_address):
    """The TP pair split over two GPUs (combine_moe_update_b200.tp), both
    emulated on this device: GPU t holds TP domain t's tokens; after the
    gather each GPU's dispatch of the pair's tokens must equal the oracle's
    AllToAllV per domain + AllGatherV bit for bit (so both GPUs hold the same
    rows), and each GPU's combine of its own tokens, reading the peer's
    partial outputs, must equal the one-GPU TP combine of those tokens bit
    for bit and the oracle's ReduceScatterV + combine element-wise."""
    from combine_moe_update_b200 import tp as TP
    S, E = 2 * ws, ws
    T, Th = S * bs, ws * bs
    rng = np.random.Generator(np.random.PCG64([127, ws, bs, mode]))
    x = gen.bf16_bits(rng.standard_normal((T, H), np.float32))
    ids = gen.topk_uniform(rng, T, E, K)
    sc = gen.softmax_scales(rng, T, K)
    table = gen.identity_table(E, ws)
    sm = rng.uniform(0.5, 2.0, size=(E, H)).astype(np.float32) if smooth else None
    res = gen.bf16_bits(rng.standard_normal((T, H), np.float32))
    sh = gen.bf16_bits(rng.standard_normal((T, H), np.float32))
    g = gen.bf16_bits(rng.uniform(0.5, 1.5, size=H).astype(np.float32))
    p0 = gen.bf16_bits(rng.standard_normal((T * K, H), np.float32))
    p1 = gen.bf16_bits(rng.standard_normal((T * K, H), np.float32))

    pair = TP.EmulatedTPPair(ws=ws, bs=bs, hidden=H, top_k=K, quant_mode=mode,
                             scales_len=0 if sm is None else sm.size)
    half = lambda a, t: a[t * Th:(t + 1) * Th]
    local = [dict(x=dev_bf16(half(x, t)), expert_ids=dev(half(ids, t)), expert_scales=dev(half(sc, t)))
             for t in (0, 1)]
    for r in pair.ranks:
        for v in r.d.values():
            if v is not None:
                poison_(v)
    full = pair.dispatch(local, dev(table), smooth=None if sm is None else dev(sm), prune_threshold=prune)
    pair.ranks[0].partial.copy_(dev_bf16(p0))
    pair.ranks[1].partial.copy_(dev_bf16(p1))
    inputs = [dict(residual=dev_bf16(half(res, t)), gamma=dev_bf16(g), shared_x=dev_bf16(half(sh, t)))
              for t in (0, 1)]
    outs = pair.combine(full, inputs, 1e-6, peer_by_address=by_address)
    one = B.combine_add_rmsnorm_tp2(dev_bf16(p0), dev_bf16(p1), pair.ranks[0].d["expand_idx"], dev(sc),
                                    dev_bf16(res), dev_bf16(g), 1e-6, shared_x=dev_bf16(sh), sources=S)
    torch.cuda.synchronize()
    assert all(r.device_errors() == 0 for r in pair.ranks)

    bal_o, bm_o, e1 = orc.update_expert(ids, table, ws, expert_scales=sc, prune_threshold=prune)
    assert e1 == 0
    od = orc.dispatch_tp(x, bal_o, E, mode, ws, bs, mask=bm_o, smooth=sm)
    n = od["n"]
    for r in pair.ranks:
        np.testing.assert_array_equal(host(r.d["expand_idx"]), od["expand_idx"])
        np.testing.assert_array_equal(host(r.d["offsets"]), od["offsets"])
        np.testing.assert_array_equal(_bytes(host(r.d["expand_x"]), 0, n), _bytes(od["expand_x"], 0, n))
        if od["dyn_scales"] is not None:
            np.testing.assert_array_equal(_bytes(host(r.d["dyn_scales"]), 0, n), _bytes(od["dyn_scales"], 0, n))
        np.testing.assert_array_equal(host(r.tp_counts), od["tp_counts"])
    oc = orc.combine_add_rmsnorm_tp(p0, p1, od["expand_idx"], sc, res, g, 1e-6, shared_x=sh)
    for t, o in enumerate(outs):
        np.testing.assert_array_equal(host(o["y"]), half(host(one["y"]), t))
        assert_close_bf16(host(o["y"]), half(oc["y_f64"], t), what=f"y of GPU {t}")
        assert_close_bf16(host(o["x_out"]), half(oc["x_f64"], t), what=f"x_out of GPU {t}")
