"""GPU parity for the instances' grouped int8 matmul (moe_grouped_matmul,
tcgen05 kind::i8) against the CPU oracle on the same seeded inputs.

The int32 sums are exact on both sides, so the only difference is the
rounding of the two scale products (binary32 on the GPU, binary64 in the
oracle) before the one bf16 rounding: results agree bit for bit except where
the exact value lies within ~2^-23 of a bf16 rounding boundary, where they
are one bf16 step apart.  The tests ask for exactly that (and for the 1e-2
bar on every element); with unit scales and single-product rows every
output is exact and must match bit for bit.  Outputs are poisoned first, so
rows the call must not write are checked too."""
import numpy as np
import pytest
import torch

from combine_moe_update_b200 import inputs as gen
from oracle import oracle as orc

from gpu_harness import POISON, assert_close_bf16, assert_gmm_parity as _assert_gmm_parity, dev, dev_bf16, \
    host, poison_

pytestmark = pytest.mark.gpu

POISON16 = POISON * 0x101


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_moe_update_b200 import binding
    return binding


def _gpu(B, gi, weight=None, weight_scales=None):
    rows, H = gi.expand_x.shape
    w = dev(gi.weight) if weight is None else weight
    ws = dev(gi.weight_scales) if weight_scales is None else weight_scales
    E, N = w.shape[0], w.shape[1]
    out = poison_(torch.empty((rows, N), dtype=torch.bfloat16, device="cuda"))
    wsp = B.new_workspace(nbytes=B.grouped_matmul_workspace_bytes(rows, H, N, E))
    B.grouped_matmul(dev(gi.expand_x), dev(gi.dyn_scales), dev(gi.offsets), w, ws, out=out, workspace=wsp)
    torch.cuda.synchronize()
    return host(out), B.read_device_error(wsp)


def _oracle(gi):
    rows, N = gi.expand_x.shape[0], gi.weight.shape[1]
    return orc.grouped_matmul(gi.expand_x, gi.dyn_scales, gi.offsets, gi.weight, gi.weight_scales,
                              out=np.full((rows, N), POISON16, np.uint16))


@pytest.mark.parametrize("H,N,counts,spare", [
    (1024, 256, [3, 0, 17, 130, 1, 128, 16], 5),  # padded N, empty instance
    (1024, 128, [300, 256, 2, 513], 1),           # 256-row slots and remainders
    (1168, 208, [5, 33, 0, 260], 0),              # ragged K tail and a partial channel slab
])
def test_gmm_single_products_bit_exact(B, H, N, counts, spare):
    """One non-zero code per row, unit scales: every output is one int8
    product, exact in bf16, so any slip in the operand layouts (swizzle, K
    step, row or channel order, instance) shows up as a wrong value."""
    gi = gen.gmm_inputs(21, counts, H, N, spare_rows=spare, one_hot=True)
    got, err = _gpu(B, gi)
    o = _oracle(gi)
    assert err == 0 and o["err"] == 0
    np.testing.assert_array_equal(got, o["out"])


@pytest.mark.parametrize("H,N,counts,spare", [
    (1024, 128, [40, 0, 1, 129, 77], 3),
    (1168, 208, [5, 33, 0, 260], 2),
    (2048, 256, [128, 256, 255, 16, 15], 0),      # slot boundaries at 128 and 256 rows
    (1024, 128, [511, 512, 513, 257, 1], 2),      # 256-row slots (N = 256) and their remainders
    (7168, 384, [24, 9, 0, 140], 1),              # the decode hidden size
])
def test_gmm_parity_random(B, H, N, counts, spare):
    gi = gen.gmm_inputs(22, counts, H, N, spare_rows=spare)
    got, err = _gpu(B, gi)
    o = _oracle(gi)
    assert err == 0 and o["err"] == 0
    _assert_gmm_parity(got, o)


def test_gmm_parity_many_instances(B):
    """256 instances with ~16 rows each (a decode batch's shape) and some
    empty ones."""
    rng = np.random.default_rng(5)
    counts = rng.poisson(16, 256)
    counts[rng.integers(0, 256, 20)] = 0
    gi = gen.gmm_inputs(23, counts, 1024, 128)
    got, err = _gpu(B, gi)
    o = _oracle(gi)
    assert err == 0 and o["err"] == 0
    _assert_gmm_parity(got, o)


@pytest.mark.parametrize("off", [[0, 3, 2, 4], [0, 1, 2, 70], [-1, 1, 2, 3]])
def test_gmm_bad_offsets(B, off):
    """Offsets that decrease, overrun the rows or start below 0 set
    MOE_DEV_BAD_ID and nothing is written (as in the oracle)."""
    gi = gen.gmm_inputs(24, [2, 1, 1], 1024, 128, spare_rows=60)
    gi.offsets = np.array(off, np.int32)
    got, err = _gpu(B, gi)
    o = _oracle(gi)
    assert err == 1 and o["err"] == orc.ERR_BAD_ID
    assert np.all(got == POISON16)


def test_gmm_full_size_sampled(B):
    """256 instances x 7168 channels x H 7168 (13 GB of int8 weights), 4096
    rows as a Bs 512, K 8 decode batch spreads them: sampled rows and
    channels against the oracle, called on those slices."""
    E, H, N = 256, 7168, 7168
    rng = np.random.default_rng(6)
    counts = np.bincount(rng.integers(0, E, 4096), minlength=E)
    gi = gen.gmm_inputs(25, counts, H, 16)  # rows and row factors; the weights are drawn on the device
    w, ws = gen.gmm_weights_device(25, E, N, H, "cuda")
    got, err = _gpu(B, gi, weight=w, weight_scales=ws)
    assert err == 0
    off = gi.offsets
    inst = np.searchsorted(off, np.arange(off[-1]), side="right") - 1
    rows = rng.choice(int(off[-1]), 48, replace=False)
    chans = np.sort(rng.choice(N, 24, replace=False))
    ct = torch.from_numpy(chans).cuda()
    for r in rows:
        e = int(inst[r])
        sub = gen.GmmInputs(expand_x=gi.expand_x[r:r + 1], dyn_scales=gi.dyn_scales[r:r + 1],
                            offsets=np.array([0, 1], np.int32),
                            weight=w[e].index_select(0, ct).cpu().numpy()[None],
                            weight_scales=ws[e].index_select(0, ct).cpu().numpy()[None])
        o = orc.grouped_matmul(sub.expand_x, sub.dyn_scales, sub.offsets, sub.weight, sub.weight_scales)
        g = got[r, chans].astype(np.int32)
        assert np.all(np.abs(g - o["out"][0].astype(np.int32)) <= 1), f"row {r}"
    del w, ws
    torch.cuda.empty_cache()


def test_dispatch_gmm_combine_pipeline(B):
    """update_expert -> dispatch (per-token int8, smooth scales) -> grouped
    matmul (N = H) -> combine+Add+RMSNorm on the GPU, against the same chain
    of oracle calls."""
    w = gen.uniform_layer("pipe", 31, bs=64, hidden=1024, num_experts=16, top_k=4, ep_world_size=4,
                          quant_mode=2, smooth=True, shared=True)
    wt = gen.gmm_inputs(32, [0] * w.num_instances, w.hidden, w.hidden)
    # GPU chain
    ids, table, sc = dev(w.expert_ids), dev(w.table), dev(w.expert_scales)
    ws = B.new_workspace(nbytes=4096)
    bal = torch.empty_like(ids)
    bm = torch.empty(ids.shape, dtype=torch.uint8, device="cuda")
    B.update_expert(ids, table, w.ep_world_size, expert_scales=sc, workspace=ws, out=(bal, bm))
    d = B.alloc_dispatch_outputs(w.bs, w.hidden, w.top_k, w.num_instances, w.quant_mode)
    B.dispatch(dev_bf16(w.x), bal, w.num_instances, w.ep_world_size, w.quant_mode, mask=bm, smooth=dev(w.smooth),
               workspace=ws, out=d)
    rows = d["expand_x"].shape[0]
    ex = torch.zeros((rows, w.hidden), dtype=torch.bfloat16, device="cuda")
    B.grouped_matmul(d["expand_x"], d["dyn_scales"], d["offsets"], dev(wt.weight), dev(wt.weight_scales), out=ex,
                     workspace=B.new_workspace(nbytes=B.grouped_matmul_workspace_bytes(rows, w.hidden, w.hidden,
                                                                                       w.num_instances)))
    c = B.combine_add_rmsnorm(ex, d["expand_idx"], sc, dev_bf16(w.residual), dev_bf16(w.gamma), w.norm_eps,
                              shared_x=dev_bf16(w.shared_x), want_x_out=True, workspace=ws)
    torch.cuda.synchronize()
    assert B.read_device_error(ws) == 0
    # oracle chain
    bal_o, bm_o, e1 = orc.update_expert(w.expert_ids, w.table, w.ep_world_size, expert_scales=w.expert_scales)
    do = orc.dispatch(w.x, bal_o, w.num_instances, w.quant_mode, mask=bm_o, smooth=w.smooth)
    go = orc.grouped_matmul(do["expand_x"], do["dyn_scales"], do["offsets"], wt.weight, wt.weight_scales,
                            out=np.zeros((rows, w.hidden), np.uint16))
    co = orc.combine_add_rmsnorm(go["out"], do["expand_idx"], w.expert_scales, w.residual, w.gamma, w.norm_eps,
                                 shared_x=w.shared_x)
    assert e1 == 0 and do["err"] == 0 and go["err"] == 0
    n = do["n"]
    np.testing.assert_array_equal(host(d["offsets"]), do["offsets"])
    np.testing.assert_array_equal(host(d["expand_x"])[:n], do["expand_x"][:n])
    _assert_gmm_parity(host(ex)[:n], dict(out=go["out"][:n], out_f64=go["out_f64"][:n]))
    assert_close_bf16(host(c["y"]), co["y_f64"], what="y")
    assert_close_bf16(host(c["x_out"]), co["x_f64"], what="x_out")


# ------------------------------------------------------------------ mxfp8

def _at_offset(a, off):
    """a's bytes on the device starting `off` bytes into a larger buffer (a
    base that is 4-byte but not 16-byte aligned when off = 4)."""
    buf = torch.zeros(a.nbytes + 16, dtype=torch.uint8, device="cuda")
    t = buf[off:off + a.nbytes]
    t.copy_(torch.from_numpy(np.ascontiguousarray(a).reshape(-1).view(np.uint8)).cuda())
    return t.view(a.shape)


def _gpu_mx(B, gi, sf_offset=0):
    rows, H = gi.expand_x.shape
    E, N = gi.weight.shape[0], gi.weight.shape[1]
    out = poison_(torch.empty((rows, N), dtype=torch.bfloat16, device="cuda"))
    wsp = B.new_workspace(nbytes=B.grouped_matmul_workspace_bytes(rows, H, N, E))
    x_sf = dev(gi.x_sf) if sf_offset == 0 else _at_offset(gi.x_sf, sf_offset)
    w_sf = dev(gi.weight_sf) if sf_offset == 0 else _at_offset(gi.weight_sf, sf_offset)
    B.grouped_matmul_mx(dev(gi.expand_x), x_sf, dev(gi.offsets), dev(gi.weight), w_sf, out=out, workspace=wsp)
    torch.cuda.synchronize()
    return host(out), B.read_device_error(wsp)


def _oracle_mx(gi):
    rows, N = gi.expand_x.shape[0], gi.weight.shape[1]
    return orc.grouped_matmul_mx(gi.expand_x, gi.x_sf, gi.offsets, gi.weight, gi.weight_sf,
                                 out=np.full((rows, N), POISON16, np.uint16))


@pytest.mark.parametrize("H,N,counts,spare", [
    (1024, 256, [3, 0, 17, 130, 1, 128, 16], 5),   # factor rows of 32 B: 16-byte factor loads
    (1152, 208, [5, 33, 0, 260], 0),               # 36 B: four-byte factor loads
    (3072, 128, [64, 1, 31], 2),                   # 96 B: 16-byte loads, six groups of four steps
])
def test_gmm_mx_single_products_bit_exact(B, H, N, counts, spare):
    """One non-zero E4M3 code per row: every output is one product of two
    E4M3 values (at most 8 significant bits) times two powers of two, exact
    in bf16, so the operand layouts and the placement of every block factor
    are checked bit for bit."""
    gi = gen.gmm_inputs_mx(41, counts, H, N, spare_rows=spare, one_hot=True)
    got, err = _gpu_mx(B, gi)
    o = _oracle_mx(gi)
    assert err == 0 and o["err"] == 0
    np.testing.assert_array_equal(got, o["out"])


@pytest.mark.parametrize("H,N,counts,spare", [
    (1024, 128, [40, 0, 1, 129, 77], 3),
    (2048, 256, [128, 256, 255, 16, 15], 0),
    (7168, 384, [24, 9, 0, 140], 1),
])
def test_gmm_mx_parity_random(B, H, N, counts, spare):
    """Full-range E4M3 rows and weights with random block factors: within the
    1e-2 bar everywhere (the tensor cores sum in fp32, the oracle in
    binary64), and nearly all outputs within one bf16 step."""
    gi = gen.gmm_inputs_mx(42, counts, H, N, spare_rows=spare)
    got, err = _gpu_mx(B, gi)
    o = _oracle_mx(gi)
    assert err == 0 and o["err"] == 0
    written = ~np.isnan(o["out_f64"])
    np.testing.assert_array_equal(got[~written], o["out"][~written])
    rows = np.flatnonzero(written.any(axis=1))
    assert_close_bf16(got[rows], o["out_f64"][rows], what="mx gmm out")
    step = np.abs(got[written].astype(np.int32) - o["out"][written].astype(np.int32))
    assert (step <= 1).mean() >= 0.99


@pytest.mark.parametrize("H", [1024, 2048])
def test_gmm_mx_factor_alignment_paths_agree(B, H):
    """Factor arrays whose bases are 4- but not 16-byte aligned take the
    four-byte factor loads; the result is the same, bit for bit, as with
    16-byte aligned bases (the 16-byte loads), and both equal the oracle on
    single products."""
    gi = gen.gmm_inputs_mx(43, [7, 40, 0, 129], H, 128, spare_rows=2, one_hot=True)
    got16, err16 = _gpu_mx(B, gi)
    got4, err4 = _gpu_mx(B, gi, sf_offset=4)
    assert err16 == 0 and err4 == 0
    np.testing.assert_array_equal(got4, got16)
    np.testing.assert_array_equal(got16, _oracle_mx(gi)["out"])


def test_dispatch_mx_gmm_combine_pipeline(B):
    """update_expert -> dispatch (mxfp8) -> mxfp8 matmul (N = H) ->
    combine+Add+RMSNorm on the GPU, against the same chain of oracle calls."""
    w = gen.uniform_layer("pipe_mx", 33, bs=64, hidden=1024, num_experts=16, top_k=4, ep_world_size=4,
                          quant_mode=4, shared=True)
    wt = gen.gmm_inputs_mx(34, [0] * w.num_instances, w.hidden, w.hidden)
    ids, table, sc = dev(w.expert_ids), dev(w.table), dev(w.expert_scales)
    ws = B.new_workspace(nbytes=4096)
    bal = torch.empty_like(ids)
    bm = torch.empty(ids.shape, dtype=torch.uint8, device="cuda")
    B.update_expert(ids, table, w.ep_world_size, expert_scales=sc, workspace=ws, out=(bal, bm))
    d = B.alloc_dispatch_outputs(w.bs, w.hidden, w.top_k, w.num_instances, w.quant_mode)
    B.dispatch(dev_bf16(w.x), bal, w.num_instances, w.ep_world_size, w.quant_mode, mask=bm, workspace=ws, out=d)
    rows = d["expand_x"].shape[0]
    ex = torch.zeros((rows, w.hidden), dtype=torch.bfloat16, device="cuda")
    B.grouped_matmul_mx(d["expand_x"].view(torch.uint8), d["dyn_scales"].view(torch.uint8), d["offsets"],
                        dev(wt.weight), dev(wt.weight_sf), out=ex,
                        workspace=B.new_workspace(nbytes=B.grouped_matmul_workspace_bytes(rows, w.hidden, w.hidden,
                                                                                          w.num_instances)))
    c = B.combine_add_rmsnorm(ex, d["expand_idx"], sc, dev_bf16(w.residual), dev_bf16(w.gamma), w.norm_eps,
                              shared_x=dev_bf16(w.shared_x), want_x_out=True, workspace=ws)
    torch.cuda.synchronize()
    assert B.read_device_error(ws) == 0
    bal_o, bm_o, e1 = orc.update_expert(w.expert_ids, w.table, w.ep_world_size, expert_scales=w.expert_scales)
    do = orc.dispatch(w.x, bal_o, w.num_instances, w.quant_mode, mask=bm_o)
    go = orc.grouped_matmul_mx(do["expand_x"], do["dyn_scales"], do["offsets"], wt.weight, wt.weight_sf,
                               out=np.zeros((rows, w.hidden), np.uint16))
    co = orc.combine_add_rmsnorm(go["out"], do["expand_idx"], w.expert_scales, w.residual, w.gamma, w.norm_eps,
                                 shared_x=w.shared_x)
    assert e1 == 0 and do["err"] == 0 and go["err"] == 0
    n = do["n"]
    np.testing.assert_array_equal(host(d["expand_x"].view(torch.uint8))[:n], do["expand_x"][:n])
    np.testing.assert_array_equal(host(d["dyn_scales"].view(torch.uint8))[:n], do["dyn_scales"][:n])
    assert_close_bf16(host(ex)[:n], go["out_f64"][:n], what="mx gmm out")
    assert_close_bf16(host(c["y"]), co["y_f64"], what="y")


def test_gmm_one_rank_region(B):
    """One simulated rank runs its own L instances on its region of the
    receive buffer: the offsets are that rank's slice of the dispatch's
    offsets (the first one above 0), the weights its L instances'.  Rows of
    the other ranks are left untouched."""
    rng = np.random.default_rng(8)
    counts = rng.poisson(20, 32)
    gi = gen.gmm_inputs(26, counts, 1024, 256, spare_rows=3)
    L, r = 8, 2  # 4 ranks of 8 instances; rank 2
    sub = gen.GmmInputs(expand_x=gi.expand_x, dyn_scales=gi.dyn_scales,
                        offsets=np.ascontiguousarray(gi.offsets[r * L:(r + 1) * L + 1]),
                        weight=np.ascontiguousarray(gi.weight[r * L:(r + 1) * L]),
                        weight_scales=np.ascontiguousarray(gi.weight_scales[r * L:(r + 1) * L]))
    assert sub.offsets[0] > 0
    got, err = _gpu(B, sub)
    o = _oracle(sub)
    assert err == 0 and o["err"] == 0
    _assert_gmm_parity(got, o)
    lo, hi = sub.offsets[0], sub.offsets[-1]
    assert np.all(got[:lo] == POISON16) and np.all(got[hi:] == POISON16)
