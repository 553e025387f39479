"""Pins for the CPU oracle, against things other than itself.

Every check here is a hand-derived worked example (tests/golden/), a brute
force on tiny inputs, a closed form, an invariant the pages imply, or a
library routine that the special case reduces to.  None of them re-types the
oracle's own formula.  CPU only.
"""
import json
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

from combine_moe_update_b200 import inputs as gen

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")))


def bits(vals):
    return gen.bf16_bits(np.asarray(vals, np.float32))


# --------------------------------------------------------------------------
# update_expert (aclnnMoeUpdateExpert)
# --------------------------------------------------------------------------

def test_update_expert_worked_example(orc):
    g = GOLDEN["update_expert_small"]
    for case in g["cases"]:
        am = None if case["active_mask"] is None else np.array(case["active_mask"], np.uint8)
        bal, bm, err = orc.update_expert(np.array(g["expert_ids"]), np.array(g["table"]),
                                         g["ep_world_size"],
                                         expert_scales=np.array(g["expert_scales"], np.float32),
                                         active_mask=am, prune_threshold=case["prune_threshold"])
        assert err == 0
        np.testing.assert_array_equal(bal, g["balanced_ids"])
        np.testing.assert_array_equal(bm, case["balanced_mask"])


@pytest.mark.parametrize("E,ws", [(8, 4), (256, 32), (1024, 256), (64, 8), (12, 3)])
def test_update_expert_identity_table_is_identity(orc, E, ws):
    rng = np.random.default_rng(E)
    ids = gen.topk_uniform(rng, 40, E, min(8, E))
    bal, bm, err = orc.update_expert(ids, gen.identity_table(E, ws), ws)
    assert err == 0
    np.testing.assert_array_equal(bal, ids)
    assert bm.all()


def test_update_expert_replicated_table_invariants(orc):
    w = gen.make("skewed_eplb")
    bal, bm, err = orc.update_expert(w.expert_ids, w.table, w.ep_world_size)
    assert err == 0 and bm.all()
    N, ws = w.num_instances, w.ep_world_size
    L = N // ws
    # the map (e, j) -> instance is a bijection onto [0, N) with L instances per rank
    seen = {}
    for e in range(w.num_logical):
        n = w.table[e, 0]
        for j in range(n):
            ids = np.full((1, 1), e, np.int32)
            # token index i = j routes to replica j (i mod n_e)
            b, _, _ = orc.update_expert(np.repeat(ids, j + 1, axis=0), w.table, ws)
            inst = int(b[j, 0])
            assert inst // L == w.table[e, 1 + j], "instance must live on the table's rank"
            seen[(e, j)] = inst
    assert sorted(seen.values()) == list(range(N))
    # every copy lands on the rank the table names for replica i mod n_e
    i = np.arange(w.bs)[:, None]
    n_e = w.table[w.expert_ids, 0]
    want_rank = w.table[w.expert_ids, 1 + (i % n_e)]
    np.testing.assert_array_equal(bal // L, want_rank)
    # instances of one rank are ordered by (logical id, replica)
    for r in range(ws):
        pairs = sorted([p for p, v in seen.items() if v // L == r])
        assert [seen[p] for p in pairs] == list(range(r * L, (r + 1) * L))


@pytest.mark.parametrize("bad", ["zero_count", "rank_out_of_range", "uneven", "too_many_cols"])
def test_update_expert_bad_table_drops_everything(orc, bad):
    t = gen.identity_table(8, 4).copy()
    if bad == "zero_count":
        t[3, 0] = 0
    elif bad == "rank_out_of_range":
        t[5, 1] = 4
    elif bad == "uneven":
        t[0, 1] = 1           # rank 0 now has 1 instance, rank 1 has 3
    elif bad == "too_many_cols":
        t[2, 0] = 2           # n_e must be <= F - 1 = 1
    ids = np.array([[0, 1], [2, 3]], np.int32)
    bal, bm, err = orc.update_expert(ids, t, 4)
    assert err & orc.ERR_BAD_TABLE
    assert (bal == -1).all() and (bm == 0).all()


def test_update_expert_bad_id_drops_only_that_copy(orc):
    ids = np.array([[0, 9], [-1, 3]], np.int32)
    bal, bm, err = orc.update_expert(ids, gen.identity_table(8, 4), 4)
    assert err == orc.ERR_BAD_ID
    np.testing.assert_array_equal(bal, [[0, -1], [-1, 3]])
    np.testing.assert_array_equal(bm, [[1, 0], [0, 1]])


def test_update_expert_pruning_fraction_max_shape(orc):
    """Pruned exactly where the weight is strictly below the threshold."""
    w = gen.make("max_shape")
    _, bm, err = orc.update_expert(w.expert_ids, w.table, w.ep_world_size,
                                   expert_scales=w.expert_scales, prune_threshold=w.prune_threshold)
    assert err == 0
    np.testing.assert_array_equal(bm == 0, w.expert_scales < np.float32(w.prune_threshold))
    assert 0.3 < (bm == 0).mean() < 0.7


# --------------------------------------------------------------------------
# dispatch: routing / index part (aclnnMoeDistributeDispatchV2)
# --------------------------------------------------------------------------

def test_dispatch_index_worked_example(orc):
    g = GOLDEN["dispatch_index_small"]
    x = np.zeros((3, 8), np.uint16)
    for case in g["cases"]:
        m = None if case["mask"] is None else np.array(case["mask"], np.uint8)
        out = orc.dispatch(x, np.array(g["instance_ids"]), g["num_instances"], 0, mask=m)
        assert out["err"] == 0
        np.testing.assert_array_equal(out["expand_idx"], case["expand_idx"])
        np.testing.assert_array_equal(out["src_of_row"], case["src_of_row"])
        np.testing.assert_array_equal(out["counts"], case["counts"])
        np.testing.assert_array_equal(out["offsets"], case["offsets"])


def _brute_rows(ids, mask):
    """Row of an active copy = number of active copies with a smaller
    (instance, token, k) key; O(n^2), no sorting."""
    bs, K = ids.shape
    i, k = np.meshgrid(np.arange(bs), np.arange(K), indexing="ij")
    key = np.stack([ids.ravel(), i.ravel(), k.ravel()], 1).astype(np.int64)
    act = mask.ravel().astype(bool)
    a, b = key[:, None, :], key[None, :, :]
    less = (b[..., 0] < a[..., 0]) | ((b[..., 0] == a[..., 0]) & (
        (b[..., 1] < a[..., 1]) | ((b[..., 1] == a[..., 1]) & (b[..., 2] < a[..., 2]))))
    rows = (less & act[None, :]).sum(1)
    return np.where(act, rows, -1).reshape(bs, K)


@pytest.mark.parametrize("seed", range(12))
def test_dispatch_index_brute_force(orc, seed):
    rng = np.random.default_rng(100 + seed)
    bs, K = int(rng.integers(1, 24)), int(rng.integers(1, 5))
    E = int(rng.integers(K, 17))
    ids = rng.integers(0, E, size=(bs, K)).astype(np.int32)   # duplicates allowed
    mask = (rng.random((bs, K)) < 0.7).astype(np.uint8)
    out = orc.dispatch(np.zeros((bs, 8), np.uint16), ids, E, 0, mask=mask)
    np.testing.assert_array_equal(out["expand_idx"], _brute_rows(ids, mask))
    np.testing.assert_array_equal(out["counts"], np.bincount(ids[mask == 1], minlength=E))


@pytest.mark.parametrize("name", ["tiny", "deepseek_decode", "skewed_eplb", "max_shape"])
def test_dispatch_index_invariants(orc, name):
    w = gen.make(name)
    bal, bm, err = orc.update_expert(w.expert_ids, w.table, w.ep_world_size,
                                     expert_scales=w.expert_scales, prune_threshold=w.prune_threshold)
    out = orc.dispatch(w.x[:, :8].copy(), bal, w.num_instances, 0, mask=bm)
    idx, src, cnt, off, n = out["expand_idx"], out["src_of_row"], out["counts"], out["offsets"], out["n"]
    assert n == int(bm.sum()) == int(cnt.sum())
    if w.prune_threshold == 0:
        assert n == w.bs * w.top_k
    assert off[0] == 0 and off[-1] == n and (np.diff(off) == cnt).all()
    act = np.nonzero(bm.ravel())[0]
    np.testing.assert_array_equal(np.sort(idx.ravel()[act]), np.arange(n))
    np.testing.assert_array_equal(src[idx.ravel()[act]], act)
    assert (idx.ravel()[bm.ravel() == 0] == -1).all()
    # every bucket holds its instance's copies in increasing (token, k) order
    for e in range(w.num_instances):
        seg = src[off[e]:off[e + 1]]
        assert (np.diff(seg) > 0).all()
        assert (bal.ravel()[seg] == e).all()
    # rank r's region is the contiguous rows of instances [r L, (r+1) L)
    L = w.num_instances // w.ep_world_size
    rank_of_row = bal.ravel()[src] // L
    assert (np.diff(rank_of_row) >= 0).all()


def test_dispatch_bad_instance_id_dropped(orc):
    ids = np.array([[0, 5], [2, 3]], np.int32)
    out = orc.dispatch(np.zeros((2, 8), np.uint16), ids, 4, 0)
    assert out["err"] == orc.ERR_BAD_ID
    np.testing.assert_array_equal(out["expand_idx"], [[0, -1], [1, 2]])
    np.testing.assert_array_equal(out["counts"], [1, 0, 1, 1])


def test_dispatch_mode0_copies_rows(orc):
    w = gen.make("tiny")
    out = orc.dispatch(w.x, w.expert_ids, w.num_instances, 0)
    src = out["src_of_row"]
    np.testing.assert_array_equal(out["expand_x"][: out["n"]], w.x[src // w.top_k])


# --------------------------------------------------------------------------
# dispatch: int8 quantization (quantMode 2 / 3)
# --------------------------------------------------------------------------

def test_int8_worked_rows(orc):
    for row in GOLDEN["quant_int8_rows"]["rows"]:
        x = bits([row["x"]])
        sm = None if row["smooth"] is None else np.array([row["smooth"]], np.float32)
        out = orc.dispatch(x, np.zeros((1, 1), np.int32), 1, 2, smooth=sm)
        np.testing.assert_array_equal(out["expand_x"][0], row["q"])
        assert out["dyn_scales"][0] == np.float32(row["scale"])
        if "scale_bits" in row:
            assert int(out["dyn_scales"][:1].view(np.uint32)[0]) == int(row["scale_bits"], 16)


def test_sources_order_and_additivity(orc):
    """Several source ranks (READING R22): S * Bs tokens, rank-major.  Counts
    are the sums of each rank's own counts (dispatching every rank alone),
    and within each instance's rows the source rank, then the token, then k
    never decrease."""
    rng = np.random.default_rng(22)
    S, bs, K, E, H = 4, 6, 3, 8, 1024
    x = gen.bf16_bits(rng.standard_normal((S * bs, H), np.float32))
    ids = gen.topk_uniform(rng, S * bs, E, K)
    full = orc.dispatch(x, ids, E, 0)
    parts = [orc.dispatch(x[r * bs:(r + 1) * bs], ids[r * bs:(r + 1) * bs], E, 0) for r in range(S)]
    np.testing.assert_array_equal(full["counts"], sum(p["counts"] for p in parts))
    src = full["src_of_row"]
    for e in range(E):
        seg = src[full["offsets"][e]:full["offsets"][e + 1]]
        key = [(int(j) // K // bs, int(j) // K % bs, int(j) % K) for j in seg]
        assert key == sorted(key)
        assert all(ids[j // K, j % K] == e for j in seg)
    # each rank's rows of instance e are its own dispatch's rows of e, in order
    for e in range(E):
        seg = src[full["offsets"][e]:full["offsets"][e + 1]]
        for r in range(S):
            mine = [int(j) - r * bs * K for j in seg if int(j) // K // bs == r]
            p = parts[r]
            np.testing.assert_array_equal(mine, p["src_of_row"][p["offsets"][e]:p["offsets"][e + 1]])


def test_plain_combine_closed_form(orc):
    """The plain combine (READING R23) on rows with closed forms: expert row k
    is the constant c_k, the shared row the constant d, so every element is
    sum_k w_k (c_k + d); a pruned copy (-1) adds nothing; and it equals the
    Add+RMSNorm combine's x minus the residual."""
    H, K = 1024, 3
    c = [1.5, -2.0, 0.25]
    d = 0.5
    ex = np.stack([np.full(H, v, np.float32) for v in c])
    idx = np.array([[0, 1, 2], [2, -1, 0]], np.int32)
    w = np.array([[0.5, 0.25, 0.25], [0.125, 0.5, 0.375]], np.float32)
    sh = np.full((2, H), d, np.float32)
    out = orc.combine(bits(ex), idx, w, shared_x=bits(sh))
    want = [0.5 * (1.5 + d) + 0.25 * (-2.0 + d) + 0.25 * (0.25 + d), 0.125 * (0.25 + d) + 0.375 * (1.5 + d)]
    for i in range(2):
        assert np.all(out["out_f64"][i] == want[i])
    res = np.zeros((2, H), np.float32)
    full = orc.combine_add_rmsnorm(bits(ex), idx, w, bits(res), bits(np.ones(H, np.float32)), 1e-6,
                                   shared_x=bits(sh))
    np.testing.assert_array_equal(out["out_f64"], full["x_f64"])


def test_static_int8_worked_rows(orc):
    """quantMode 1 on hand-derived rows (scale (1,)): rounding half to even,
    saturation to [-128, 127], and the NaN of 0 * inf casting to 0."""
    for row in GOLDEN["quant_static_int8"]["rows"]:
        scale = np.float32(np.inf) if row["scale"] == "inf" else np.float32(row["scale"])
        out = orc.dispatch(bits([row["x"]]), np.zeros((1, 1), np.int32), 1, 1, smooth=np.array([scale]))
        np.testing.assert_array_equal(out["expand_x"][0], row["q"])
        assert out["dyn_scales"] is None


@pytest.mark.parametrize("shape", ["one", "per_column", "per_instance"])
def test_static_int8_matches_numpy_rint(orc, shape):
    """Every scale shape against numpy's own round-half-to-even and clip on
    the fp32 product, with the scale taken from the copy's destination
    instance for (E, H) scales."""
    rng = np.random.default_rng(21)
    bs, H, K, E = 9, 1024, 3, 5
    x = gen.bf16_bits(rng.standard_normal((bs, H), np.float32) * 40)
    ids = gen.topk_uniform(rng, bs, E, K)
    sc = {"one": np.array([1.7], np.float32), "per_column": rng.uniform(0.5, 3, H).astype(np.float32),
          "per_instance": rng.uniform(0.5, 3, (E, H)).astype(np.float32)}[shape]
    out = orc.dispatch(x, ids, E, 1, smooth=sc)
    xf = gen.bf16_to_f32(x).astype(np.float32)
    for r in range(out["n"]):
        j = out["src_of_row"][r]
        i, k = divmod(int(j), K)
        s = sc if shape != "per_instance" else sc[ids[i, k]]
        want = np.clip(np.rint((xf[i] * s).astype(np.float32)), -128, 127).astype(np.int8)
        np.testing.assert_array_equal(out["expand_x"][r], want)


def test_static_int8_needs_scales(orc):
    with pytest.raises(ValueError):
        orc.dispatch(bits([[1.0] * 1024]), np.zeros((1, 1), np.int32), 1, 1)


def test_int8_per_tile_worked(orc):
    """Tile t of a per-tile row behaves like a per-token row on its own
    128 elements: tile 0 = first worked row, tile 1 = second, last tile
    partial (H = 264 -> tiles of 128, 128, 8)."""
    rows = GOLDEN["quant_int8_rows"]["rows"]
    H = 264
    x = np.zeros(H, np.float32)
    x[0:8] = rows[0]["x"]
    x[128:136] = rows[1]["x"]
    x[256:264] = rows[2]["x"]
    out = orc.dispatch(bits([x]), np.zeros((1, 1), np.int32), 1, 3)
    q, s = out["expand_x"][0], out["dyn_scales"][0]
    assert s.shape == (3,)
    np.testing.assert_array_equal(q[0:8], rows[0]["q"])
    np.testing.assert_array_equal(q[128:136], rows[1]["q"])
    assert s[0] == 1.0 and s[1] == 2.0
    # third tile: amax 127 with no smooth -> codes = x rounded, scale 1
    np.testing.assert_array_equal(q[256:264], np.rint(np.array(rows[2]["x"], np.float64)))
    assert s[2] == 1.0
    assert not q[8:128].any() and not q[136:256].any()


def _f32(xbits):
    return gen.bf16_to_f32(xbits).astype(np.float32)


@pytest.mark.parametrize("mode", [2, 3])
def test_int8_error_bound_and_extremes(orc, mode):
    """Spec bound: |q * scale - xFp32| <= amax / 254 (half a step);
    the largest element maps to +-127; codes in [-127, 127]; codes are
    monotone in xFp32."""
    w = gen.make("deepseek_decode", bs=24)
    w.x[3] = 0   # one all-zero token
    out = orc.dispatch(w.x, w.expert_ids, w.num_instances, mode, smooth=w.smooth)
    q = out["expand_x"].astype(np.float64)
    src = out["src_of_row"]
    inst = w.expert_ids.ravel()[src]
    xf = (_f32(w.x)[src // w.top_k] * w.smooth[inst]).astype(np.float64)  # exact product in f64
    n, H = len(src), w.hidden
    seg = H if mode == 2 else 128
    nt = (H + seg - 1) // seg
    sc = out["dyn_scales"].reshape(n, nt).astype(np.float64)
    assert (np.abs(q[:n]) <= 127).all()
    for t in range(nt):
        xs, qs = xf[:, t * seg:(t + 1) * seg], q[:n, t * seg:(t + 1) * seg]
        # the fp32 product differs from the f64 one by at most half an ulp
        amax = np.abs(xs).max(1)
        err = np.abs(qs * sc[:, t:t + 1] - xs).max(1)
        assert (err <= amax / 254 * (1 + 2 ** -16) + 1e-30).all()
        nz = amax > 0
        j = np.abs(xs).argmax(1)
        np.testing.assert_array_equal(np.abs(qs[np.arange(n), j])[nz], 127)
        assert (qs[~nz] == 0).all() and (sc[~nz, t] == 0).all()
        o = np.argsort(xs, axis=1)
        assert (np.diff(np.take_along_axis(qs, o, 1), axis=1) >= 0).all()


def test_int8_smooth_power_of_two_scales_only_the_scale(orc):
    """A power-of-two smooth row 2^p (one per instance) leaves every code as
    it is and multiplies the sent scale by exactly 2^p; this pins that the
    smooth row is picked by the destination instance (reading R9)."""
    w = gen.make("deepseek_decode", bs=16)
    p = (np.arange(w.num_instances) % 7) - 3
    smooth = np.repeat((2.0 ** p)[:, None], w.hidden, 1).astype(np.float32)
    base = orc.dispatch(w.x, w.expert_ids, w.num_instances, 2)
    sm = orc.dispatch(w.x, w.expert_ids, w.num_instances, 2, smooth=smooth)
    np.testing.assert_array_equal(base["expand_x"], sm["expand_x"])
    inst = w.expert_ids.ravel()[base["src_of_row"]]
    np.testing.assert_array_equal(sm["dyn_scales"][: base["n"]],
                                  base["dyn_scales"][: base["n"]] * (2.0 ** p[inst]).astype(np.float32))
    ones = orc.dispatch(w.x, w.expert_ids, w.num_instances, 3, smooth=np.ones_like(smooth))
    none = orc.dispatch(w.x, w.expert_ids, w.num_instances, 3)
    np.testing.assert_array_equal(ones["expand_x"], none["expand_x"])
    np.testing.assert_array_equal(ones["dyn_scales"], none["dyn_scales"])


def test_int8_single_tile_equals_per_token(orc):
    w = gen.make("deepseek_decode", bs=8)
    x = w.x[:, :128].copy()
    a = orc.dispatch(x, w.expert_ids, w.num_instances, 2, smooth=w.smooth[:, :128].copy())
    b = orc.dispatch(x, w.expert_ids, w.num_instances, 3, smooth=w.smooth[:, :128].copy())
    np.testing.assert_array_equal(a["expand_x"], b["expand_x"])
    np.testing.assert_array_equal(a["dyn_scales"], b["dyn_scales"][:, 0])


# --------------------------------------------------------------------------
# dispatch: mxfp8 (quantMode 4) and the e4m3 encoder
# --------------------------------------------------------------------------

def e4m3_decode(c):
    """OCP FP8 E4M3 decode from the format definition (bias 7, no inf,
    S.1111.111 = NaN)."""
    c = int(c)
    s = -1.0 if c & 0x80 else 1.0
    e, m = (c >> 3) & 0xF, c & 7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return s * m * 2.0 ** -9
    return s * (1 + m / 8) * 2.0 ** (e - 7)


DEC = np.array([e4m3_decode(c) for c in range(256)])


def test_e4m3_roundtrip_all_codes(orc):
    for c in range(256):
        v = DEC[c]
        if math.isnan(v):
            continue
        assert orc.e4m3_encode(np.float32(v)) == c, hex(c)


def test_e4m3_against_library_all_bf16(orc):
    """All 65536 bf16 values: below 464 the result equals ml_dtypes' and
    torch's float8_e4m3fn cast (round to nearest even); at or above it, the
    oracle saturates to +-448 where those libraries give NaN."""
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    v = gen.bf16_to_f32(b)
    fin = np.isfinite(v)
    got = orc.e4m3_encode(v[fin])
    lib = v[fin].astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    tch = torch.from_numpy(v[fin].copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    small = np.abs(v[fin]) < 464
    np.testing.assert_array_equal(got[small], lib[small])
    np.testing.assert_array_equal(got[small], tch[small])
    big = ~small
    np.testing.assert_array_equal(got[big], np.where(np.signbit(v[fin][big]), 0xFE, 0x7E))


def test_e4m3_brute_force_nearest(orc):
    """Random fp32 values and every exact midpoint between neighbouring
    codes: the code is the nearest finite value, ties to the even code."""
    rng = np.random.default_rng(7)
    mag = 2.0 ** rng.uniform(-13, 9.2, 3000)
    vals = (mag * rng.choice([-1, 1], 3000)).astype(np.float32)
    pos = np.sort(DEC[np.isfinite(DEC) & (DEC >= 0)])
    mids = ((pos[1:] + pos[:-1]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, -mids])
    got = orc.e4m3_encode(vals)
    finite_codes = np.array([c for c in range(256) if not math.isnan(DEC[c])])
    for v, g in zip(vals, got):
        if abs(v) >= 448:
            assert DEC[g] == math.copysign(448.0, v)
            continue
        d = np.abs(DEC[finite_codes] - float(v))
        best = finite_codes[d == d.min()]
        if len(best) > 1:   # a tie: the code with an even mantissa (for 0: the sign of v)
            best = [c for c in best if (c & 1) == 0 and (DEC[c] != 0 or (c >> 7) == np.signbit(v))]
        assert g == best[0], (v, g, best)


def test_mxfp8_worked_blocks(orc):
    for blk in GOLDEN["quant_mxfp8_blocks"]["blocks"]:
        x = np.zeros(32, np.float32)
        x[: len(blk["x_head"])] = blk["x_head"]
        out = orc.dispatch(bits([x]), np.zeros((1, 1), np.int32), 1, 4)
        assert out["dyn_scales"][0, 0] == blk["scale_byte"]
        np.testing.assert_array_equal(out["expand_x"][0, : len(blk["q_head"])], blk["q_head"])


def test_mxfp8_block_invariants(orc):
    w = gen.make("skewed_eplb", bs=32)
    out = orc.dispatch(w.x, w.expert_ids, w.num_instances, 4)
    n, H = out["n"], w.hidden
    x = gen.bf16_to_f32(w.x)[out["src_of_row"] // w.top_k].astype(np.float64).reshape(n, H // 32, 32)
    se = out["dyn_scales"][:n].astype(np.int64) - 127
    amax = np.abs(x).max(2)
    r = amax * 2.0 ** (-se)
    assert ((r >= 256) & (r < 512)).all()      # floor(log2 amax) - 8 exactly
    deq = DEC[out["expand_x"][:n].reshape(n, H // 32, 32)] * 2.0 ** se[..., None]
    v = np.abs(x) * 2.0 ** (-se[..., None])
    sat = v >= 448
    np.testing.assert_array_equal(np.abs(deq[sat]), (448 * 2.0 ** se[..., None] * np.ones_like(x))[sat])
    norm = (v >= 2 ** -6) & ~sat
    assert (np.abs(deq[norm] - x[norm]) <= np.abs(x[norm]) * 2 ** -4).all()
    sub = v < 2 ** -6
    assert (np.abs(deq - x)[sub] <= (2.0 ** -10 * 2.0 ** se[..., None] * np.ones_like(x))[sub]).all()
    assert sat.any()   # the x20 outliers do saturate somewhere


# --------------------------------------------------------------------------
# combine + Add + RMSNorm (aclnnMoeDistributeCombineAddRmsNorm)
# --------------------------------------------------------------------------

def test_bf16_rounding_against_library(orc):
    rng = np.random.default_rng(3)
    f = (rng.standard_normal(20000) * 2.0 ** rng.integers(-30, 30, 20000)).astype(np.float32)
    np.testing.assert_array_equal(orc.bf16_from_double(f.astype(np.float64)),
                                  f.astype(ml_dtypes.bfloat16).view(np.uint16))
    # exact midpoints go to the even neighbour; a hair above goes up
    lo = np.array([1.0, 1.0078125, 3.0, -5.0], np.float64)      # bf16 values; ulp 2^-7 * 2^e
    ulp = np.array([2 ** -7, 2 ** -7, 2 ** -6, 2 ** -5])
    mid = lo + np.sign(lo) * ulp / 2
    up = gen.bf16_bits((lo + np.sign(lo) * ulp).astype(np.float32))
    lob = gen.bf16_bits(lo.astype(np.float32))
    even = np.where((lob & 1) == 0, lob, up)
    np.testing.assert_array_equal(orc.bf16_from_double(mid), even)
    np.testing.assert_array_equal(orc.bf16_from_double(mid + np.sign(lo) * ulp * 2 ** -30), up)


def test_combine_constant_row_closed_form(orc):
    g = GOLDEN["combine_constant_row"]
    H = g["hidden"]
    ex = bits(np.full((1, H), g["expert_value"]))
    res = bits(np.full((1, H), g["residual_value"]))
    gam = bits(np.full(H, g["gamma_value"]))
    out = orc.combine_add_rmsnorm(ex, np.zeros((1, 1), np.int32), np.ones((1, 1), np.float32),
                                  res, gam, g["norm_eps"])
    c = g["expert_value"] + g["residual_value"]
    want = c / math.sqrt(c * c + g["norm_eps"]) * g["gamma_value"]
    np.testing.assert_allclose(out["y_f64"], want, rtol=1e-14)
    assert out["rstd"][0] == np.float32(1 / math.sqrt(c * c + g["norm_eps"]))


def _rms_norm_lib(x, gamma, eps):
    t = torch.from_numpy(np.asarray(x, np.float64))
    return torch.nn.functional.rms_norm(t, (t.shape[-1],), torch.from_numpy(gamma), eps).numpy()


def test_combine_single_expert_is_rmsnorm(orc):
    """K = 1, weight 1, zero residual, no shared expert: y = RMSNorm(row)."""
    w = gen.make("deepseek_decode", bs=6)
    rows = w.expert_out[:6]
    idx = np.arange(6, dtype=np.int32)[:, None]
    out = orc.combine_add_rmsnorm(rows, idx, np.ones((6, 1), np.float32), np.zeros_like(w.residual),
                                  w.gamma, 1e-6)
    g = gen.bf16_to_f32(w.gamma).astype(np.float64)
    np.testing.assert_allclose(out["y_f64"], _rms_norm_lib(gen.bf16_to_f32(rows), g, 1e-6),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("name", ["tiny", "deepseek_decode_bs512_bf16"])
def test_identity_expert_invariant(orc, name):
    """quantMode 0, identity experts, weights summing to 1, no shared
    expert: dispatch then combine returns RMSNorm(x + residual)."""
    w = gen.make(name, bs=16)
    d = orc.dispatch(w.x, w.expert_ids, w.num_instances, 0)
    out = orc.combine_add_rmsnorm(d["expand_x"], d["expand_idx"], w.expert_scales, w.residual,
                                  w.gamma, w.norm_eps)
    x = gen.bf16_to_f32(w.x).astype(np.float64) + gen.bf16_to_f32(w.residual)
    want = _rms_norm_lib(x, gen.bf16_to_f32(w.gamma).astype(np.float64), w.norm_eps)
    np.testing.assert_allclose(out["y_f64"], want, rtol=0, atol=1e-5)


def test_combine_linear_in_scales_and_prune_skips(orc):
    w = gen.make("deepseek_decode", bs=8)
    d = orc.dispatch(w.x, w.expert_ids, w.num_instances, 0)
    zero = np.zeros_like(w.residual)
    s1 = (np.round(w.expert_scales * 64) / 64).astype(np.float32)  # dyadic: s1 + s2 is exact
    s2 = np.roll(s1, 1, axis=1)
    run = lambda s, idx=d["expand_idx"], sh=None: orc.combine_add_rmsnorm(
        d["expand_x"], idx, s, zero, w.gamma, 1e-6, shared_x=sh)["x_f64"]
    np.testing.assert_allclose(run(2 * s1), 2 * run(s1), rtol=1e-15)
    np.testing.assert_allclose(run(s1 + s2), run(s1) + run(s2), rtol=1e-12, atol=1e-12)
    # a pruned copy (row -1) contributes exactly what a zero weight does
    idx = d["expand_idx"].copy()
    idx[:, 3] = -1
    s0 = s1.copy()
    s0[:, 3] = 0
    np.testing.assert_array_equal(run(s1, idx), run(s0))


def test_combine_shared_expert_weighting(orc):
    """Reading R5: Sum_k(s_k * ata_k + s_k * shared) weights the shared row by
    the sum of the kept weights (1 when no copy is pruned)."""
    w = gen.make("deepseek_decode", bs=4)
    K = w.top_k
    zero_rows = np.zeros((4 * K, w.hidden), np.uint16)
    idx = np.arange(4 * K, dtype=np.int32).reshape(4, K)
    idx[1, :3] = -1
    s = np.full((4, K), 0.125, np.float32)
    out = orc.combine_add_rmsnorm(zero_rows, idx, s, np.zeros_like(w.residual), w.gamma, 1e-6,
                                  shared_x=w.shared_x)
    sh = gen.bf16_to_f32(w.shared_x).astype(np.float64)
    np.testing.assert_array_equal(out["x_f64"][0], sh[0])            # 8 * 0.125 = 1
    np.testing.assert_array_equal(out["x_f64"][1], sh[1] * 0.625)    # 5 kept copies


# --------------------------------------------------------------------------
# grouped matmul between dispatch and combine (reading R24)
# --------------------------------------------------------------------------

def _gmm_inputs(rng, counts, H, N, lo, hi, spare=2):
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(off[-1]) + spare
    q = rng.integers(lo, hi, (rows, H), dtype=np.int8, endpoint=True)
    w = rng.integers(lo, hi, (len(counts), N, H), dtype=np.int8, endpoint=True)
    return off, q, w


def test_grouped_matmul_small_integers_equal_numpy_matmul(orc):
    """Unit scales and |acc| <= 144: every output is an integer that bf16 holds
    exactly, so each instance's block must equal numpy's integer matmul of its
    rows with its own weight, bit for bit; empty instances are skipped and
    rows past the last offset keep their content."""
    rng = np.random.default_rng(11)
    counts = [3, 0, 5, 1, 0, 4]
    H, N = 16, 24
    off, q, w = _gmm_inputs(rng, counts, H, N, -3, 3)
    E, rows = len(counts), q.shape[0]
    sentinel = np.full((rows, N), 0x7FC1, np.uint16)
    r = orc.grouped_matmul(q, np.ones(rows, np.float32), off, w, np.ones((E, N), np.float32), out=sentinel)
    assert r["err"] == 0
    for e in range(E):
        blk = q[off[e]:off[e + 1]].astype(np.int64) @ w[e].astype(np.int64).T
        assert np.abs(blk).max(initial=0) <= 144
        want = blk.astype(np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)
        np.testing.assert_array_equal(r["out"][off[e]:off[e + 1]], want)
    np.testing.assert_array_equal(r["out"][off[-1]:], sentinel[off[-1]:])


def test_grouped_matmul_scaled_against_numpy(orc):
    """Full-range codes and weights with random row and channel scales: the
    f64 result is numpy's int64 matmul times the two scales (exact integers
    below 2^53, so only the two products round), and the bf16 output is that
    value rounded by ml_dtypes."""
    rng = np.random.default_rng(12)
    counts = [7, 2, 0, 9]
    H, N = 64, 32
    off, q, w = _gmm_inputs(rng, counts, H, N, -128, 127)
    E, rows = len(counts), q.shape[0]
    ds = rng.uniform(1e-3, 2e-2, rows).astype(np.float32)
    ws = rng.uniform(1e-3, 1e-2, (E, N)).astype(np.float32)
    r = orc.grouped_matmul(q, ds, off, w, ws)
    assert r["err"] == 0
    for e in range(E):
        s = slice(off[e], off[e + 1])
        acc = q[s].astype(np.int64) @ w[e].astype(np.int64).T
        want = acc.astype(np.float64) * ds[s].astype(np.float64)[:, None] * ws[e].astype(np.float64)[None, :]
        np.testing.assert_allclose(r["out_f64"][s], want, rtol=1e-15, atol=0)
        np.testing.assert_array_equal(r["out"][s], want.astype(ml_dtypes.bfloat16).view(np.uint16))


def test_grouped_matmul_extreme_magnitude_closed_form(orc):
    """H = 8192 with every code 127 and every weight -128 (instance 0) or 127
    (instance 1): acc = -127*128*8192 = -133169152 and 127*127*8192 =
    132128768.  With dyn = 2^-7 and weight scale 2^-10 the outputs are
    -1016 exactly and 1008.0078125, which bf16 (spacing 4 in [512, 1024))
    rounds to 1008."""
    H, N = 8192, 2
    q = np.full((3, H), 127, np.int8)
    w = np.stack([np.full((N, H), -128, np.int8), np.full((N, H), 127, np.int8)])
    off = np.array([0, 2, 3], np.int32)
    r = orc.grouped_matmul(q, np.full(3, 2.0 ** -7, np.float32), off, w, np.full((2, N), 2.0 ** -10, np.float32))
    assert r["err"] == 0
    np.testing.assert_array_equal(r["out_f64"][:2], -1016.0)
    np.testing.assert_array_equal(r["out_f64"][2], 132128768 * 2.0 ** -17)
    np.testing.assert_array_equal(r["out"][:2], bits([-1016.0])[0])
    np.testing.assert_array_equal(r["out"][2], bits([1008.0])[0])


def test_grouped_matmul_identity_weight_dequantizes(orc):
    """An identity weight (N = H, unit channel scales) turns the matmul into
    the dispatch's dequantization: out[r][h] = q[r][h] * dyn[r]."""
    rng = np.random.default_rng(13)
    H = 48
    q = rng.integers(-127, 127, (9, H), dtype=np.int8, endpoint=True)
    ds = rng.uniform(1e-3, 1.0, 9).astype(np.float32)
    eye = np.eye(H, dtype=np.int8)
    r = orc.grouped_matmul(q, ds, np.array([0, 4, 9], np.int32), np.stack([eye, eye]), np.ones((2, H), np.float32))
    assert r["err"] == 0
    want = q.astype(np.float64) * ds.astype(np.float64)[:, None]
    np.testing.assert_array_equal(r["out_f64"], want)
    np.testing.assert_array_equal(r["out"], want.astype(ml_dtypes.bfloat16).view(np.uint16))


@pytest.mark.parametrize("off", [[0, 3, 2, 4], [0, 1, 2, 6], [-1, 1, 2, 3]])
def test_grouped_matmul_rejects_bad_offsets(orc, off):
    """Offsets that decrease, overrun the rows (5 here) or start below 0 are an
    error and nothing is written."""
    q = np.ones((5, 16), np.int8)
    pre = np.full((5, 16), 0x1234, np.uint16)
    r = orc.grouped_matmul(q, np.ones(5, np.float32), np.array(off, np.int32), np.ones((3, 16, 16), np.int8),
                           np.ones((3, 16), np.float32), out=pre)
    assert r["err"] == orc.ERR_BAD_ID
    np.testing.assert_array_equal(r["out"], pre)


def test_e4m3_decode_against_library(orc):
    """All 256 E4M3 codes against ml_dtypes' float8_e4m3fn."""
    codes = np.arange(256, dtype=np.uint8)
    want = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    got = orc.e4m3_decode(codes)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(want[ok]))


def _mx_dequant(codes, sf):
    v = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return np.ldexp(v, np.repeat(sf.astype(np.int64) - 127, 32, axis=-1))


def test_grouped_matmul_mx_against_numpy(orc):
    """mxfp8 rows and weights dequantized by ml_dtypes and np.ldexp, then
    numpy's matmul per instance: the products are exact in binary64, so only
    the summation order differs."""
    counts = [5, 0, 9, 3]
    H, N = 128, 48
    gi = gen.gmm_inputs_mx(14, counts, H, N, spare_rows=1)
    r = orc.grouped_matmul_mx(gi.expand_x, gi.x_sf, gi.offsets, gi.weight, gi.weight_sf)
    assert r["err"] == 0
    off = gi.offsets
    for e in range(len(counts)):
        s = slice(off[e], off[e + 1])
        want = _mx_dequant(gi.expand_x[s], gi.x_sf[s]) @ _mx_dequant(gi.weight[e], gi.weight_sf[e]).T
        np.testing.assert_allclose(r["out_f64"][s], want, rtol=1e-12, atol=1e-300)
    assert np.isnan(r["out_f64"][off[-1]:]).all()
    np.testing.assert_array_equal(r["out"][:off[-1]],
                                  r["out_f64"][:off[-1]].astype(ml_dtypes.bfloat16).view(np.uint16))


def test_grouped_matmul_mx_block_factors_closed_form(orc):
    """Codes all 1.0 (0x38): block j contributes 32 * 2^(a_j + b_j) with
    row factor 2^a_j and weight factor 2^b_j, so the output is
    32 * Sum_j 2^(a_j + b_j); a single factor moved by one doubles only its
    own block's share."""
    H, N = 128, 2
    x = np.full((1, H), 0x38, np.uint8)
    w = np.full((1, N, H), 0x38, np.uint8)
    xs = np.array([[127, 128, 126, 130]], np.uint8)   # a = 0, 1, -1, 3
    ws = np.array([[[127, 127, 129, 120], [127, 127, 127, 127]]], np.uint8)  # b = (0, 0, 2, -7), 0
    r = orc.grouped_matmul_mx(x, xs, np.array([0, 1], np.int32), w, ws)
    assert r["err"] == 0
    assert r["out_f64"][0, 0] == 32 * (1 + 2 + 2.0 ** 1 + 2.0 ** -4)
    assert r["out_f64"][0, 1] == 32 * (1 + 2 + 0.5 + 8)


# --------------------------------------------------------------------------
# TP domain of two ranks (READING R26)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("mode,smooth", [(0, False), (2, True), (3, False), (4, False)])
def test_tp_dispatch_is_the_tp_major_multi_source_order(orc, mode, smooth):
    """Each TP domain's AllToAllV followed by the pair's AllGatherV (the
    pages' two steps, done separately) gives, with one instance per rank,
    the same rows as one dispatch of all 2 * ws * Bs tokens numbered
    TP-major; tp_counts are the per-domain counts by brute force."""
    rng = np.random.default_rng(26)
    ws, bs, K, H = 8, 5, 3, 1024
    E, T = ws, 2 * ws * bs
    x = gen.bf16_bits(rng.standard_normal((T, H), np.float32))
    ids = gen.topk_uniform(rng, T, E, K)
    mask = (rng.random((T, K)) > 0.2).astype(np.uint8)
    sm = rng.uniform(0.5, 2.0, size=(E, H)).astype(np.float32) if smooth else None
    tp = orc.dispatch_tp(x, ids, E, mode, ws, bs, mask=mask, smooth=sm)
    one = orc.dispatch(x, ids, E, mode, mask=mask, smooth=sm)
    assert tp["err"] == 0 and one["err"] == 0
    n = one["n"]
    assert tp["n"] == n
    for key in ("expand_idx", "counts", "offsets", "src_of_row"):
        np.testing.assert_array_equal(tp[key], one[key])
    np.testing.assert_array_equal(tp["expand_x"][:n], one["expand_x"][:n])
    if one["dyn_scales"] is not None:
        np.testing.assert_array_equal(tp["dyn_scales"][:n], one["dyn_scales"][:n])
    for t in range(2):
        dom = slice(t * ws * bs, (t + 1) * ws * bs)
        for e in range(E):
            assert tp["tp_counts"][e, t] == int(((ids[dom] == e) & (mask[dom] != 0)).sum())


def test_tp_reduce_against_ml_dtypes(orc):
    """ReduceScatterV's bf16 result: the exact sum of two bf16 values
    (exact in binary64) rounded by ml_dtypes' bfloat16 cast; includes exact
    ties (1 + 2^-8 -> 1, (1 + 2^-7) + 2^-8 -> 1 + 2^-6), a partial of zero,
    and swapped operands."""
    rng = np.random.default_rng(126)
    a = gen.bf16_bits(rng.standard_normal(4096, np.float32) * np.exp2(rng.integers(-20, 20, 4096)))
    b = gen.bf16_bits(rng.standard_normal(4096, np.float32) * np.exp2(rng.integers(-20, 20, 4096)))
    ties = bits([1.0, 1.0 + 2.0 ** -7, -1.0])
    tie_b = bits([2.0 ** -8, 2.0 ** -8, -(2.0 ** -8)])
    a, b = np.concatenate([a, ties]), np.concatenate([b, tie_b])
    got = orc.tp_reduce(a, b)
    f = lambda u: (u.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    want = (f(a) + f(b)).astype(ml_dtypes.bfloat16).view(np.uint16)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(got[-3:], bits([1.0, 1.0 + 2.0 ** -6, -1.0]))
    np.testing.assert_array_equal(orc.tp_reduce(b, a), got)
    nz = f(a) != 0
    np.testing.assert_array_equal(orc.tp_reduce(a, np.zeros_like(a))[nz], a[nz])


def test_tp_combine_closed_forms(orc):
    """With one partial zero the TP combine is the combine of the other;
    with two equal partials of exactly representable doubles it is the
    combine of the doubled rows."""
    rng = np.random.default_rng(226)
    bs, K, H, rows = 6, 3, 1024, 18
    p0 = gen.bf16_bits(rng.standard_normal((rows, H), np.float32))
    idx = rng.permutation(rows).reshape(bs, K).astype(np.int32)
    idx[0, 1] = -1
    w = rng.random((bs, K)).astype(np.float32)
    res = gen.bf16_bits(rng.standard_normal((bs, H), np.float32))
    g = gen.bf16_bits(rng.uniform(0.5, 1.5, H).astype(np.float32))
    a = orc.combine_add_rmsnorm_tp(p0, np.zeros_like(p0), idx, w, res, g, 1e-6)
    b = orc.combine_add_rmsnorm(p0, idx, w, res, g, 1e-6)
    np.testing.assert_array_equal(a["y"], b["y"])
    f = (p0.astype(np.uint32) << 16).view(np.float32)
    doubled = gen.bf16_bits(f * 2.0)  # exact: a power-of-two scale
    c = orc.combine_add_rmsnorm_tp(p0, p0, idx, w, res, g, 1e-6)
    d = orc.combine_add_rmsnorm(doubled, idx, w, res, g, 1e-6)
    np.testing.assert_array_equal(c["y"], d["y"])
