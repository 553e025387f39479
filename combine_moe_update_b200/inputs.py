"""Seeded synthetic workloads for the MoE update-expert / dispatch / combine path.

This module only draws inputs: it holds none of the operators' arithmetic,
and both the CUDA path and the CPU oracle are fed from it.  Every array is
numpy; bf16 tensors are returned as ``uint16`` bit patterns (fp32 draws
rounded to nearest even), everything else in its natural dtype.

Workloads follow the shapes and limits of the operator pages
(aclnnMoeUpdateExpert, aclnnMoeDistributeDispatchV2,
aclnnMoeDistributeCombineAddRmsNorm): Bs <= 512, H in [1024, 8192],
K <= 16, at most 1024 experts / instances.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np


def bf16_bits(a) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_to_f32(b) -> np.ndarray:
    """bf16 bit patterns -> fp32 values (exact)."""
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Workload:
    """One MoE layer's inputs.  Shapes: x/residual/shared [bs, H] bf16 bits;
    expert_ids [bs, K] logical ids; table [num_logical, F]; expert_scales
    [bs, K] f32; smooth [num_instances, H] f32 or None; expert_out
    [bs*K, H] bf16 bits (the stand-in for the expert FFN's output rows)."""
    name: str
    bs: int
    hidden: int
    top_k: int
    num_logical: int
    num_instances: int
    ep_world_size: int
    quant_mode: int
    x: np.ndarray
    expert_ids: np.ndarray
    expert_scales: np.ndarray
    table: np.ndarray
    residual: np.ndarray
    gamma: np.ndarray
    norm_eps: float
    prune_threshold: float = 0.0
    active_mask: Optional[np.ndarray] = None
    smooth: Optional[np.ndarray] = None
    shared_x: Optional[np.ndarray] = None
    expert_out: Optional[np.ndarray] = None
    meta: dict = field(default_factory=dict)


def identity_table(num_experts: int, ep_world_size: int) -> np.ndarray:
    """One instance per logical expert, expert e on rank e // L: the mapping
    is then the identity (instance id == logical id)."""
    L = num_experts // ep_world_size
    t = np.empty((num_experts, 2), np.int32)
    t[:, 0] = 1
    t[:, 1] = np.arange(num_experts) // L
    return t


def replicated_table(rng, num_logical, replicas, ep_world_size):
    """Table with ``replicas[e]`` instances of expert e, placed on ranks by a
    seeded permutation of the rank slots, re-drawn until no two instances of
    one expert share a rank.  Columns past n_e are padded with -1."""
    replicas = np.asarray(replicas, np.int64)
    total = int(replicas.sum())
    assert total % ep_world_size == 0
    L = total // ep_world_size
    F = int(replicas.max()) + 1
    owners = np.repeat(np.arange(num_logical), replicas)
    for _ in range(10000):
        slot_rank = rng.permutation(total) // L
        ok = True
        for e in np.nonzero(replicas > 1)[0]:
            r = slot_rank[owners == e]
            if len(np.unique(r)) != len(r):
                ok = False
                break
        if ok:
            break
    else:  # pragma: no cover
        raise RuntimeError("could not place replicas")
    t = np.full((num_logical, F), -1, np.int32)
    t[:, 0] = replicas
    fill = np.zeros(num_logical, np.int64)
    for s in range(total):
        e = owners[s]
        t[e, 1 + fill[e]] = slot_rank[s]
        fill[e] += 1
    return t


def topk_uniform(rng, bs, num_experts, k):
    """K distinct expert ids per token, uniform without replacement."""
    return np.argsort(rng.random((bs, num_experts)), axis=1)[:, :k].astype(np.int32)


def topk_weighted(rng, bs, popularity, k):
    """K distinct ids per token drawn one after another without replacement
    with probabilities proportional to ``popularity`` (Gumbel-top-k)."""
    logp = np.log(np.asarray(popularity, np.float64))
    g = rng.gumbel(size=(bs, len(logp)))
    return np.argsort(-(logp[None, :] + g), axis=1)[:, :k].astype(np.int32)


def softmax_scales(rng, bs, k, sigma=1.0):
    """expertScales: fp32 softmax over K logits drawn ~ N(0, sigma^2)."""
    z = rng.normal(0.0, sigma, size=(bs, k))
    z = np.exp(z - z.max(axis=1, keepdims=True))
    return (z / z.sum(axis=1, keepdims=True)).astype(np.float32)


def _common(rng, bs, hidden, top_k, rows):
    return dict(
        residual=bf16_bits(rng.standard_normal((bs, hidden), np.float32)),
        gamma=bf16_bits(rng.uniform(0.5, 1.5, size=hidden).astype(np.float32)),
        expert_out=bf16_bits(rng.standard_normal((rows, hidden), np.float32)),
    )


def make(name: str, seed: Optional[int] = None, bs: Optional[int] = None) -> Workload:
    """Build one named workload.  ``seed`` / ``bs`` override the defaults."""
    spec = dict(WORKLOADS[name])
    if seed is not None:
        spec["seed"] = seed
    if bs is not None:
        spec["bs"] = bs
    return spec.pop("builder")(name, **spec)


def uniform_layer(name, seed, bs, hidden, num_experts, top_k, ep_world_size, quant_mode,
                   smooth=False, shared=False, prune_threshold=0.0, logit_sigma=1.0):
    rng = np.random.Generator(np.random.PCG64(seed))
    x = bf16_bits(rng.standard_normal((bs, hidden), np.float32))
    ids = topk_uniform(rng, bs, num_experts, top_k)
    scales = softmax_scales(rng, bs, top_k, logit_sigma)
    w = Workload(name=name, bs=bs, hidden=hidden, top_k=top_k, num_logical=num_experts,
                 num_instances=num_experts, ep_world_size=ep_world_size, quant_mode=quant_mode,
                 x=x, expert_ids=ids, expert_scales=scales,
                 table=identity_table(num_experts, ep_world_size), norm_eps=1e-6,
                 prune_threshold=prune_threshold, **_common(rng, bs, hidden, top_k, bs * top_k))
    if smooth:
        w.smooth = rng.uniform(0.5, 2.0, size=(num_experts, hidden)).astype(np.float32)
    if shared:
        w.shared_x = bf16_bits(rng.standard_normal((bs, hidden), np.float32))
    return w


def _skewed_eplb(name, seed, bs, hidden=4096, num_logical=128, top_k=8, ep_world_size=16,
                 hot=16, hot_replicas=3, zipf_s=1.2, outlier_p=0.01, outlier_scale=20.0):
    """Zipf expert popularity (hot = low ids), the hot experts replicated so
    the instance count divides evenly over the ranks, X with rare outliers,
    mxfp8 dispatch."""
    rng = np.random.Generator(np.random.PCG64(seed))
    xf = rng.standard_normal((bs, hidden), np.float32)
    out = rng.random((bs, hidden)) < outlier_p
    xf[out] *= np.float32(outlier_scale)
    pop = (np.arange(num_logical) + 1.0) ** (-zipf_s)
    ids = topk_weighted(rng, bs, pop, top_k)
    scales = softmax_scales(rng, bs, top_k)
    replicas = np.ones(num_logical, np.int64)
    replicas[:hot] = hot_replicas
    table = replicated_table(rng, num_logical, replicas, ep_world_size)
    return Workload(name=name, bs=bs, hidden=hidden, top_k=top_k, num_logical=num_logical,
                    num_instances=int(replicas.sum()), ep_world_size=ep_world_size, quant_mode=4,
                    x=bf16_bits(xf), expert_ids=ids, expert_scales=scales, table=table,
                    norm_eps=1e-6, **_common(rng, bs, hidden, top_k, bs * top_k))


def _all_ranks_layer(name, seed, bs, sources, **kw):
    """Every one of `sources` simulated ranks sends its own Bs tokens: a
    uniform layer of sources * bs tokens, rank-major, tagged with the number
    of source ranks."""
    w = uniform_layer(name, seed, bs=bs * sources, **kw)
    w.meta["sources"] = sources
    return w


def _tp_layer(name, seed, bs, ep_world_size, **kw):
    """A TP domain of two ranks: 2 * ep_world_size devices of Bs tokens each
    (TP-major), one instance per EP rank, and the TP pair's second partial
    expert output of every row (the first is the workload's expert_out)."""
    S = 2 * ep_world_size
    w = uniform_layer(name, seed, bs=bs * S, num_experts=ep_world_size, ep_world_size=ep_world_size, **kw)
    rng = np.random.Generator(np.random.PCG64([seed, 26]))
    w.meta.update(sources=S, tp=2, expert_out_tp1=bf16_bits(rng.standard_normal(w.expert_out.shape, np.float32)))
    return w


def _static_layer(name, seed, **kw):
    """A uniform layer with static int8 quantization (quantMode 1): per-instance
    static scales U(10, 40), so x ~ N(0, 1) fills much of the int8 range and
    the tails saturate."""
    w = uniform_layer(name, seed, quant_mode=1, **kw)
    rng = np.random.Generator(np.random.PCG64([seed, 21]))
    w.smooth = rng.uniform(10.0, 40.0, size=(w.num_instances, w.hidden)).astype(np.float32)
    return w


def _expert_layer(name, seed, expert_out_dim, **kw):
    """A uniform layer whose step includes the instances' grouped int8 matmul
    between dispatch and combine: every instance owns an int8 weight
    [expert_out_dim, H] with per-channel factors (drawn on the device by
    gmm_weights_device from meta["weight_seed"]); expert_out_dim = H, so the
    matmul's rows are what the combine gathers."""
    w = uniform_layer(name, seed, **kw)
    w.meta["expert_out_dim"] = expert_out_dim
    w.meta["weight_seed"] = 500 + seed
    return w


WORKLOADS = {
    # Bs 8, H 1024, 8 experts, K 2, 4 simulated ranks, no quantization.
    "tiny": dict(builder=uniform_layer, seed=0, bs=8, hidden=1024, num_experts=8, top_k=2,
                 ep_world_size=4, quant_mode=0),
    # Decode batch of a DeepSeek-like layer: 256 experts, K 8, 32 ranks, per-token
    # int8 with per-expert smooth scales, one shared expert.
    "deepseek_decode": dict(builder=uniform_layer, seed=1, bs=256, hidden=7168, num_experts=256,
                            top_k=8, ep_world_size=32, quant_mode=2, smooth=True, shared=True),
    # The same layer at the largest batch the pages allow (Bs 512).
    "deepseek_decode_bs512": dict(builder=uniform_layer, seed=1, bs=512, hidden=7168,
                                  num_experts=256, top_k=8, ep_world_size=32, quant_mode=2,
                                  smooth=True, shared=True),
    # ... and its unquantized variant (bf16 rows, no smooth, no shared expert).
    "deepseek_decode_bs512_bf16": dict(builder=uniform_layer, seed=1, bs=512, hidden=7168,
                                       num_experts=256, top_k=8, ep_world_size=32, quant_mode=0),
    # The Bs 512 layer with static int8 quantization and per-instance scales.
    "deepseek_decode_bs512_static": dict(builder=_static_layer, seed=1, bs=512, hidden=7168,
                                         num_experts=256, top_k=8, ep_world_size=32, shared=True),
    # All ranks as sources: the DeepSeek-like layer on 8 simulated ranks (32
    # experts each), every rank sending its own Bs = 512 tokens (4096 tokens,
    # 32768 copies).
    "deepseek_ep8_all_ranks": dict(builder=_all_ranks_layer, seed=1, bs=512, sources=8, hidden=7168,
                                   num_experts=256, top_k=8, ep_world_size=8, quant_mode=2, smooth=True,
                                   shared=True),
    # The Bs 512 decode layer with the instances' int8 matmul in the step:
    # 256 instance weights of 7168 x 7168 int8 (13.2 GB, resident).
    "deepseek_decode_bs512_expert": dict(builder=_expert_layer, seed=1, bs=512, hidden=7168, num_experts=256,
                                         top_k=8, ep_world_size=32, quant_mode=2, smooth=True, shared=True,
                                         expert_out_dim=7168),
    # The Bs 512 layer dispatched as mxfp8 (quantMode 4, E8M0 block factors)
    # with mxfp8 instance weights of 7168 x 7168 (13.2 GB + 0.4 GB of factors).
    "deepseek_decode_bs512_expert_mx": dict(builder=_expert_layer, seed=1, bs=512, hidden=7168, num_experts=256,
                                            top_k=8, ep_world_size=32, quant_mode=4, shared=True,
                                            expert_out_dim=7168),
    # The same layer cut to 32 instances and Bs 128 (1.6 GB of weights), small
    # enough for a profiler capture of the matmul kernel.
    "expert_e32_bs128": dict(builder=_expert_layer, seed=1, bs=128, hidden=7168, num_experts=32, top_k=8,
                             ep_world_size=8, quant_mode=2, smooth=True, shared=True, expert_out_dim=7168),
    # ... and its mxfp8 form, for the profiler capture of the block-scaled kernel.
    "expert_e32_bs128_mx": dict(builder=_expert_layer, seed=1, bs=128, hidden=7168, num_experts=32, top_k=8,
                                ep_world_size=8, quant_mode=4, shared=True, expert_out_dim=7168),
    # Zipf(1.2) routing over 128 experts, 160 instances on 16 ranks, mxfp8.
    "skewed_eplb": dict(builder=_skewed_eplb, seed=2, bs=512),
    # A TP domain of two ranks: 32 EP ranks with one expert each, every EP rank
    # a TP pair (64 devices of Bs 64 tokens, 4096 tokens, 32768 copies), H
    # 7168, K 8, per-token int8 with smooth scales, shared expert; the combine
    # reads both TP ranks' partial outputs of every row.
    "tp2_decode": dict(builder=_tp_layer, seed=5, bs=64, ep_world_size=32, hidden=7168, top_k=8, quant_mode=2,
                       smooth=True, shared=True),
    # Largest shapes: H 8192, 1024 experts, K 16, 256 ranks, per-128-tile int8,
    # threshold pruning at 0.05 on softmax weights of N(0, 2) logits.
    "max_shape": dict(builder=uniform_layer, seed=3, bs=512, hidden=8192, num_experts=1024,
                      top_k=16, ep_world_size=256, quant_mode=3, prune_threshold=0.05,
                      logit_sigma=float(np.sqrt(2.0))),
}


@dataclass
class LayerStack:
    """Inputs of L chained MoE layers: X_0, residual_0, and per layer the
    routing (ids, scales) and gamma.  Layer l+1 takes X = y_l and
    residual = x_out_l; the expert is the identity (combine reads the rows
    dispatch wrote)."""
    bs: int
    hidden: int
    top_k: int
    num_experts: int
    ep_world_size: int
    layers: int
    x0: np.ndarray
    residual0: np.ndarray
    expert_ids: list
    expert_scales: list
    gammas: list
    table: np.ndarray
    norm_eps: float = 1e-6


def make_layer_stack(seed=4, layers=32, bs=128, hidden=2048, num_experts=64, top_k=6,
                     ep_world_size=8) -> LayerStack:
    rng0 = np.random.Generator(np.random.PCG64([seed, 1000]))
    x0 = bf16_bits(rng0.standard_normal((bs, hidden), np.float32))
    r0 = bf16_bits(rng0.standard_normal((bs, hidden), np.float32))
    ids, scs, gs = [], [], []
    for l in range(layers):
        rng = np.random.Generator(np.random.PCG64([seed, l]))
        ids.append(topk_uniform(rng, bs, num_experts, top_k))
        scs.append(softmax_scales(rng, bs, top_k))
        gs.append(bf16_bits(rng.uniform(0.5, 1.5, size=hidden).astype(np.float32)))
    return LayerStack(bs=bs, hidden=hidden, top_k=top_k, num_experts=num_experts,
                      ep_world_size=ep_world_size, layers=layers, x0=x0, residual0=r0,
                      expert_ids=ids, expert_scales=scs, gammas=gs,
                      table=identity_table(num_experts, ep_world_size))


# --------------------------------------------------------------------------
# the instances' grouped matmul between dispatch and combine
# --------------------------------------------------------------------------

@dataclass
class GmmInputs:
    """One grouped-matmul call: int8 rows (the dispatch's expert-major receive
    buffer) with one dequantization factor each, the per-instance offsets,
    and every instance's int8 weight [N, H] with one factor per channel."""
    expand_x: np.ndarray       # [rows, H] int8
    dyn_scales: np.ndarray     # [rows] f32
    offsets: np.ndarray        # [E + 1] int32
    weight: np.ndarray         # [E, N, H] int8
    weight_scales: np.ndarray  # [E, N] f32


def gmm_inputs(seed, counts, hidden, out_dim, spare_rows=0, one_hot=False) -> GmmInputs:
    """``counts[e]`` rows for instance e, ``spare_rows`` unused rows after
    them.  Codes and weights are uniform over [-127, 127] (weights down to
    -128); row factors ~U(0.005, 0.05) (a row max of 0.6..6 over 127), channel
    factors ~U(1e-4, 1e-3).  ``one_hot``: each row holds a single non-zero
    code in [-15, 15] at a random position and weights lie in [-15, 15], so
    every output is one product, exact in bf16 with unit factors."""
    rng = np.random.Generator(np.random.PCG64([seed, 77]))
    counts = np.asarray(counts, np.int64)
    E = len(counts)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(off[-1]) + int(spare_rows)
    if one_hot:
        x = np.zeros((rows, hidden), np.int8)
        pos = rng.integers(0, hidden, rows)
        x[np.arange(rows), pos] = rng.integers(-15, 15, rows, endpoint=True).astype(np.int8)
        w = rng.integers(-15, 15, (E, out_dim, hidden), dtype=np.int8, endpoint=True)
        ds = np.ones(rows, np.float32)
        ws = np.ones((E, out_dim), np.float32)
    else:
        x = rng.integers(-127, 127, (rows, hidden), dtype=np.int8, endpoint=True)
        w = rng.integers(-128, 127, (E, out_dim, hidden), dtype=np.int8, endpoint=True)
        ds = rng.uniform(0.005, 0.05, rows).astype(np.float32)
        ws = rng.uniform(1e-4, 1e-3, (E, out_dim)).astype(np.float32)
    return GmmInputs(expand_x=x, dyn_scales=ds, offsets=off, weight=w, weight_scales=ws)


def gmm_weights_device(seed, num_instances, out_dim, hidden, device):
    """Instance weights too large to draw on the host (E x N x H int8, e.g.
    256 x 7168 x 7168 = 13 GB), drawn on ``device`` by torch's seeded
    generator: codes uniform over [-128, 127], channel factors ~U(1e-4, 1e-3).
    Returns (weight [E, N, H] int8, weight_scales [E, N] f32)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    w = torch.empty((num_instances, out_dim, hidden), dtype=torch.int8, device=device)
    for e in range(num_instances):  # one instance at a time bounds the int64 scratch
        w[e] = torch.randint(-128, 128, (out_dim, hidden), generator=g, device=device, dtype=torch.int8)
    ws = torch.rand((num_instances, out_dim), generator=g, device=device) * 9e-4 + 1e-4
    return w, ws


def gmm_weights_host(seed, instances, out_dim, hidden):
    """Host-side weights for the given instances, for CPU runs that touch only
    a few of them: per instance an independent seeded stream, codes uniform
    over [-128, 127], channel factors ~U(1e-4, 1e-3) (the distribution of
    gmm_weights_device; the values differ).  Returns {e: (w [N, H] int8,
    ws [N] f32)}."""
    out = {}
    for e in instances:
        rng = np.random.Generator(np.random.PCG64([seed, 9000 + int(e)]))
        out[int(e)] = (rng.integers(-128, 127, (out_dim, hidden), dtype=np.int8, endpoint=True),
                       rng.uniform(1e-4, 1e-3, out_dim).astype(np.float32))
    return out


@dataclass
class GmmMxInputs:
    """One grouped-matmul call on mxfp8: E4M3 rows with one E8M0 factor per
    32-element block (the dispatch's quantMode-4 output) and E4M3 instance
    weights with their own E8M0 block factors."""
    expand_x: np.ndarray   # [rows, H] uint8 E4M3 codes
    x_sf: np.ndarray       # [rows, H/32] uint8 E8M0
    offsets: np.ndarray    # [E + 1] int32
    weight: np.ndarray     # [E, N, H] uint8 E4M3 codes
    weight_sf: np.ndarray  # [E, N, H/32] uint8 E8M0


def _e4m3_codes(rng, shape):
    """Uniform over the 254 finite E4M3 codes (S.1111.111 is NaN)."""
    c = rng.integers(0, 254, shape, dtype=np.uint16)  # 0..253 -> skip 0x7F and 0xFF
    c = c + (c >= 0x7F) + (c >= 0xFE)
    return c.astype(np.uint8)


def gmm_inputs_mx(seed, counts, hidden, out_dim, spare_rows=0, one_hot=False) -> GmmMxInputs:
    """Row codes and weights uniform over the finite E4M3 codes, block
    factors 2^(b - 127) with b uniform in [117, 137].  ``one_hot``: one
    non-zero row code per row (at a random position) and weights whose
    codes are exact small values, so every output is a single scaled
    product."""
    rng = np.random.Generator(np.random.PCG64([seed, 78]))
    counts = np.asarray(counts, np.int64)
    E = len(counts)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(off[-1]) + int(spare_rows)
    B = hidden // 32
    xs = rng.integers(117, 137, (rows, B), dtype=np.uint8, endpoint=True)
    wsf = rng.integers(117, 137, (E, out_dim, B), dtype=np.uint8, endpoint=True)
    if one_hot:
        x = np.zeros((rows, hidden), np.uint8)
        x[np.arange(rows), rng.integers(0, hidden, rows)] = _e4m3_codes(rng, rows)
    else:
        x = _e4m3_codes(rng, (rows, hidden))
    w = _e4m3_codes(rng, (E, out_dim, hidden))
    return GmmMxInputs(expand_x=x, x_sf=xs, offsets=off, weight=w, weight_sf=wsf)


def gmm_weights_device_mx(seed, num_instances, out_dim, hidden, device):
    """mxfp8 instance weights drawn on ``device`` by torch's seeded generator:
    codes uniform over the 254 finite E4M3 codes, block factors 2^(b - 127)
    with b uniform in [117, 137].  Returns (weight [E, N, H] uint8,
    weight_sf [E, N, H/32] uint8)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    w = torch.empty((num_instances, out_dim, hidden), dtype=torch.uint8, device=device)
    for e in range(num_instances):
        c = torch.randint(0, 254, (out_dim, hidden), generator=g, device=device, dtype=torch.int16)
        w[e] = (c + (c >= 0x7F).to(torch.int16) + (c >= 0xFE).to(torch.int16)).to(torch.uint8)
    sf = torch.randint(117, 138, (num_instances, out_dim, hidden // 32), generator=g, device=device,
                       dtype=torch.int16).to(torch.uint8)
    return w, sf


def gmm_weights_host_mx(seed, instances, out_dim, hidden):
    """Host-side mxfp8 weights for the given instances (the distribution of
    gmm_weights_device_mx; the values differ): {e: (codes [N, H] uint8,
    factors [N, H/32] uint8)}."""
    out = {}
    for e in instances:
        rng = np.random.Generator(np.random.PCG64([seed, 9500 + int(e)]))
        out[int(e)] = (_e4m3_codes(rng, (out_dim, hidden)),
                       rng.integers(117, 137, (out_dim, hidden // 32), dtype=np.uint8, endpoint=True))
    return out
