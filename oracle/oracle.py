"""Python front of the CPU oracle (oracle/moe_oracle.c).

TEST INFRASTRUCTURE ONLY.  Only the test-suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this module.  It builds
the C oracle with gcc (``-O2 -fno-fast-math -ffp-contract=off``), loads it
with ctypes and marshals numpy arrays; all arithmetic lives in the C file.
It never imports the product package and the product never imports it.

bf16 arrays are numpy ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_HDR = os.path.join(_HERE, "moe_oracle.h")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "libmoe_oracle.so")
CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared"]

ERR_BAD_ID = 1
ERR_BAD_TABLE = 2

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/libmoe_oracle.so`` if stale."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    newest_src = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < newest_src:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            vp, i32, f32, f64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_double
            L.orc_update_expert.restype = ctypes.c_uint32
            L.orc_update_expert.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, f32, vp, vp, vp]
            L.orc_dispatch.restype = ctypes.c_uint32
            L.orc_dispatch.argtypes = [i32, i32, i32, i32, i32, vp, vp, vp, vp, ctypes.c_int64, vp, vp, vp, vp,
                                       vp, vp]
            L.orc_combine_add_rmsnorm.restype = None
            L.orc_combine_add_rmsnorm.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp, f64,
                                                  vp, vp, vp, vp, vp]
            L.orc_combine.restype = None
            L.orc_combine.argtypes = [i32, i32, i32, vp, vp, vp, vp, vp, vp]
            L.orc_e4m3_encode.restype = ctypes.c_uint8
            L.orc_grouped_matmul.restype = ctypes.c_uint32
            L.orc_grouped_matmul.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]
            L.orc_grouped_matmul_mx.restype = ctypes.c_uint32
            L.orc_grouped_matmul_mx.argtypes = [i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp]
            L.orc_e4m3_decode.restype = f64
            L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
            L.orc_e4m3_encode.argtypes = [f32]
            L.orc_bf16_from_double.restype = ctypes.c_uint16
            L.orc_bf16_from_double.argtypes = [f64]
            L.orc_tp_allgather.restype = None
            L.orc_tp_allgather.argtypes = [i32, ctypes.c_int64, vp, vp, vp, vp, vp, vp, vp, vp]
            L.orc_tp_reduce.restype = None
            L.orc_tp_reduce.argtypes = [ctypes.c_int64, vp, vp, vp]
            _lib = L
    return _lib


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def update_expert(expert_ids, table, ep_world_size, expert_scales=None, active_mask=None,
                  prune_threshold=0.0):
    """aclnnMoeUpdateExpert: returns (balanced_ids [bs,K] int32, balanced_mask [bs,K] uint8, err)."""
    ids = _c(expert_ids, np.int32)
    tab = _c(table, np.int32)
    bs, k = ids.shape
    sc = _c(expert_scales, np.float32)
    am = _c(active_mask, np.uint8)
    bal = np.empty((bs, k), np.int32)
    bm = np.empty((bs, k), np.uint8)
    err = lib().orc_update_expert(bs, k, tab.shape[0], tab.shape[1], int(ep_world_size),
                                  _p(ids), _p(sc), _p(am), float(prune_threshold), _p(tab),
                                  _p(bal), _p(bm))
    return bal, bm, int(err)


def dispatch(x_bf16, instance_ids, num_instances, quant_mode, mask=None, smooth=None):
    """aclnnMoeDistributeDispatchV2 on one simulated source rank.

    Returns a dict: expand_x [bs*K, H] (uint16 bf16 bits for mode 0, int8 for
    modes 1/2/3, uint8 e4m3 codes for mode 4), dyn_scales (None for modes 0
    and 1; [rows] f32, [rows, ceil(H/128)] f32, or [rows, H/32] uint8 E8M0),
    expand_idx [bs,K], src_of_row [n], counts [E], offsets [E+1], n, err.
    smooth: modes 2/3 the (E, H) smooth scales or None; mode 1 the static
    scales, shape (1,), (H,) or (E, H).
    """
    x = _c(x_bf16, np.uint16)
    ids = _c(instance_ids, np.int32)
    bs, H = x.shape
    k = ids.shape[1]
    rows = bs * k
    m = _c(mask, np.uint8)
    sm = _c(smooth, np.float32)
    if quant_mode == 0:
        ex = np.zeros((rows, H), np.uint16)
        ds = None
    elif quant_mode == 1:
        if sm is None or sm.size not in (1, H, num_instances * H):
            raise ValueError("static quantization needs scales of shape (1,), (H,) or (E, H)")
        ex = np.zeros((rows, H), np.int8)
        ds = None
    elif quant_mode == 2:
        ex = np.zeros((rows, H), np.int8)
        ds = np.zeros((rows,), np.float32)
    elif quant_mode == 3:
        ex = np.zeros((rows, H), np.int8)
        ds = np.zeros((rows, (H + 127) // 128), np.float32)
    elif quant_mode == 4:
        ex = np.zeros((rows, H), np.uint8)
        ds = np.zeros((rows, H // 32), np.uint8)
    else:
        raise ValueError(f"oracle has no quant_mode {quant_mode}")
    idx = np.empty((bs, k), np.int32)
    src = np.full((rows,), -1, np.int32)
    cnt = np.empty((num_instances,), np.int32)
    off = np.empty((num_instances + 1,), np.int32)
    err = lib().orc_dispatch(bs, H, k, int(num_instances), int(quant_mode), _p(x), _p(ids), _p(m),
                             _p(sm), ctypes.c_int64(0 if sm is None else sm.size), _p(ex), _p(ds), _p(idx),
                             _p(src), _p(cnt), _p(off))
    n = int(off[-1])
    return dict(expand_x=ex, dyn_scales=ds, expand_idx=idx, src_of_row=src[:n], counts=cnt,
                offsets=off, n=n, err=int(err))


def combine_add_rmsnorm(expand_x_bf16, expand_idx, expert_scales, residual_x, gamma, norm_eps,
                        shared_x=None):
    """aclnnMoeDistributeCombineAddRmsNorm.  Returns a dict with y / x_out as
    bf16 bits, their unrounded float64 values, and rstd (float32)."""
    ex = _c(expand_x_bf16, np.uint16)
    idx = _c(expand_idx, np.int32)
    sc = _c(expert_scales, np.float32)
    res = _c(residual_x, np.uint16)
    g = _c(gamma, np.uint16)
    sh = _c(shared_x, np.uint16)
    bs, k = idx.shape
    H = res.shape[1]
    y = np.empty((bs, H), np.uint16)
    xo = np.empty((bs, H), np.uint16)
    rstd = np.empty((bs,), np.float32)
    y64 = np.empty((bs, H), np.float64)
    x64 = np.empty((bs, H), np.float64)
    lib().orc_combine_add_rmsnorm(bs, H, k, _p(ex), _p(idx), _p(sc), _p(sh), _p(res), _p(g),
                                  float(norm_eps), _p(y), _p(xo), _p(rstd), _p(y64), _p(x64))
    return dict(y=y, x_out=xo, rstd=rstd, y_f64=y64, x_f64=x64)


def combine(expand_x_bf16, expand_idx, expert_scales, shared_x=None):
    """The plain combine (CombineV2 series): combineOut = sum_k (s_k * row_k +
    s_k * shared) per token, no residual, no RMSNorm.  Returns out (bf16
    bits) and out_f64."""
    ex = _c(expand_x_bf16, np.uint16)
    idx = _c(expand_idx, np.int32)
    sc = _c(expert_scales, np.float32)
    sh = _c(shared_x, np.uint16)
    bs, k = idx.shape
    H = ex.shape[1]
    out = np.empty((bs, H), np.uint16)
    o64 = np.empty((bs, H), np.float64)
    lib().orc_combine(bs, H, k, _p(ex), _p(idx), _p(sc), _p(sh), _p(out), _p(o64))
    return dict(out=out, out_f64=o64)


def grouped_matmul(expand_x, dyn_scales, expert_offsets, weight, weight_scales, out=None):
    """The instances' grouped matmul between dispatch and combine: rows
    [off[e], off[e+1]) of expand_x (int8) times instance e's int8 weight
    [N, H], scaled by each row's dyn_scale and each output channel's weight
    scale.  ``out`` (bf16 bits, [rows, N]) may be given pre-filled: rows the
    call does not own keep their content.  Returns out, out_f64 (NaN where
    not written) and the error word."""
    ex = _c(expand_x, np.int8)
    ds = _c(dyn_scales, np.float32)
    off = _c(expert_offsets, np.int32)
    w = _c(weight, np.int8)
    ws = _c(weight_scales, np.float32)
    rows, H = ex.shape
    E, N = w.shape[0], w.shape[1]
    assert w.shape == (E, N, H) and ws.shape == (E, N) and off.shape == (E + 1,) and ds.shape == (rows,)
    out = np.zeros((rows, N), np.uint16) if out is None else _c(out, np.uint16).copy()
    o64 = np.full((rows, N), np.nan, np.float64)
    err = lib().orc_grouped_matmul(rows, H, N, E, _p(ex), _p(ds), _p(off), _p(w), _p(ws), _p(out), _p(o64))
    return dict(out=out, out_f64=o64, err=int(err))


def grouped_matmul_mx(expand_x, x_sf, expert_offsets, weight, weight_sf, out=None):
    """grouped_matmul on mxfp8: E4M3 rows [rows, H] with E8M0 block factors
    x_sf [rows, H/32], E4M3 weights [E, N, H] with weight_sf [E, N, H/32].
    Returns out (bf16 bits), out_f64 (NaN where not written) and err."""
    ex = _c(expand_x, np.uint8)
    xs = _c(x_sf, np.uint8)
    off = _c(expert_offsets, np.int32)
    w = _c(weight, np.uint8)
    wsf = _c(weight_sf, np.uint8)
    rows, H = ex.shape
    E, N = w.shape[0], w.shape[1]
    assert w.shape == (E, N, H) and wsf.shape == (E, N, H // 32) and xs.shape == (rows, H // 32)
    assert off.shape == (E + 1,) and H % 32 == 0
    out = np.zeros((rows, N), np.uint16) if out is None else _c(out, np.uint16).copy()
    o64 = np.full((rows, N), np.nan, np.float64)
    err = lib().orc_grouped_matmul_mx(rows, H, N, E, _p(ex), _p(xs), _p(off), _p(w), _p(wsf), _p(out), _p(o64))
    return dict(out=out, out_f64=o64, err=int(err))


def e4m3_decode(codes):
    f = lib().orc_e4m3_decode
    c = np.asarray(codes, np.uint8).ravel()
    return np.array([f(int(t)) for t in c], np.float64).reshape(np.shape(codes))


def e4m3_encode(values):
    """Element-wise oracle e4m3 encoder (slow: one ctypes call per value)."""
    f = lib().orc_e4m3_encode
    v = np.asarray(values, np.float32).ravel()
    return np.array([f(float(t)) for t in v], np.uint8).reshape(np.shape(values))


def bf16_from_double(values):
    f = lib().orc_bf16_from_double
    v = np.asarray(values, np.float64).ravel()
    return np.array([f(float(t)) for t in v], np.uint16).reshape(np.shape(values))


def dispatch_tp(x_bf16, instance_ids, num_instances, quant_mode, ep_world_size, bs, mask=None, smooth=None):
    """aclnnMoeDistributeDispatchV2 with a TP domain of two ranks (READING
    R26): 2 * ep_world_size devices of bs tokens each, TP-major (device
    t * ep_world_size + g is EP rank g of TP domain t).  Each TP domain runs
    its own EP AllToAllV (the one-rank-per-source dispatch of its tokens),
    then every EP rank's pair gathers both domains' rows (AllGatherV).
    Needs one instance per rank.  Returns the dispatch dict over all
    2 * ep_world_size * bs tokens (expand_idx and src_of_row in global
    numbering) plus tp_counts [E, 2]."""
    if num_instances != ep_world_size:
        raise ValueError("the TP domain needs one instance per EP rank")
    x = _c(x_bf16, np.uint16)
    ids = _c(instance_ids, np.int32)
    m = _c(mask, np.uint8)
    K = ids.shape[1]
    T = 2 * ep_world_size * bs
    if x.shape[0] != T or ids.shape[0] != T:
        raise ValueError("x and the ids hold 2 * ep_world_size * bs tokens")
    dom = [slice(t * ep_world_size * bs, (t + 1) * ep_world_size * bs) for t in range(2)]
    d = [dispatch(x[s], ids[s], num_instances, quant_mode, mask=None if m is None else m[s], smooth=smooth)
         for s in dom]
    n = d[0]["n"] + d[1]["n"]
    E = num_instances

    def gather(a0, a1):
        rb = int(a0[0].nbytes) if a0.ndim > 1 else a0.dtype.itemsize
        out = np.zeros((T * K,) + a0.shape[1:], a0.dtype)
        m0 = np.full((a0.shape[0],), -1, np.int32)
        m1 = np.full((a1.shape[0],), -1, np.int32)
        tc = np.zeros((E, 2), np.int32)
        lib().orc_tp_allgather(E, rb, _p(np.ascontiguousarray(a0)), _p(d[0]["offsets"]),
                               _p(np.ascontiguousarray(a1)), _p(d[1]["offsets"]), _p(out), _p(m0), _p(m1), _p(tc))
        return out, m0, m1, tc

    ex, m0, m1, tc = gather(d[0]["expand_x"], d[1]["expand_x"])
    ds = None if d[0]["dyn_scales"] is None else gather(d[0]["dyn_scales"], d[1]["dyn_scales"])[0]
    idx = np.empty((T, K), np.int32)
    for t, mp in enumerate((m0, m1)):
        di = d[t]["expand_idx"]
        idx[dom[t]] = np.where(di >= 0, mp[np.maximum(di, 0)], -1)
    src = np.empty((n,), np.int32)
    for t, mp in enumerate((m0, m1)):
        nt = d[t]["n"]
        src[mp[:nt]] = d[t]["src_of_row"] + t * ep_world_size * bs * K
    cnt = tc.sum(axis=1).astype(np.int32)
    off = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)
    return dict(expand_x=ex, dyn_scales=ds, expand_idx=idx, src_of_row=src, counts=cnt, offsets=off, n=n,
                tp_counts=tc, err=d[0]["err"] | d[1]["err"])


def tp_reduce(p0_bf16, p1_bf16):
    """ReduceScatterV of the TP pair (READING R26): bf16 of the exact sum of
    the two partial outputs of each row."""
    a = _c(p0_bf16, np.uint16)
    b = _c(p1_bf16, np.uint16)
    if a.shape != b.shape:
        raise ValueError("the two partial outputs must have the same shape")
    out = np.empty_like(a)
    lib().orc_tp_reduce(a.size, _p(a), _p(b), _p(out))
    return out


def combine_add_rmsnorm_tp(p0_bf16, p1_bf16, expand_idx, expert_scales, residual_x, gamma, norm_eps,
                           shared_x=None):
    """aclnnMoeDistributeCombineAddRmsNorm with a TP domain of two ranks:
    rsOut = ReduceScatterV(expandX), then the AllToAllV back, the weighted
    sum, the residual and RMSNorm as without TP."""
    return combine_add_rmsnorm(tp_reduce(p0_bf16, p1_bf16), expand_idx, expert_scales, residual_x, gamma,
                               norm_eps, shared_x=shared_x)
