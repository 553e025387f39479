"""Calls enqueued back to back on one stream, the way a model runs
consecutive layers, with nothing in between: the combine of layer l writes
y_l and the dispatch of layer l+1 reads it as its x at once; the grouped
matmul writes the rows the combine gathers.  Every kernel of the library is
launched as a programmatic dependent of the kernel before it, so these tests
are what shows that no kernel reads an input before the kernel that writes
it has finished (the calling sequence of aclnnMoeUpdateExpert: each operator
consumes its predecessor's output).

Each layer is compared with the oracle run on the inputs the GPU actually
had (its own outputs of the layer before), so the comparison stays
element-wise at every layer.  Outputs are poisoned before the chain runs:
a read that came too early would see the poison, and its codes would differ.
The chains run eagerly and captured in one CUDA graph."""
import numpy as np
import pytest
import torch

from combine_moe_update_b200 import inputs as gen
from oracle import oracle as orc

from gpu_harness import assert_close_bf16, assert_gmm_parity, dev, dev_bf16, host, poison_

pytestmark = pytest.mark.gpu

EPS = 1e-6


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_moe_update_b200 import binding
    return binding


def _bytes(a, n):
    return np.ascontiguousarray(a).view(np.uint8).reshape(a.shape[0], -1)[:n]


def _run(chain, graph, buffers):
    """Run `chain` eagerly or as a replayed CUDA graph; every buffer in
    `buffers` is poisoned right before the run that is checked."""
    if graph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            chain()  # warm-up outside the capture
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            chain()
        for t in buffers:
            poison_(t)
        g.replay()
    else:
        for t in buffers:
            poison_(t)
        chain()
    torch.cuda.synchronize()


def _check_dispatch(got, want):
    n = want["n"]
    np.testing.assert_array_equal(host(got["expand_idx"]), want["expand_idx"])
    np.testing.assert_array_equal(host(got["counts"]), want["counts"])
    np.testing.assert_array_equal(host(got["offsets"]), want["offsets"])
    np.testing.assert_array_equal(host(got["src_of_row"])[:n], want["src_of_row"])
    np.testing.assert_array_equal(_bytes(host(got["expand_x"]), n), _bytes(want["expand_x"], n))
    if want["dyn_scales"] is not None:
        np.testing.assert_array_equal(_bytes(host(got["dyn_scales"]), n), _bytes(want["dyn_scales"], n))


@pytest.mark.parametrize("graph", [False, True], ids=["stream", "graph"])
@pytest.mark.parametrize("bs,H,E,K,ws,mode,smooth", [
    (64, 2048, 32, 4, 8, 0, False),   # 256 copies: the scatter blocks route themselves (the call's first kernel)
    (64, 2048, 32, 4, 8, 2, True),    # the same path with per-instance smooth scales
    (96, 1024, 16, 8, 4, 3, False),   # 768 copies, per-tile int8
    (40, 7168, 64, 8, 8, 2, True),    # 320 copies of the decode row length
    (256, 1024, 64, 8, 8, 2, True),   # 2048 copies: a route kernel is the call's first kernel
    (256, 1024, 64, 8, 8, 0, False),
])
def test_combine_feeds_next_dispatch(B, graph, bs, H, E, K, ws, mode, smooth):
    L = 8
    rng = np.random.Generator(np.random.PCG64([77, bs, H, mode]))
    ids = [gen.topk_uniform(rng, bs, E, K) for _ in range(L)]  # identity table: instance = expert
    scs = [gen.softmax_scales(rng, bs, K) for _ in range(L)]
    gms = [gen.bf16_bits(rng.uniform(0.5, 1.5, size=H).astype(np.float32)) for _ in range(L)]
    rows = [gen.bf16_bits(rng.standard_normal((bs * K, H), np.float32)) for _ in range(L)]
    sm = rng.uniform(0.5, 2.0, size=(E, H)).astype(np.float32) if smooth else None
    x0 = gen.bf16_bits(rng.standard_normal((bs, H), np.float32))
    r0 = gen.bf16_bits(rng.standard_normal((bs, H), np.float32))

    d_ids, d_scs, d_gms = [dev(a) for a in ids], [dev(a) for a in scs], [dev_bf16(a) for a in gms]
    d_rows = [dev_bf16(a) for a in rows]
    d_sm = None if sm is None else dev(sm)
    d_x0, d_r0 = dev_bf16(x0), dev_bf16(r0)
    wsp = B.new_workspace()
    dsp = [B.alloc_dispatch_outputs(bs, H, K, E, mode) for _ in range(L)]
    outs = [dict(y=torch.empty((bs, H), dtype=torch.bfloat16, device="cuda"),
                 x_out=torch.empty((bs, H), dtype=torch.bfloat16, device="cuda"), rstd=None) for _ in range(L)]

    def chain():
        x, r = d_x0, d_r0
        for l in range(L):
            B.dispatch(x, d_ids[l], E, ws, mode, smooth=d_sm, workspace=wsp, out=dsp[l])
            ex = dsp[l]["expand_x"] if mode == 0 else d_rows[l]  # mode 0: the identity expert
            B.combine_add_rmsnorm(ex, dsp[l]["expand_idx"], d_scs[l], r, d_gms[l], EPS, workspace=wsp, out=outs[l])
            x, r = outs[l]["y"], outs[l]["x_out"]

    bufs = [o[k] for o in outs for k in ("y", "x_out")] + [t for d in dsp for t in d.values() if t is not None]
    _run(chain, graph, bufs)
    assert B.read_device_error(wsp) == 0

    x, r = x0, r0
    for l in range(L):
        want = orc.dispatch(x, ids[l], E, mode, smooth=sm)
        _check_dispatch(dsp[l], want)
        ex = host(dsp[l]["expand_x"]) if mode == 0 else rows[l]
        c = orc.combine_add_rmsnorm(ex, host(dsp[l]["expand_idx"]), scs[l], r, gms[l], EPS)
        y, xo = host(outs[l]["y"]), host(outs[l]["x_out"])
        assert_close_bf16(y, c["y_f64"], what=f"y layer {l}")
        assert_close_bf16(xo, c["x_f64"], what=f"x_out layer {l}")
        x, r = y, xo  # the next layer's inputs, as the GPU had them


@pytest.mark.parametrize("graph", [False, True], ids=["stream", "graph"])
def test_matmul_feeds_combine_feeds_next_dispatch(B, graph):
    """dispatch (int8 with smooth scales) -> grouped matmul (N = H) ->
    combine+Add+RMSNorm reading the matmul's rows, and its y as the next
    layer's x, for six layers."""
    L, bs, H, E, K, ws = 6, 64, 1024, 16, 4, 4
    rng = np.random.Generator(np.random.PCG64(78))
    ids = [gen.topk_uniform(rng, bs, E, K) for _ in range(L)]
    scs = [gen.softmax_scales(rng, bs, K) for _ in range(L)]
    gms = [gen.bf16_bits(rng.uniform(0.5, 1.5, size=H).astype(np.float32)) for _ in range(L)]
    sm = rng.uniform(0.5, 2.0, size=(E, H)).astype(np.float32)
    x0 = gen.bf16_bits(rng.standard_normal((bs, H), np.float32))
    r0 = gen.bf16_bits(rng.standard_normal((bs, H), np.float32))
    wt = gen.gmm_inputs(79, [0] * E, H, H)
    rows = bs * K

    d_ids, d_scs, d_gms = [dev(a) for a in ids], [dev(a) for a in scs], [dev_bf16(a) for a in gms]
    d_sm, d_x0, d_r0 = dev(sm), dev_bf16(x0), dev_bf16(r0)
    d_w, d_wsc = dev(wt.weight), dev(wt.weight_scales)
    wsp = B.new_workspace()
    gws = B.new_workspace(nbytes=B.grouped_matmul_workspace_bytes(rows, H, H, E))
    dsp = [B.alloc_dispatch_outputs(bs, H, K, E, 2) for _ in range(L)]
    exs = [torch.empty((rows, H), dtype=torch.bfloat16, device="cuda") for _ in range(L)]
    outs = [dict(y=torch.empty((bs, H), dtype=torch.bfloat16, device="cuda"),
                 x_out=torch.empty((bs, H), dtype=torch.bfloat16, device="cuda"), rstd=None) for _ in range(L)]

    def chain():
        x, r = d_x0, d_r0
        for l in range(L):
            B.dispatch(x, d_ids[l], E, ws, 2, smooth=d_sm, workspace=wsp, out=dsp[l])
            B.grouped_matmul(dsp[l]["expand_x"], dsp[l]["dyn_scales"], dsp[l]["offsets"], d_w, d_wsc, out=exs[l],
                             workspace=gws)
            B.combine_add_rmsnorm(exs[l], dsp[l]["expand_idx"], d_scs[l], r, d_gms[l], EPS, workspace=wsp,
                                  out=outs[l])
            x, r = outs[l]["y"], outs[l]["x_out"]

    bufs = exs + [o[k] for o in outs for k in ("y", "x_out")] + [t for d in dsp for t in d.values() if t is not None]
    _run(chain, graph, bufs)
    assert B.read_device_error(wsp) == 0 and B.read_device_error(gws) == 0

    x, r = x0, r0
    for l in range(L):
        want = orc.dispatch(x, ids[l], E, 2, smooth=sm)
        _check_dispatch(dsp[l], want)
        n = want["n"]
        ex = host(exs[l])
        go = orc.grouped_matmul(want["expand_x"], want["dyn_scales"], want["offsets"], wt.weight, wt.weight_scales,
                                out=ex.copy())
        assert go["err"] == 0
        assert_gmm_parity(ex[:n], dict(out=go["out"][:n], out_f64=go["out_f64"][:n]))
        c = orc.combine_add_rmsnorm(ex, host(dsp[l]["expand_idx"]), scs[l], r, gms[l], EPS)
        y, xo = host(outs[l]["y"]), host(outs[l]["x_out"])
        assert_close_bf16(y, c["y_f64"], what=f"y layer {l}")
        assert_close_bf16(xo, c["x_f64"], what=f"x_out layer {l}")
        x, r = y, xo
