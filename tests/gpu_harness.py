"""Shared helpers of the GPU parity tests: move a seeded workload to the
device, run the three C-ABI calls, run the oracle on the same inputs, and
compare.  Imported by tests only."""
from __future__ import annotations

import numpy as np
import torch

from combine_moe_update_b200 import inputs as gen
from oracle import oracle as orc

POISON = 0xA5  # byte written into outputs before a call, to catch unwritten / overwritten rows


def dev(a) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def dev_bf16(bits) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def poison_(t: torch.Tensor) -> torch.Tensor:
    t.view(torch.uint8).fill_(POISON)
    return t


def assert_close_bf16(got_bits, want_f64, rtol=1e-2, what="y"):
    """|got - want| <= rtol * max(|want|, rms(want row)) element-wise; the
    rms floor keeps near-zero elements from failing on bf16 rounding."""
    got = gen.bf16_to_f32(got_bits).astype(np.float64)
    want = np.asarray(want_f64, np.float64)
    rms = np.sqrt(np.mean(want * want, axis=-1, keepdims=True))
    tol = rtol * np.maximum(np.abs(want), rms)
    bad = np.abs(got - want) > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements off; first at "
                           f"{np.argwhere(bad)[0].tolist()}: got {got[bad][0]}, want {want[bad][0]}")


def run_gpu(w: gen.Workload, B, workspace=None, combine_rows=None, want_x_out=True, sources=1):
    """update_expert -> dispatch -> combine on the GPU.  Outputs are poisoned
    first.  combine reads `combine_rows` (bf16 bits) or the workload's
    synthetic expert outputs.  sources: the workload's w.bs tokens are that
    many source ranks' tokens, rank-major."""
    sl = 0 if w.smooth is None else w.smooth.size
    ws = workspace if workspace is not None else B.new_workspace(nbytes=B.dispatch_workspace_bytes(
        w.bs // sources, w.hidden, w.top_k, w.ep_world_size, w.num_instances, w.quant_mode, sl, sources))
    ids, table, sc = dev(w.expert_ids), dev(w.table), dev(w.expert_scales)
    am = None if w.active_mask is None else dev(w.active_mask)
    bal = poison_(torch.empty_like(ids))
    bm = poison_(torch.empty(ids.shape, dtype=torch.uint8, device="cuda"))
    B.update_expert(ids, table, w.ep_world_size, expert_scales=sc, active_mask=am,
                    prune_threshold=w.prune_threshold, workspace=ws, out=(bal, bm), sources=sources)
    d = B.alloc_dispatch_outputs(w.bs, w.hidden, w.top_k, w.num_instances, w.quant_mode)
    for v in d.values():
        if v is not None:
            poison_(v)
    x = dev_bf16(w.x)
    sm = None if w.smooth is None else dev(w.smooth)
    B.dispatch(x, bal, w.num_instances, w.ep_world_size, w.quant_mode, mask=bm, smooth=sm, workspace=ws, out=d,
               sources=sources)
    rows = combine_rows if combine_rows is not None else w.expert_out
    ex = dev_bf16(rows)
    sh = None if w.shared_x is None else dev_bf16(w.shared_x)
    c = B.combine_add_rmsnorm(ex, d["expand_idx"], sc, dev_bf16(w.residual), dev_bf16(w.gamma), w.norm_eps,
                              shared_x=sh, want_x_out=want_x_out, want_rstd=True, workspace=ws, sources=sources)
    torch.cuda.synchronize()
    out = dict(balanced_ids=host(bal), balanced_mask=host(bm), err=B.read_device_error(ws))
    for k, v in d.items():
        out[k] = None if v is None else host(v)
    out["y"] = host(c["y"])
    out["x_out"] = None if c["x_out"] is None else host(c["x_out"])
    out["rstd"] = host(c["rstd"])
    return out


def run_oracle(w: gen.Workload, combine_rows=None):
    bal, bm, e1 = orc.update_expert(w.expert_ids, w.table, w.ep_world_size, expert_scales=w.expert_scales,
                                    active_mask=w.active_mask, prune_threshold=w.prune_threshold)
    d = orc.dispatch(w.x, bal, w.num_instances, w.quant_mode, mask=bm, smooth=w.smooth)
    rows = combine_rows if combine_rows is not None else w.expert_out
    c = orc.combine_add_rmsnorm(rows, d["expand_idx"], w.expert_scales, w.residual, w.gamma, w.norm_eps,
                                shared_x=w.shared_x)
    return dict(balanced_ids=bal, balanced_mask=bm, err=e1 | d["err"], dispatch=d, combine=c)


def assert_parity(w: gen.Workload, g: dict, o: dict):
    """Bit-exact routing, indices, counts, codes and scales; 1e-2 on bf16."""
    np.testing.assert_array_equal(g["balanced_ids"], o["balanced_ids"])
    np.testing.assert_array_equal(g["balanced_mask"], o["balanced_mask"])
    d = o["dispatch"]
    n = d["n"]
    np.testing.assert_array_equal(g["expand_idx"], d["expand_idx"])
    np.testing.assert_array_equal(g["counts"], d["counts"])
    np.testing.assert_array_equal(g["offsets"], d["offsets"])
    np.testing.assert_array_equal(g["src_of_row"][:n], d["src_of_row"])
    ge = g["expand_x"].view(np.uint8).reshape(g["expand_x"].shape[0], -1)
    oe = d["expand_x"].view(np.uint8).reshape(d["expand_x"].shape[0], -1)
    np.testing.assert_array_equal(ge[:n], oe[:n])
    assert (ge[n:] == POISON).all(), "rows past the used region must stay untouched"
    assert (g["src_of_row"][n:].view(np.uint8) == POISON).all()
    if w.quant_mode in (0, 1):  # no scales are sent
        assert g["dyn_scales"] is None and d["dyn_scales"] is None
    else:
        gs = g["dyn_scales"].view(np.uint8).reshape(g["dyn_scales"].shape[0], -1)
        os_ = d["dyn_scales"].view(np.uint8).reshape(d["dyn_scales"].shape[0], -1)
        np.testing.assert_array_equal(gs[:n], os_[:n])
        assert (gs[n:] == POISON).all()
    c = o["combine"]
    assert_close_bf16(g["y"], c["y_f64"], what="y")
    if g["x_out"] is not None:
        assert_close_bf16(g["x_out"], c["x_f64"], what="x_out")
    np.testing.assert_allclose(g["rstd"], c["rstd"], rtol=1e-5)
    assert g["err"] == o["err"]


def assert_gmm_parity(got, o):
    """The grouped int8 matmul's bar: outputs equal the oracle's bit for bit
    or sit one bf16 step away (only the binary32 scale products differ from
    the oracle's binary64), at least 99.9 % bit-identical, all within the
    1e-2 bar; rows the call does not own keep their content."""
    want = o["out"]
    written = ~np.isnan(o["out_f64"])
    np.testing.assert_array_equal(got[~written], want[~written])
    g, w = got[written].astype(np.int32), want[written].astype(np.int32)
    same = g == w
    assert np.all(np.abs(g - w)[~same] == 1), "a bf16 output is more than one step from the oracle"
    assert same.mean() >= 0.999, f"only {same.mean():.5f} of the outputs are bit-identical"
    if written.any():
        rows = np.flatnonzero(written.any(axis=1))
        assert_close_bf16(got[rows], o["out_f64"][rows], what="gmm out")
