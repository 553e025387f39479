"""The bounded waits' timeout path, through the C ABI of a test-only build.

Every wait of the library for an asynchronous copy is bounded (about a
second of device time): if the copy never lands, the kernel records
MOE_DEV_TIMEOUT in the workspace's error word, drops what it could not
finish, and returns, so the GPU context stays usable.  The shipped library
never leaves a copy out; the test build (-DMOE_FAULT_INJECTION,
libmoe_b200_faultinj.so) leaves out one bulk copy per kernel -- the mapping
table of update_expert, and the second smooth row that the first block of
token 0 in the smooth-scale scatter fetches -- so that nothing is in flight when the wait
runs out.  The tests check the error bit, the outputs that were still
produced, that the wait really ran its course, and that the shipped library
works on the same context afterwards."""
import ctypes
import time

import numpy as np
import pytest
import torch

from combine_moe_update_b200 import inputs as gen
from oracle import oracle as orc

from gpu_harness import POISON, dev, dev_bf16, host, poison_

pytestmark = pytest.mark.gpu

DEV_TIMEOUT = 4


@pytest.fixture(scope="module")
def B():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from combine_moe_update_b200 import binding
    return binding


@pytest.fixture(scope="module")
def FL(B):
    from combine_moe_update_b200 import build
    L = ctypes.CDLL(build.build(fault_injection=True))
    vp, sz, P = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER
    L.moe_update_expert.argtypes = [P(B.UpdateParams), vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_dispatch.argtypes = [P(B.DispatchParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_update_expert.restype = L.moe_dispatch.restype = ctypes.c_int
    return L


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def test_update_expert_table_copy_times_out(B, FL):
    w = gen.make("tiny")  # a 64-byte table: staged in shared memory by one bulk copy
    ws = B.new_workspace()
    ids, table = dev(w.expert_ids), dev(w.table)
    bal = poison_(torch.empty_like(ids))
    bm = poison_(torch.empty(ids.shape, dtype=torch.uint8, device="cuda"))
    p = B.UpdateParams(w.bs, w.top_k, w.table.shape[0], w.table.shape[1], w.ep_world_size, 0.0, 1)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert FL.moe_update_expert(ctypes.byref(p), _p(ids), None, None, _p(table), _p(bal), _p(bm), _p(ws), 256,
                                _stream()) == 0
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert B.read_device_error(ws) & DEV_TIMEOUT
    assert 0.5 < waited < 30.0, waited  # the bounded wait ran its course, then gave up
    assert (host(bal) == -1).all() and (host(bm) == 0).all()  # every copy dropped
    # the context is still usable: the shipped library maps the same ids
    ws2 = B.new_workspace()
    bal2, bm2 = B.update_expert(ids, table, w.ep_world_size, workspace=ws2)
    ob, om, _ = orc.update_expert(w.expert_ids, w.table, w.ep_world_size)
    np.testing.assert_array_equal(host(bal2), ob)
    np.testing.assert_array_equal(host(bm2), om)
    assert B.read_device_error(ws2) == 0


@pytest.mark.parametrize("bs", [4, 160])  # 32 copies (the blocks route themselves), 1280 (a route kernel first)
def test_smooth_scatter_row_copy_times_out(B, FL, bs):
    w = gen.make("deepseek_decode", bs=bs)
    ws = B.new_workspace()
    bal, bm = B.update_expert(dev(w.expert_ids), dev(w.table), w.ep_world_size, workspace=ws)
    x, sm = dev_bf16(w.x), dev(w.smooth)
    d = B.alloc_dispatch_outputs(w.bs, w.hidden, w.top_k, w.num_instances, 2)
    for v in d.values():
        poison_(v)
    p = B.DispatchParams(w.bs, w.hidden, w.top_k, w.ep_world_size, w.num_instances, 2, w.smooth.size, 1)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert FL.moe_dispatch(ctypes.byref(p), _p(x), _p(bal), _p(bm), _p(sm), _p(d["expand_x"]), _p(d["dyn_scales"]),
                           _p(d["expand_idx"]), _p(d["src_of_row"]), _p(d["counts"]), _p(d["offsets"]), _p(ws), 256,
                           _stream()) == 0
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert B.read_device_error(ws) & DEV_TIMEOUT
    assert 0.5 < waited < 30.0, waited
    # The routing is complete.  Token 0's sent copies are split over P
    # blocks (copy groups: block p takes sent copies p, p + P, ...); its
    # block 0 wrote sent copy 0, timed out waiting for copy P's row and
    # stopped, so of token 0 exactly the copies c with c == 0 or c % P != 0
    # are written, for one P in 1, 2, 4.  Every other token wrote all of its
    # copies.
    ob, om, _ = orc.update_expert(w.expert_ids, w.table, w.ep_world_size)
    od = orc.dispatch(w.x, ob, w.num_instances, 2, mask=om, smooth=w.smooth)
    np.testing.assert_array_equal(host(d["expand_idx"]), od["expand_idx"])
    ge = host(d["expand_x"]).view(np.uint8)
    gs = host(d["dyn_scales"]).view(np.uint8).reshape(-1, 4)
    oe, os_ = od["expand_x"].view(np.uint8), od["dyn_scales"].view(np.uint8).reshape(-1, 4)
    sent = [r for r in od["expand_idx"][0] if r >= 0]  # token 0's copies in k order
    assert len(sent) > 4
    written = []
    for r in sent:
        if (ge[r] == POISON).all() and (gs[r] == POISON).all():
            written.append(False)
        else:
            np.testing.assert_array_equal(ge[r], oe[r])
            np.testing.assert_array_equal(gs[r], os_[r])
            written.append(True)
    assert any(written == [c == 0 or c % P != 0 for c in range(len(sent))] for P in (1, 2, 4)), written
    rows = od["expand_idx"][1:].ravel()
    rows = rows[rows >= 0]
    np.testing.assert_array_equal(ge[rows], oe[rows])
    np.testing.assert_array_equal(gs[rows], os_[rows])
    # the context is still usable
    d2 = B.dispatch(x, bal, w.num_instances, w.ep_world_size, 2, mask=bm, smooth=sm, workspace=B.new_workspace())
    torch.cuda.synchronize()
    n = od["n"]
    np.testing.assert_array_equal(host(d2["expand_x"]).view(np.uint8)[:n], oe[:n])
