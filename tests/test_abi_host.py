"""Host-side checks of the C ABI; no GPU needed.

The library must load without a GPU, export every function the header
declares, size workspaces, and reject out-of-contract arguments with the
documented status before it would launch anything.  Only argument sets that
fail validation are passed to the launching entry points here, so nothing
below can reach a kernel.
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

# The negative cases below hand fake (never dereferenced) pointers to calls
# that must reject their arguments first.  Should validation ever regress, a
# launch on such pointers must not be able to reach a real GPU.
pytestmark = pytest.mark.skipif(torch.cuda.is_available(),
                                reason="fake-pointer validation checks run only where no GPU is visible")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def L():
    from combine_moe_update_b200 import build
    build.build()
    from combine_moe_update_b200 import binding
    return binding


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_page_operations():
    names = declared_functions()
    for n in ("moe_update_expert", "moe_dispatch", "moe_combine_add_rmsnorm",
              "moe_update_expert_workspace_size", "moe_dispatch_workspace_size",
              "moe_combine_add_rmsnorm_workspace_size", "moe_read_device_error"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    from combine_moe_update_b200 import build
    out = subprocess.run(["nm", "-D", "--defined-only", build.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\S+)$", out, flags=re.M))
    for n in declared_functions():
        assert n in exported, n
        assert getattr(L.lib, n) is not None
    # nothing beyond the ABI leaks out
    assert {e for e in exported if e.startswith("moe_")} == set(declared_functions())


def test_status_strings(L):
    assert L.lib.moe_status_string(0) == b"MOE_OK"
    assert L.lib.moe_status_string(3) == b"MOE_ERR_WORKSPACE"


def ws_size(L, fn, params):
    n = ctypes.c_size_t(0)
    st = getattr(L.lib, fn)(ctypes.byref(params), ctypes.byref(n))
    return st, n.value


@pytest.mark.parametrize("scales_len", [1, 1024, 8 * 1024])
def test_static_quant_params_accepted(L, scales_len):
    """quantMode 1 with scales of shape (1,), (H,) or (E, H) passes validation."""
    assert ws_size(L, "moe_dispatch_workspace_size", L.DispatchParams(8, 1024, 2, 4, 8, 1, scales_len)) == (0, 256)


def test_workspace_sizes_for_valid_params(L):
    assert ws_size(L, "moe_update_expert_workspace_size", L.UpdateParams(512, 16, 1024, 257, 256, 0.05)) == (0, 256)
    assert ws_size(L, "moe_dispatch_workspace_size", L.DispatchParams(512, 7168, 8, 32, 256, 2)) == (0, 256)
    assert ws_size(L, "moe_dispatch_workspace_size", L.DispatchParams(512, 8192, 16, 256, 1024, 3)) == (0, 256)
    assert L.WORKSPACE_BYTES == 256  # the largest any call needs, and the binding's default
    assert ws_size(L, "moe_combine_add_rmsnorm_workspace_size", L.CombineParams(512, 8192, 16, 8192, 1e-6)) == (0, 256)


UPDATE_BAD = [
    dict(bs=0), dict(bs=513), dict(top_k=0), dict(top_k=17), dict(num_logical=0), dict(num_logical=1025),
    dict(top_k=9, num_logical=8), dict(ep_world_size=1), dict(ep_world_size=769), dict(table_cols=1),
    dict(table_cols=34), dict(prune_threshold=float("nan")),
]


@pytest.mark.parametrize("bad", UPDATE_BAD)
def test_update_expert_rejects(L, bad):
    base = dict(bs=8, top_k=2, num_logical=8, table_cols=2, ep_world_size=32, prune_threshold=0.0)
    base.update(bad)
    p = L.UpdateParams(*base.values())
    assert ws_size(L, "moe_update_expert_workspace_size", p)[0] == L.MOE_ERR_INVALID_ARG
    fake = ctypes.c_void_p(0x10000)
    st = L.lib.moe_update_expert(ctypes.byref(p), fake, None, None, fake, fake, fake, fake, 256, None)
    assert st == L.MOE_ERR_INVALID_ARG


DISPATCH_BAD = [
    (dict(bs=0), 1), (dict(bs=513), 1), (dict(hidden=1008), 1), (dict(hidden=8208), 1), (dict(hidden=1032), 1),
    (dict(top_k=0), 1), (dict(top_k=17), 1), (dict(num_instances=1025), 1), (dict(num_instances=0), 1),
    (dict(ep_world_size=1), 1), (dict(ep_world_size=769), 1), (dict(ep_world_size=24), 1),
    (dict(quant_mode=5), 1), (dict(quant_mode=-1), 1),
    (dict(quant_mode=4, hidden=1040), 1),
    # scales_len must match the mode: static scales (1,), (H,) or (E, H); smooth (E, H); none in modes 0 and 4
    (dict(quant_mode=1, scales_len=0), 1), (dict(quant_mode=1, scales_len=3), 1),
    (dict(quant_mode=2, scales_len=1024), 1), (dict(quant_mode=3, scales_len=1), 1),
    (dict(quant_mode=0, scales_len=1), 1), (dict(quant_mode=4, scales_len=8 * 1024), 1),
]


@pytest.mark.parametrize("bad,status", DISPATCH_BAD)
def test_dispatch_rejects(L, bad, status):
    base = dict(bs=8, hidden=1024, top_k=2, ep_world_size=4, num_instances=8, quant_mode=0, scales_len=0)
    base.update(bad)
    p = L.DispatchParams(*base.values())
    assert ws_size(L, "moe_dispatch_workspace_size", p)[0] == status
    f = ctypes.c_void_p(0x10000)
    st = L.lib.moe_dispatch(ctypes.byref(p), f, f, None, None, f, f if base["quant_mode"] else None,
                            f, f, f, f, f, 256, None)
    assert st == status


def _dispatch_call(L, mode=2, **ptrs):
    p = L.DispatchParams(8, 1024, 2, 4, 8, mode)
    f = ctypes.c_void_p(0x10000)
    args = dict(x=f, ids=f, mask=None, smooth=None, ex=f, ds=f if mode else None, idx=f, src=f, cnt=f,
                off=f, ws=f, wsb=256)
    args.update(ptrs)
    return L.lib.moe_dispatch(ctypes.byref(p), args["x"], args["ids"], args["mask"], args["smooth"],
                              args["ex"], args["ds"], args["idx"], args["src"], args["cnt"], args["off"],
                              args["ws"], args["wsb"], None)


def test_dispatch_pointer_rules(L):
    f8 = ctypes.c_void_p(0x10008)  # 8-byte aligned only
    assert _dispatch_call(L, x=None) == L.MOE_ERR_INVALID_ARG
    assert _dispatch_call(L, x=f8) == L.MOE_ERR_INVALID_ARG          # bf16 rows need 16 bytes
    assert _dispatch_call(L, ex=f8) == L.MOE_ERR_INVALID_ARG
    assert _dispatch_call(L, mode=2, ds=None) == L.MOE_ERR_INVALID_ARG   # mode 2 needs scales out
    assert _dispatch_call(L, mode=0, ds=ctypes.c_void_p(0x10000)) == L.MOE_ERR_INVALID_ARG
    assert _dispatch_call(L, mode=4, smooth=ctypes.c_void_p(0x10000)) == L.MOE_ERR_INVALID_ARG
    assert _dispatch_call(L, mode=0, smooth=ctypes.c_void_p(0x10000)) == L.MOE_ERR_INVALID_ARG
    assert _dispatch_call(L, ws=None) == L.MOE_ERR_WORKSPACE
    assert _dispatch_call(L, wsb=255) == L.MOE_ERR_WORKSPACE


COMBINE_BAD = [dict(bs=0), dict(bs=513), dict(hidden=1000), dict(hidden=9000), dict(top_k=0), dict(top_k=17),
               dict(expand_rows=0), dict(norm_eps=-1.0), dict(norm_eps=float("nan")), dict(norm_eps=float("inf"))]


@pytest.mark.parametrize("bad", COMBINE_BAD)
def test_combine_rejects(L, bad):
    base = dict(bs=8, hidden=1024, top_k=2, expand_rows=16, norm_eps=1e-6)
    base.update(bad)
    p = L.CombineParams(*base.values())
    assert ws_size(L, "moe_combine_add_rmsnorm_workspace_size", p)[0] == L.MOE_ERR_INVALID_ARG
    f = ctypes.c_void_p(0x10000)
    st = L.lib.moe_combine_add_rmsnorm(ctypes.byref(p), f, f, f, None, f, f, f, None, None, f, 256, None)
    assert st == L.MOE_ERR_INVALID_ARG


def test_combine_pointer_rules(L):
    p = L.CombineParams(8, 1024, 2, 16, 1e-6)
    f, f8 = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10008)
    call = lambda ex=f, res=f, y=f, sh=None, ws=f: L.lib.moe_combine_add_rmsnorm(
        ctypes.byref(p), ex, f, f, sh, res, f, y, None, None, ws, 256, None)
    assert call(ex=None) == L.MOE_ERR_INVALID_ARG
    assert call(res=f8) == L.MOE_ERR_INVALID_ARG
    assert call(y=f8) == L.MOE_ERR_INVALID_ARG
    assert call(sh=f8) == L.MOE_ERR_INVALID_ARG
    assert call(ws=None) == L.MOE_ERR_WORKSPACE


GMM_BAD = [dict(rows=0), dict(num_instances=0), dict(num_instances=1025), dict(hidden=1000), dict(hidden=9000),
           dict(hidden=1032), dict(out_dim=0), dict(out_dim=8), dict(out_dim=200), dict(out_dim=65552),
           dict(rows=(65535 - 1024) * 128 + 1, num_instances=1024)]


def _gmm_params(L, **over):
    base = dict(rows=4096, hidden=7168, out_dim=7168, num_instances=256)
    base.update(over)
    return L.GmmParams(base["rows"], base["hidden"], base["out_dim"], base["num_instances"])


@pytest.mark.parametrize("bad", GMM_BAD)
def test_grouped_matmul_rejects(L, bad):
    p = _gmm_params(L, **bad)
    assert ws_size(L, "moe_grouped_matmul_workspace_size", p)[0] == L.MOE_ERR_INVALID_ARG
    f = ctypes.c_void_p(0x10000)
    assert L.lib.moe_grouped_matmul(ctypes.byref(p), f, f, f, f, f, f, f, 1 << 20, None) == L.MOE_ERR_INVALID_ARG


def test_grouped_matmul_workspace_and_pointer_rules(L):
    p = _gmm_params(L)
    st, n = ws_size(L, "moe_grouped_matmul_workspace_size", p)
    assert st == L.MOE_OK and n == 256 + 16 + 16 * (256 + 4096 // 128)
    edge = _gmm_params(L, rows=(65535 - 1024) * 128, num_instances=1024)  # the last row count grid.y allows
    assert ws_size(L, "moe_grouped_matmul_workspace_size", edge)[0] == L.MOE_OK
    f, f8, f2 = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10008), ctypes.c_void_p(0x10002)
    call = lambda x=f, ds=f, off=f, w=f, wsc=f, out=f, ws=f, wsb=n: L.lib.moe_grouped_matmul(
        ctypes.byref(p), x, ds, off, w, wsc, out, ws, wsb, None)
    for kw in (dict(x=None), dict(ds=None), dict(off=None), dict(w=None), dict(wsc=None), dict(out=None),
               dict(x=f8), dict(w=f8), dict(out=f8), dict(ds=f2), dict(off=f2), dict(wsc=f2)):
        assert call(**kw) == L.MOE_ERR_INVALID_ARG, kw
    assert call(ws=None) == L.MOE_ERR_WORKSPACE
    assert call(wsb=n - 16) == L.MOE_ERR_WORKSPACE


def test_no_cpu_fallback_in_product():
    """The product package never reaches the oracle."""
    pkg = os.path.join(ROOT, "combine_moe_update_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b|moe_oracle|orc_", src, re.M), fn


def test_grouped_matmul_mx_rules(L):
    """mxfp8 adds H % 128 == 0 (one 4-byte factor word per row and step) and
    4-byte aligned factor arrays."""
    f, f2, f8 = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10002), ctypes.c_void_p(0x10008)
    p = _gmm_params(L)
    n = ws_size(L, "moe_grouped_matmul_workspace_size", p)[1]
    call = lambda p=p, x=f, xs=f, off=f, w=f, wsf=f, out=f, ws=f, wsb=n: L.lib.moe_grouped_matmul_mx(
        ctypes.byref(p), x, xs, off, w, wsf, out, ws, wsb, None)
    assert call(p=_gmm_params(L, hidden=1056)) == L.MOE_ERR_INVALID_ARG  # % 32 but not % 128
    for kw in (dict(x=None), dict(xs=None), dict(wsf=None), dict(x=f8), dict(w=f8), dict(xs=f2), dict(wsf=f2),
               dict(off=f2)):
        assert call(**kw) == L.MOE_ERR_INVALID_ARG, kw
    assert call(wsb=n - 16) == L.MOE_ERR_WORKSPACE


def test_binding_refuses_host_workspaces(L):
    """A workspace is device memory the kernels write: the binding refuses a
    host tensor (or one of another dtype) before any call is made."""
    host_ws = torch.zeros(256, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA"):
        L.read_device_error(host_ws)
    with pytest.raises(ValueError, match="CUDA"):
        L.clear_device_error(host_ws)
    with pytest.raises(ValueError, match="CUDA"):
        L.grouped_matmul(torch.zeros((4, 1024), dtype=torch.int8), torch.ones(4), torch.zeros(2, dtype=torch.int32),
                         torch.zeros((1, 16, 1024), dtype=torch.int8), torch.ones((1, 16)), workspace=host_ws)


def test_binding_refuses_host_outputs(L):
    """Outputs a caller passes in are written through raw device pointers:
    host tensors, wrong dtypes and missing entries are refused before any
    call is made."""
    rows, H, K, E = 16, 1024, 2, 8
    host = dict(expand_x=torch.zeros((rows, H), dtype=torch.bfloat16), dyn_scales=None,
                expand_idx=torch.zeros((8, K), dtype=torch.int32), src_of_row=torch.zeros(rows, dtype=torch.int32),
                counts=torch.zeros(E, dtype=torch.int32), offsets=torch.zeros(E + 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="CUDA"):
        L._check_dispatch_out(host, 8, H, K, E, 0)
    with pytest.raises(TypeError, match="expand_x"):
        L._check_dispatch_out(dict(host, expand_x=None), 8, H, K, E, 0)
    with pytest.raises(TypeError):
        L._check_dispatch_out([1, 2], 8, H, K, E, 0)
    with pytest.raises(ValueError, match="CUDA"):
        L._check_combine_out(dict(y=torch.zeros((8, H), dtype=torch.bfloat16)), 8, H)


# --------------------------------------------------------------------------
# expert parallelism (fused), the routing-only dispatch, the TP domain
# --------------------------------------------------------------------------

def test_dispatch_route_rules(L):
    f = ctypes.c_void_p(0x10000)
    p = L.DispatchParams(64, 1024, 4, 8, 32, 0, 0, 1)
    call = lambda p_=p, idx=f, ws=f, wsb=256: L.lib.moe_dispatch_route(ctypes.byref(p_), f, None, idx, f, f, f, ws,
                                                                        wsb, None)
    assert call(idx=None) == L.MOE_ERR_INVALID_ARG
    assert call(p_=L.DispatchParams(0, 1024, 4, 8, 32, 0, 0, 1)) == L.MOE_ERR_INVALID_ARG
    assert call(ws=None) == L.MOE_ERR_WORKSPACE


def test_ep_dispatch_rules(L):
    """The EP dispatch checks its parameters against the EP ones (same bs, K,
    E; one source; row and scale bytes of the mode) before anything runs."""
    f = ctypes.c_void_p(0x10000)
    dp = lambda mode=2, bs=64, sources=1: L.DispatchParams(bs, 1024, 4, 8, 32, mode, 32 * 1024 if mode == 2 else 0,
                                                           sources)
    ep = lambda bs=64, row=1024, sc=4: L.EpParams(bs, 4, 32, 2, 0, row, sc, 512)
    n = ctypes.c_size_t(0)
    assert L.lib.moe_ep_workspace_size(ctypes.byref(ep()), ctypes.byref(n)) == L.MOE_OK
    big = n.value

    def call(d=None, e=None, peer=f, scales=f, gidx=f, wsb=None):
        d = d or dp()
        e = e or ep()
        return L.lib.moe_ep_dispatch(ctypes.byref(d), ctypes.byref(e), f, f, None, f, f, f, peer, scales, None,
                                     gidx, f, big if wsb is None else wsb, None)
    assert call(d=dp(bs=32)) == L.MOE_ERR_INVALID_ARG          # bs differs from the EP parameters'
    assert call(d=dp(sources=2)) == L.MOE_ERR_INVALID_ARG      # one source per GPU
    assert call(e=ep(row=2048)) == L.MOE_ERR_INVALID_ARG       # int8 rows are H bytes
    assert call(e=ep(sc=0)) == L.MOE_ERR_INVALID_ARG           # mode 2 sends a 4-byte scale
    assert call(d=dp(mode=0), e=ep(row=2048, sc=0), scales=f) == L.MOE_ERR_INVALID_ARG  # no scale table in mode 0
    assert call(peer=None) == L.MOE_ERR_INVALID_ARG
    assert call(gidx=None) == L.MOE_ERR_INVALID_ARG
    assert call(wsb=16) == L.MOE_ERR_WORKSPACE


def test_ep_combine_rules(L):
    f = ctypes.c_void_p(0x10000)
    cp = lambda bs=64, sources=1: L.CombineParams(bs, 1024, 4, 512, 1e-6, sources)
    ep = lambda row=2048: L.EpParams(64, 4, 32, 2, 0, row, 0, 512)
    n = ctypes.c_size_t(0)
    assert L.lib.moe_ep_workspace_size(ctypes.byref(ep()), ctypes.byref(n)) == L.MOE_OK

    def call(c=None, e=None, peer=f, gidx=f, wsb=None):
        c = c or cp()
        e = e or ep()
        return L.lib.moe_ep_combine_add_rmsnorm(ctypes.byref(c), ctypes.byref(e), peer, gidx, f, None, f, f, f,
                                                None, None, f, n.value if wsb is None else wsb, None)
    assert call(c=cp(bs=32)) == L.MOE_ERR_INVALID_ARG
    assert call(c=cp(sources=2)) == L.MOE_ERR_INVALID_ARG
    assert call(e=ep(row=1024)) == L.MOE_ERR_INVALID_ARG       # bf16 outputs are 2H bytes
    assert call(peer=None) == L.MOE_ERR_INVALID_ARG
    assert call(gidx=None) == L.MOE_ERR_INVALID_ARG
    assert call(wsb=16) == L.MOE_ERR_WORKSPACE


def test_tp_rules(L):
    """The TP counts need one instance per EP rank and 2 * ws TP-major
    sources; the TP combine needs both partial buffers, 16-byte aligned."""
    f, f8 = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10008)
    tp = lambda E=8, S=16: L.DispatchParams(16, 1024, 2, 8, E, 0, 0, S)
    call = lambda p, out=f: L.lib.moe_dispatch_tp_counts(ctypes.byref(p), f, f, out, f, 256, None)
    assert call(tp(S=8)) == L.MOE_ERR_INVALID_ARG        # sources != 2 * ws
    assert call(tp(E=16)) == L.MOE_ERR_INVALID_ARG       # two instances per rank
    assert call(tp(S=17)) == L.MOE_ERR_INVALID_ARG       # past 2 * ws
    assert call(tp(), out=None) == L.MOE_ERR_INVALID_ARG
    cp = L.CombineParams(8, 1024, 2, 16, 1e-6, 1)
    comb = lambda x1: L.lib.moe_combine_add_rmsnorm_tp2(ctypes.byref(cp), f, x1, f, f, None, f, f, f, None, None,
                                                        f, 256, None)
    assert comb(None) == L.MOE_ERR_INVALID_ARG
    assert comb(f8) == L.MOE_ERR_INVALID_ARG


def test_sources_up_to_twice_the_ranks(L):
    """With a TP domain of two ranks all 2 * ws devices are sources; more
    are refused."""
    n = ctypes.c_size_t(0)
    ok = L.DispatchParams(64, 1024, 4, 8, 32, 0, 0, 16)
    bad = L.DispatchParams(64, 1024, 4, 8, 32, 0, 0, 17)
    assert L.lib.moe_dispatch_workspace_size(ctypes.byref(ok), ctypes.byref(n)) == L.MOE_OK
    assert L.lib.moe_dispatch_workspace_size(ctypes.byref(bad), ctypes.byref(n)) == L.MOE_ERR_INVALID_ARG
