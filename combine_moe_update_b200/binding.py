"""Thin ctypes binding of libmoe_b200.so (include/moe_b200.h).

Argument marshalling only: tensors are checked for device, dtype and
contiguity, outputs are allocated with torch when the caller passes none,
and raw pointers plus the current CUDA stream go to the C ABI.  Every step
of the computation runs in the library's CUDA kernels; there is no CPU or
PyTorch fallback, and a missing or unloadable library raises at import.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import build as _build

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA = range(5)
DEV_BAD_ID, DEV_BAD_TABLE = 1, 2
WORKSPACE_BYTES = 256  # MOE_MAX_WORKSPACE_BYTES: serves every call


class MoeError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {_status_name(status)}")


class UpdateParams(ctypes.Structure):
    _fields_ = [("bs", ctypes.c_int32), ("top_k", ctypes.c_int32), ("num_logical", ctypes.c_int32),
                ("table_cols", ctypes.c_int32), ("ep_world_size", ctypes.c_int32),
                ("prune_threshold", ctypes.c_float), ("sources", ctypes.c_int32)]


class DispatchParams(ctypes.Structure):
    _fields_ = [("bs", ctypes.c_int32), ("hidden", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("ep_world_size", ctypes.c_int32), ("num_instances", ctypes.c_int32),
                ("quant_mode", ctypes.c_int32), ("scales_len", ctypes.c_int32), ("sources", ctypes.c_int32)]


class CombineParams(ctypes.Structure):
    _fields_ = [("bs", ctypes.c_int32), ("hidden", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("expand_rows", ctypes.c_int32), ("norm_eps", ctypes.c_float), ("sources", ctypes.c_int32)]


class EpParams(ctypes.Structure):
    _fields_ = [("bs", ctypes.c_int32), ("top_k", ctypes.c_int32), ("num_instances", ctypes.c_int32),
                ("gpus", ctypes.c_int32), ("rank", ctypes.c_int32), ("row_bytes", ctypes.c_int32),
                ("scale_bytes", ctypes.c_int32), ("recv_rows", ctypes.c_int32)]


class GmmParams(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int32), ("hidden", ctypes.c_int32), ("out_dim", ctypes.c_int32),
                ("num_instances", ctypes.c_int32)]


EXPORTS = (
    "moe_workspace_init", "moe_read_device_error", "moe_clear_device_error", "moe_status_string",
    "moe_update_expert_workspace_size", "moe_update_expert",
    "moe_dispatch_workspace_size", "moe_dispatch", "moe_dispatch_route", "moe_dispatch_tp_counts",
    "moe_combine_add_rmsnorm_workspace_size", "moe_combine_add_rmsnorm", "moe_combine_add_rmsnorm_tp2",
    "moe_combine",
    "moe_dispatch_noalloc", "moe_grouped_matmul_workspace_size", "moe_grouped_matmul", "moe_grouped_matmul_mx",
    "moe_ep_workspace_size", "moe_ep_plan", "moe_ep_push", "moe_ep_pull", "moe_ep_dispatch",
    "moe_ep_combine_add_rmsnorm",
    "moe_ipc_export", "moe_ipc_import", "moe_ipc_close",
)


def _load():
    path = _build.LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"libmoe_b200.so is not built ({path}); run combine_moe_update_b200.build")
    L = ctypes.CDLL(path)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    P = ctypes.POINTER
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_status_string.argtypes = [ctypes.c_int]
    L.moe_workspace_init.argtypes = [vp, sz, vp]
    L.moe_read_device_error.argtypes = [vp, P(ctypes.c_uint32), vp]
    L.moe_clear_device_error.argtypes = [vp, vp]
    L.moe_update_expert_workspace_size.argtypes = [P(UpdateParams), P(sz)]
    L.moe_update_expert.argtypes = [P(UpdateParams), vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_dispatch_workspace_size.argtypes = [P(DispatchParams), P(sz)]
    L.moe_dispatch.argtypes = [P(DispatchParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_combine_add_rmsnorm_workspace_size.argtypes = [P(CombineParams), P(sz)]
    L.moe_combine_add_rmsnorm.argtypes = [P(CombineParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_combine.argtypes = [P(CombineParams), vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_dispatch_noalloc.argtypes = [P(DispatchParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.moe_grouped_matmul_workspace_size.argtypes = [P(GmmParams), P(sz)]
    L.moe_grouped_matmul.argtypes = [P(GmmParams), vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_grouped_matmul_mx.argtypes = [P(GmmParams), vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_ep_workspace_size.argtypes = [P(EpParams), P(sz)]
    L.moe_ep_plan.argtypes = [P(EpParams), vp, vp, vp, vp, sz, vp]
    L.moe_ep_push.argtypes = [P(EpParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_ep_pull.argtypes = [P(EpParams), vp, vp, vp, vp, sz, vp]
    L.moe_dispatch_route.argtypes = [P(DispatchParams), vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_dispatch_tp_counts.argtypes = [P(DispatchParams), vp, vp, vp, vp, sz, vp]
    L.moe_combine_add_rmsnorm_tp2.argtypes = [P(CombineParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.moe_ep_dispatch.argtypes = [P(DispatchParams), P(EpParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                  vp]
    L.moe_ep_combine_add_rmsnorm.argtypes = [P(CombineParams), P(EpParams), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                             sz, vp]
    L.moe_ipc_export.argtypes = [vp, vp, P(ctypes.c_uint64)]
    L.moe_ipc_import.argtypes = [vp, ctypes.c_uint64, P(vp), P(vp)]
    L.moe_ipc_close.argtypes = [vp]
    for name in EXPORTS:
        if name != "moe_status_string":
            getattr(L, name).restype = ctypes.c_int
    return L


lib = _load()


def _status_name(s):
    return lib.moe_status_string(int(s)).decode()


def _check(fn, status):
    if status != MOE_OK:
        raise MoeError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _req(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _opt(t, name, dtype, shape=None):
    return None if t is None else _req(t, name, dtype, shape)


def _same_device(dev, *named):
    """Every tensor of a call lives on the device of its first input: the
    library launches on that device's current stream and looks per-device
    state up with that device current."""
    for name, t in named:
        if t is not None and t.device != dev:
            raise ValueError(f"{name} is on {t.device}, the call's inputs on {dev}")


def _check_dispatch_out(out, bs, hidden, top_k, num_instances, quant_mode):
    """A caller-supplied output dict must hold exactly what
    alloc_dispatch_outputs would allocate: the kernels write up to bs*K rows
    of expand_x and every entry through raw device pointers."""
    if not isinstance(out, dict):
        raise TypeError("out must be a dict like alloc_dispatch_outputs returns")
    rows = bs * top_k
    _req(out.get("expand_x"), "out['expand_x']", expand_dtype(quant_mode), (rows, hidden))
    ss = scales_shape(quant_mode, rows, hidden)
    if ss is None:
        if out.get("dyn_scales") is not None:
            raise ValueError(f"quant_mode {quant_mode} sends no scales: out['dyn_scales'] must be None")
    else:
        _req(out.get("dyn_scales"), "out['dyn_scales']", ss[1], ss[0])
    _req(out.get("expand_idx"), "out['expand_idx']", torch.int32, (bs, top_k))
    _req(out.get("src_of_row"), "out['src_of_row']", torch.int32, (rows,))
    _req(out.get("counts"), "out['counts']", torch.int32, (num_instances,))
    _req(out.get("offsets"), "out['offsets']", torch.int32, (num_instances + 1,))
    return out


def _check_combine_out(out, bs, hidden):
    if not isinstance(out, dict):
        raise TypeError("out must be a dict with y (and optionally x_out, rstd)")
    _req(out.get("y"), "out['y']", torch.bfloat16, (bs, hidden))
    _opt(out.get("x_out"), "out['x_out']", torch.bfloat16, (bs, hidden))
    _opt(out.get("rstd"), "out['rstd']", torch.float32, (bs,))
    return out


# --------------------------------------------------------------------------
# workspace / device errors
# --------------------------------------------------------------------------

def new_workspace(device=None, stream=None, nbytes=WORKSPACE_BYTES) -> torch.Tensor:
    """A zeroed workspace (holds the sticky device error word; dispatch with
    several source ranks may need more than the default, see
    dispatch_workspace_bytes)."""
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")
    with torch.cuda.device(ws.device):
        _check("moe_workspace_init", lib.moe_workspace_init(_ptr(ws), nbytes, _stream(stream)))
    return ws


def _per_source(tokens, sources, what):
    if sources < 1 or tokens % sources:
        raise ValueError(f"{what}: {tokens} tokens do not split over {sources} source ranks")
    return tokens // sources


def dispatch_workspace_bytes(bs, hidden, top_k, ep_world_size, num_instances, quant_mode, scales_len=0,
                             sources=1):
    """Workspace bytes moe_dispatch needs (bs = tokens per source rank)."""
    n = ctypes.c_size_t(0)
    p = DispatchParams(bs, hidden, top_k, int(ep_world_size), int(num_instances), int(quant_mode),
                       int(scales_len), int(sources))
    _check("moe_dispatch_workspace_size", lib.moe_dispatch_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return max(int(n.value), WORKSPACE_BYTES)


def read_device_error(workspace: torch.Tensor, stream=None) -> int:
    _req(workspace, "workspace", torch.uint8)
    bits = ctypes.c_uint32(0)
    with torch.cuda.device(workspace.device):
        _check("moe_read_device_error",
               lib.moe_read_device_error(_ptr(workspace), ctypes.byref(bits), _stream(stream)))
    return int(bits.value)


def clear_device_error(workspace: torch.Tensor, stream=None) -> None:
    _req(workspace, "workspace", torch.uint8)
    with torch.cuda.device(workspace.device):
        _check("moe_clear_device_error", lib.moe_clear_device_error(_ptr(workspace), _stream(stream)))


# --------------------------------------------------------------------------
# the three operations
# --------------------------------------------------------------------------

def update_expert(expert_ids, table, ep_world_size, expert_scales=None, active_mask=None,
                  prune_threshold=0.0, workspace=None, out=None, stream=None, sources=1):
    """moe_update_expert.  Returns (balanced_ids int32 [bs,K], balanced_mask uint8 [bs,K]).
    With sources = S the arrays hold S source ranks' tokens, rank-major."""
    _req(expert_ids, "expert_ids", torch.int32)
    bs, k = expert_ids.shape
    dev = expert_ids.device
    _req(table, "table", torch.int32)
    _opt(expert_scales, "expert_scales", torch.float32, (bs, k))
    _opt(active_mask, "active_mask", torch.uint8, (bs,))
    p = UpdateParams(_per_source(bs, sources, "update_expert"), k, table.shape[0], table.shape[1],
                     int(ep_world_size), float(prune_threshold), int(sources))
    if out is None:
        out = (torch.empty((bs, k), dtype=torch.int32, device=dev),
               torch.empty((bs, k), dtype=torch.uint8, device=dev))
    bal, bm = out
    _req(bal, "balanced_ids", torch.int32, (bs, k))
    _req(bm, "balanced_mask", torch.uint8, (bs, k))
    with torch.cuda.device(dev):
        ws = _req(workspace, "workspace", torch.uint8) if workspace is not None else new_workspace(dev, stream)
        _same_device(dev, ("table", table), ("expert_scales", expert_scales), ("active_mask", active_mask),
                     ("balanced_ids", bal), ("balanced_mask", bm), ("workspace", ws))
        _check("moe_update_expert", lib.moe_update_expert(
            ctypes.byref(p), _ptr(expert_ids), _ptr(expert_scales), _ptr(active_mask), _ptr(table),
            _ptr(bal), _ptr(bm), _ptr(ws), ws.numel(), _stream(stream)))
    return bal, bm


def expand_dtype(quant_mode):
    return {0: torch.bfloat16, 1: torch.int8, 2: torch.int8, 3: torch.int8, 4: torch.uint8}[quant_mode]


def scales_shape(quant_mode, rows, hidden):
    return {0: None, 1: None, 2: ((rows,), torch.float32), 3: ((rows, (hidden + 127) // 128), torch.float32),
            4: ((rows, hidden // 32), torch.uint8)}[quant_mode]


def _check_scales(smooth, quant_mode, num_instances, hidden):
    """quant_mode 1: static scales of shape (1,), (H,) or (E, H); modes 2/3:
    optional (E, H) smooth scales."""
    if quant_mode == 1:
        if smooth is None or smooth.dtype != torch.float32 or not smooth.is_contiguous() or \
                smooth.numel() not in (1, hidden, int(num_instances) * hidden):
            raise ValueError("quant_mode 1 needs float32 scales of shape (1,), (H,) or (num_instances, H)")
    else:
        _opt(smooth, "smooth", torch.float32, (num_instances, hidden))


def alloc_dispatch_outputs(bs, hidden, top_k, num_instances, quant_mode, device="cuda"):
    rows = bs * top_k
    ss = scales_shape(quant_mode, rows, hidden)
    return dict(
        expand_x=torch.empty((rows, hidden), dtype=expand_dtype(quant_mode), device=device),
        dyn_scales=None if ss is None else torch.empty(ss[0], dtype=ss[1], device=device),
        expand_idx=torch.empty((bs, top_k), dtype=torch.int32, device=device),
        src_of_row=torch.empty((rows,), dtype=torch.int32, device=device),
        counts=torch.empty((num_instances,), dtype=torch.int32, device=device),
        offsets=torch.empty((num_instances + 1,), dtype=torch.int32, device=device),
    )


def dispatch(x, instance_ids, num_instances, ep_world_size, quant_mode, mask=None, smooth=None,
             workspace=None, out=None, stream=None, sources=1):
    """moe_dispatch.  Returns a dict with expand_x, dyn_scales, expand_idx,
    src_of_row, counts and offsets (see include/moe_b200.h for layouts)."""
    _req(x, "x", torch.bfloat16)
    bs, H = x.shape
    dev = x.device
    _req(instance_ids, "instance_ids", torch.int32)
    k = instance_ids.shape[1]
    _req(instance_ids, "instance_ids", torch.int32, (bs, k))
    _opt(mask, "mask", torch.uint8, (bs, k))
    _check_scales(smooth, quant_mode, num_instances, H)
    if out is None:
        out = alloc_dispatch_outputs(bs, H, k, num_instances, quant_mode, dev)
    _check_dispatch_out(out, bs, H, k, num_instances, quant_mode)
    sl = 0 if smooth is None else smooth.numel()
    p = DispatchParams(_per_source(bs, sources, "dispatch"), H, k, int(ep_world_size), int(num_instances),
                       int(quant_mode), sl, int(sources))
    with torch.cuda.device(dev):
        ws = _req(workspace, "workspace", torch.uint8) if workspace is not None else new_workspace(
            dev, stream, dispatch_workspace_bytes(p.bs, H, k, ep_world_size, num_instances, quant_mode, sl,
                                                  sources))
        _same_device(dev, ("instance_ids", instance_ids), ("mask", mask), ("smooth", smooth), ("workspace", ws),
                     *((f"out['{n}']", t) for n, t in out.items()))
        _check("moe_dispatch", lib.moe_dispatch(
            ctypes.byref(p), _ptr(x), _ptr(instance_ids), _ptr(mask), _ptr(smooth), _ptr(out["expand_x"]),
            _ptr(out["dyn_scales"]), _ptr(out["expand_idx"]), _ptr(out["src_of_row"]), _ptr(out["counts"]),
            _ptr(out["offsets"]), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def dispatch_route(instance_ids, num_instances, ep_world_size, hidden, quant_mode, mask=None, scales_len=0,
                   workspace=None, out=None, stream=None):
    """moe_dispatch_route: the routing outputs of moe_dispatch (expand_idx,
    src_of_row, counts, offsets), no rows moved.  hidden, quant_mode and
    scales_len are the later moe_ep_dispatch's (they size the workspace)."""
    _req(instance_ids, "instance_ids", torch.int32)
    bs, k = instance_ids.shape
    dev = instance_ids.device
    _opt(mask, "mask", torch.uint8, (bs, k))
    rows = bs * k
    if out is None:
        out = dict(expand_idx=torch.empty((bs, k), dtype=torch.int32, device=dev),
                   src_of_row=torch.empty((rows,), dtype=torch.int32, device=dev),
                   counts=torch.empty((num_instances,), dtype=torch.int32, device=dev),
                   offsets=torch.empty((num_instances + 1,), dtype=torch.int32, device=dev))
    if not isinstance(out, dict):
        raise TypeError("out must be a dict with expand_idx, src_of_row, counts and offsets")
    _req(out.get("expand_idx"), "out['expand_idx']", torch.int32, (bs, k))
    _req(out.get("src_of_row"), "out['src_of_row']", torch.int32, (rows,))
    _req(out.get("counts"), "out['counts']", torch.int32, (num_instances,))
    _req(out.get("offsets"), "out['offsets']", torch.int32, (num_instances + 1,))
    p = DispatchParams(bs, int(hidden), k, int(ep_world_size), int(num_instances), int(quant_mode),
                       int(scales_len), 1)
    with torch.cuda.device(dev):
        ws = _req(workspace, "workspace", torch.uint8) if workspace is not None else new_workspace(
            dev, stream, dispatch_workspace_bytes(bs, hidden, k, ep_world_size, num_instances, quant_mode,
                                                  scales_len))
        _same_device(dev, ("mask", mask), ("workspace", ws), *((f"out['{n}']", t) for n, t in out.items()))
        _check("moe_dispatch_route", lib.moe_dispatch_route(
            ctypes.byref(p), _ptr(instance_ids), _ptr(mask), _ptr(out["expand_idx"]), _ptr(out["src_of_row"]),
            _ptr(out["counts"]), _ptr(out["offsets"]), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def combine_add_rmsnorm(expand_x, expand_idx, expert_scales, residual_x, gamma, norm_eps,
                        shared_x=None, want_x_out=False, want_rstd=False, workspace=None, out=None,
                        stream=None, sources=1):
    """moe_combine_add_rmsnorm.  Returns a dict with y (and x_out / rstd when asked)."""
    _req(expand_x, "expand_x", torch.bfloat16)
    rows, H = expand_x.shape
    dev = expand_x.device
    _req(expand_idx, "expand_idx", torch.int32)
    bs, k = expand_idx.shape
    _req(expert_scales, "expert_scales", torch.float32, (bs, k))
    _req(residual_x, "residual_x", torch.bfloat16, (bs, H))
    _req(gamma, "gamma", torch.bfloat16, (H,))
    _opt(shared_x, "shared_x", torch.bfloat16, (bs, H))
    if out is None:
        out = dict(y=torch.empty((bs, H), dtype=torch.bfloat16, device=dev),
                   x_out=torch.empty((bs, H), dtype=torch.bfloat16, device=dev) if want_x_out else None,
                   rstd=torch.empty((bs,), dtype=torch.float32, device=dev) if want_rstd else None)
    _check_combine_out(out, bs, H)
    p = CombineParams(_per_source(bs, sources, "combine_add_rmsnorm"), H, k, rows, float(norm_eps), int(sources))
    with torch.cuda.device(dev):
        ws = _req(workspace, "workspace", torch.uint8) if workspace is not None else new_workspace(dev, stream)
        _same_device(dev, ("expand_idx", expand_idx), ("expert_scales", expert_scales), ("residual_x", residual_x),
                     ("gamma", gamma), ("shared_x", shared_x), ("workspace", ws),
                     *((f"out['{n}']", t) for n, t in out.items()))
        _check("moe_combine_add_rmsnorm", lib.moe_combine_add_rmsnorm(
            ctypes.byref(p), _ptr(expand_x), _ptr(expand_idx), _ptr(expert_scales), _ptr(shared_x),
            _ptr(residual_x), _ptr(gamma), _ptr(out["y"]), _ptr(out.get("x_out")), _ptr(out.get("rstd")),
            _ptr(ws), ws.numel(), _stream(stream)))
    return out


def dispatch_tp_counts(route: dict, bs, hidden, top_k, ep_world_size, quant_mode, scales_len=0, workspace=None,
                       out=None, stream=None):
    """moe_dispatch_tp_counts: [E, 2] rows per (instance, TP domain) of a
    dispatch over 2 * ep_world_size TP-major sources with one instance per
    rank.  route: the dispatch's output dict (src_of_row, offsets)."""
    E = ep_world_size
    S = 2 * ep_world_size
    if not isinstance(route, dict):
        raise TypeError("route must be the dispatch's output dict")
    src, off = route.get("src_of_row"), route.get("offsets")
    _req(src, "route['src_of_row']", torch.int32, (S * bs * top_k,))
    _req(off, "route['offsets']", torch.int32, (E + 1,))
    dev = src.device
    if out is None:
        out = torch.empty((E, 2), dtype=torch.int32, device=dev)
    _req(out, "out", torch.int32, (E, 2))
    p = DispatchParams(int(bs), int(hidden), int(top_k), int(ep_world_size), E, int(quant_mode), int(scales_len), S)
    with torch.cuda.device(dev):
        ws = _req(workspace, "workspace", torch.uint8) if workspace is not None else new_workspace(dev, stream)
        _same_device(dev, ("route['offsets']", off), ("out", out), ("workspace", ws))
        _check("moe_dispatch_tp_counts", lib.moe_dispatch_tp_counts(
            ctypes.byref(p), _ptr(src), _ptr(off), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def combine_add_rmsnorm_tp2(expand_x0, expand_x1, expand_idx, expert_scales, residual_x, gamma, norm_eps,
                            shared_x=None, want_x_out=False, want_rstd=False, workspace=None, out=None,
                            stream=None, sources=1):
    """moe_combine_add_rmsnorm_tp2: the combine whose rows are the bf16 sums
    of the TP pair's two partial outputs.  Returns a dict like
    combine_add_rmsnorm.  Either partial may be given as an int: the device
    address, as this device dereferences it, of a [rows, H] bf16 buffer with
    the other's shape (another GPU's buffer mapped by ipc_import); a tensor
    partial sets the shape and the device."""
    peer0, peer1 = isinstance(expand_x0, int), isinstance(expand_x1, int)
    if peer0 and peer1:
        raise TypeError("at least one partial must be a tensor (it gives the shape and the device)")
    if peer0:  # the same call with the partials' roles swapped: the sum is symmetric
        expand_x0, expand_x1, peer1 = expand_x1, expand_x0, True
    _req(expand_x0, "expand_x0", torch.bfloat16)
    if peer1:
        if expand_x1 <= 0 or expand_x1 % 16:
            raise ValueError("a peer partial's address must be non-null and 16-byte aligned")
    else:
        _req(expand_x1, "expand_x1", torch.bfloat16, tuple(expand_x0.shape))
    rows, H = expand_x0.shape
    dev = expand_x0.device
    _req(expand_idx, "expand_idx", torch.int32)
    bs, k = expand_idx.shape
    _req(expert_scales, "expert_scales", torch.float32, (bs, k))
    _req(residual_x, "residual_x", torch.bfloat16, (bs, H))
    _req(gamma, "gamma", torch.bfloat16, (H,))
    _opt(shared_x, "shared_x", torch.bfloat16, (bs, H))
    if out is None:
        out = dict(y=torch.empty((bs, H), dtype=torch.bfloat16, device=dev),
                   x_out=torch.empty((bs, H), dtype=torch.bfloat16, device=dev) if want_x_out else None,
                   rstd=torch.empty((bs,), dtype=torch.float32, device=dev) if want_rstd else None)
    _check_combine_out(out, bs, H)
    p = CombineParams(_per_source(bs, sources, "combine_add_rmsnorm_tp2"), H, k, rows, float(norm_eps), int(sources))
    with torch.cuda.device(dev):
        ws = _req(workspace, "workspace", torch.uint8) if workspace is not None else new_workspace(dev, stream)
        _same_device(dev, ("expand_x1", None if peer1 else expand_x1), ("expand_idx", expand_idx),
                     ("expert_scales", expert_scales), ("residual_x", residual_x), ("gamma", gamma),
                     ("shared_x", shared_x), ("workspace", ws), *((f"out['{n}']", t) for n, t in out.items()))
        x1 = ctypes.c_void_p(expand_x1) if peer1 else _ptr(expand_x1)
        _check("moe_combine_add_rmsnorm_tp2", lib.moe_combine_add_rmsnorm_tp2(
            ctypes.byref(p), _ptr(expand_x0), x1, _ptr(expand_idx), _ptr(expert_scales),
            _ptr(shared_x), _ptr(residual_x), _ptr(gamma), _ptr(out["y"]), _ptr(out.get("x_out")),
            _ptr(out.get("rstd")), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def combine(expand_x, expand_idx, expert_scales, shared_x=None, workspace=None, out=None, stream=None, sources=1):
    """moe_combine (the plain CombineV2-series combine): combineOut [bs, H] bf16."""
    _req(expand_x, "expand_x", torch.bfloat16)
    rows, H = expand_x.shape
    dev = expand_x.device
    _req(expand_idx, "expand_idx", torch.int32)
    bs, k = expand_idx.shape
    _req(expert_scales, "expert_scales", torch.float32, (bs, k))
    _opt(shared_x, "shared_x", torch.bfloat16, (bs, H))
    if out is None:
        out = torch.empty((bs, H), dtype=torch.bfloat16, device=dev)
    _req(out, "out", torch.bfloat16, (bs, H))
    p = CombineParams(_per_source(bs, sources, "combine"), H, k, rows, 0.0, int(sources))
    with torch.cuda.device(dev):
        ws = _req(workspace, "workspace", torch.uint8) if workspace is not None else new_workspace(dev, stream)
        _same_device(dev, ("expand_idx", expand_idx), ("expert_scales", expert_scales), ("shared_x", shared_x),
                     ("out", out), ("workspace", ws))
        _check("moe_combine", lib.moe_combine(
            ctypes.byref(p), _ptr(expand_x), _ptr(expand_idx), _ptr(expert_scales), _ptr(shared_x), _ptr(out),
            _ptr(ws), ws.numel(), _stream(stream)))
    return out


def dispatch_noalloc(x, instance_ids, num_instances, ep_world_size, quant_mode, mask=None, smooth=None,
                     out=None, device_error=None, stream=None, sources=1):
    """moe_dispatch_noalloc: moe_dispatch with the library's own static scratch
    instead of a workspace.  device_error: optional int32 CUDA tensor of one
    element that receives the call's device error word."""
    _req(x, "x", torch.bfloat16)
    bs, H = x.shape
    dev = x.device
    _req(instance_ids, "instance_ids", torch.int32)
    k = instance_ids.shape[1]
    _req(instance_ids, "instance_ids", torch.int32, (bs, k))
    _opt(mask, "mask", torch.uint8, (bs, k))
    _check_scales(smooth, quant_mode, num_instances, H)
    _opt(device_error, "device_error", torch.int32, (1,))
    if out is None:
        out = alloc_dispatch_outputs(bs, H, k, num_instances, quant_mode, dev)
    _check_dispatch_out(out, bs, H, k, num_instances, quant_mode)
    _same_device(dev, ("instance_ids", instance_ids), ("mask", mask), ("smooth", smooth),
                 ("device_error", device_error), *((f"out['{n}']", t) for n, t in out.items()))
    p = DispatchParams(_per_source(bs, sources, "dispatch_noalloc"), H, k, int(ep_world_size),
                       int(num_instances), int(quant_mode), 0 if smooth is None else smooth.numel(), int(sources))
    with torch.cuda.device(dev):  # the library picks the scratch array of the current device
        _check("moe_dispatch_noalloc", lib.moe_dispatch_noalloc(
            ctypes.byref(p), _ptr(x), _ptr(instance_ids), _ptr(mask), _ptr(smooth), _ptr(out["expand_x"]),
            _ptr(out["dyn_scales"]), _ptr(out["expand_idx"]), _ptr(out["src_of_row"]), _ptr(out["counts"]),
            _ptr(out["offsets"]), _ptr(device_error), _stream(stream)))
    return out


def grouped_matmul_workspace_bytes(rows, hidden, out_dim, num_instances) -> int:
    p = GmmParams(int(rows), int(hidden), int(out_dim), int(num_instances))
    n = ctypes.c_size_t(0)
    _check("moe_grouped_matmul_workspace_size", lib.moe_grouped_matmul_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return n.value


def grouped_matmul(expand_x, dyn_scales, expert_offsets, weight, weight_scales, out=None, workspace=None,
                   stream=None):
    """moe_grouped_matmul: out[r] = (expand_x[r] . weight[e]^T) * dyn_scales[r] * weight_scales[e] for the
    rows r of each instance e, [expert_offsets[e], expert_offsets[e+1]).  expand_x [rows, H] int8,
    weight [E, N, H] int8, weight_scales [E, N] f32; returns out [rows, N] bf16 (rows outside the
    offsets keep whatever ``out`` held)."""
    _req(expand_x, "expand_x", torch.int8)
    rows, H = expand_x.shape
    _req(weight, "weight", torch.int8)
    E, N = weight.shape[0], weight.shape[1]
    _req(weight, "weight", torch.int8, (E, N, H))
    _req(weight_scales, "weight_scales", torch.float32, (E, N))
    _req(dyn_scales, "dyn_scales", torch.float32, (rows,))
    _req(expert_offsets, "expert_offsets", torch.int32, (E + 1,))
    if out is None:
        out = torch.empty((rows, N), dtype=torch.bfloat16, device=expand_x.device)
    _req(out, "out", torch.bfloat16, (rows, N))
    p = GmmParams(rows, H, N, E)
    dev = expand_x.device
    with torch.cuda.device(dev):
        ws = _req(workspace, "workspace", torch.uint8) if workspace is not None else new_workspace(
            dev, stream, grouped_matmul_workspace_bytes(rows, H, N, E))
        _same_device(dev, ("dyn_scales", dyn_scales), ("expert_offsets", expert_offsets), ("weight", weight),
                     ("weight_scales", weight_scales), ("out", out), ("workspace", ws))
        _check("moe_grouped_matmul", lib.moe_grouped_matmul(
            ctypes.byref(p), _ptr(expand_x), _ptr(dyn_scales), _ptr(expert_offsets), _ptr(weight),
            _ptr(weight_scales), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def grouped_matmul_mx(expand_x, x_sf, expert_offsets, weight, weight_sf, out=None, workspace=None, stream=None):
    """moe_grouped_matmul_mx: the instances' matmul on mxfp8 (E4M3 codes as uint8 with E8M0 block factors):
    expand_x [rows, H], x_sf [rows, H/32], weight [E, N, H], weight_sf [E, N, H/32]; returns out [rows, N]
    bf16."""
    _req(expand_x, "expand_x", torch.uint8)
    rows, H = expand_x.shape
    _req(weight, "weight", torch.uint8)
    E, N = weight.shape[0], weight.shape[1]
    _req(weight, "weight", torch.uint8, (E, N, H))
    _req(x_sf, "x_sf", torch.uint8, (rows, H // 32))
    _req(weight_sf, "weight_sf", torch.uint8, (E, N, H // 32))
    _req(expert_offsets, "expert_offsets", torch.int32, (E + 1,))
    if out is None:
        out = torch.empty((rows, N), dtype=torch.bfloat16, device=expand_x.device)
    _req(out, "out", torch.bfloat16, (rows, N))
    p = GmmParams(rows, H, N, E)
    dev = expand_x.device
    with torch.cuda.device(dev):
        ws = _req(workspace, "workspace", torch.uint8) if workspace is not None else new_workspace(
            dev, stream, grouped_matmul_workspace_bytes(rows, H, N, E))
        _same_device(dev, ("x_sf", x_sf), ("expert_offsets", expert_offsets), ("weight", weight),
                     ("weight_sf", weight_sf), ("out", out), ("workspace", ws))
        _check("moe_grouped_matmul_mx", lib.moe_grouped_matmul_mx(
            ctypes.byref(p), _ptr(expand_x), _ptr(x_sf), _ptr(expert_offsets), _ptr(weight), _ptr(weight_sf),
            _ptr(out), _ptr(ws), ws.numel(), _stream(stream)))
    return out


# --------------------------------------------------------------------------
# expert parallelism across GPUs (see combine_moe_update_b200/ep.py)
# --------------------------------------------------------------------------

IPC_HANDLE_BYTES = 64
DEV_CAPACITY = 8


def ep_row_bytes(quant_mode, hidden):
    """(row_bytes, scale_bytes) of a dispatched row in quant_mode."""
    return ((2 * hidden if quant_mode == 0 else hidden),
            {0: 0, 1: 0, 2: 4, 3: 4 * ((hidden + 127) // 128), 4: hidden // 32}[quant_mode])


def ep_params(bs, top_k, num_instances, gpus, rank, row_bytes, scale_bytes, recv_rows):
    return EpParams(int(bs), int(top_k), int(num_instances), int(gpus), int(rank), int(row_bytes),
                    int(scale_bytes), int(recv_rows))


def ep_workspace_bytes(p: EpParams) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_ep_workspace_size", lib.moe_ep_workspace_size(ctypes.byref(p), ctypes.byref(n)))
    return int(n.value)


def _ptr_table(t, name):
    """A [G] int64 CUDA tensor of device addresses (the pointer tables)."""
    return _req(t, name, torch.int64)


def ep_plan(p: EpParams, counts_all, recv_counts, recv_offsets, workspace, stream=None):
    G, E = p.gpus, p.num_instances
    _req(counts_all, "counts_all", torch.int32, (G, E))
    _req(recv_counts, "recv_counts", torch.int32, (E // G,))
    _req(recv_offsets, "recv_offsets", torch.int32, (E // G + 1,))
    _req(workspace, "workspace", torch.uint8)
    dev = counts_all.device
    _same_device(dev, ("recv_counts", recv_counts), ("recv_offsets", recv_offsets), ("workspace", workspace))
    with torch.cuda.device(dev):
        _check("moe_ep_plan", lib.moe_ep_plan(ctypes.byref(p), _ptr(counts_all), _ptr(recv_counts),
                                              _ptr(recv_offsets), _ptr(workspace), workspace.numel(),
                                              _stream(stream)))


def ep_push(p: EpParams, local: dict, instance_ids, peer_rows, peer_scales, peer_src, global_idx, workspace,
            stream=None):
    """local: moe_dispatch's outputs on this GPU (alloc_dispatch_outputs layout)."""
    rows = p.bs * p.top_k
    _req(local["expand_x"], "expand_x", local["expand_x"].dtype)
    if local["expand_x"].numel() * local["expand_x"].element_size() != rows * p.row_bytes:
        raise ValueError("expand_x does not hold bs * K rows of row_bytes")
    sc = local.get("dyn_scales")
    if p.scale_bytes:
        _req(sc, "dyn_scales", sc.dtype if sc is not None else torch.float32)
        if sc.numel() * sc.element_size() != rows * p.scale_bytes:
            raise ValueError("dyn_scales does not hold bs * K rows of scale_bytes")
        _ptr_table(peer_scales, "peer_scales")
    _req(local["offsets"], "offsets", torch.int32, (p.num_instances + 1,))
    _req(local["src_of_row"], "src_of_row", torch.int32, (rows,))
    _req(local["expand_idx"], "expand_idx", torch.int32, (p.bs, p.top_k))
    _req(instance_ids, "instance_ids", torch.int32, (p.bs, p.top_k))
    _req(global_idx, "global_idx", torch.int32, (p.bs, p.top_k))
    _ptr_table(peer_rows, "peer_rows")
    if peer_src is not None:
        _ptr_table(peer_src, "peer_src")
    dev = instance_ids.device
    with torch.cuda.device(dev):
        _check("moe_ep_push", lib.moe_ep_push(
            ctypes.byref(p), _ptr(local["expand_x"]), _ptr(sc if p.scale_bytes else None), _ptr(local["offsets"]),
            _ptr(local["src_of_row"]), _ptr(local["expand_idx"]), _ptr(instance_ids), _ptr(peer_rows),
            _ptr(peer_scales if p.scale_bytes else None), _ptr(peer_src), _ptr(global_idx), _ptr(workspace),
            workspace.numel(), _stream(stream)))


def ep_pull(p: EpParams, peer_rows, local_offsets, local_rows, workspace, stream=None):
    _ptr_table(peer_rows, "peer_rows")
    _req(local_offsets, "local_offsets", torch.int32, (p.num_instances + 1,))
    _req(local_rows, "local_rows", local_rows.dtype)
    if local_rows.numel() * local_rows.element_size() != p.bs * p.top_k * p.row_bytes:
        raise ValueError("local_rows does not hold bs * K rows of row_bytes")
    with torch.cuda.device(local_rows.device):
        _check("moe_ep_pull", lib.moe_ep_pull(ctypes.byref(p), _ptr(peer_rows), _ptr(local_offsets),
                                              _ptr(local_rows), _ptr(workspace), workspace.numel(),
                                              _stream(stream)))


def ep_dispatch(p: EpParams, x, instance_ids, ep_world_size, quant_mode, route: dict, peer_rows, peer_scales,
                peer_src, global_idx, workspace, mask=None, smooth=None, stream=None):
    """moe_ep_dispatch: quantize this GPU's tokens and store every sent copy
    into its owner's receive buffer.  route: dispatch_route's outputs."""
    _req(x, "x", torch.bfloat16)
    if x.dim() != 2 or x.shape[0] != p.bs:
        raise ValueError(f"x must have shape ({p.bs}, H), got {tuple(x.shape)}")
    H = x.shape[1]
    dev = x.device
    _req(instance_ids, "instance_ids", torch.int32, (p.bs, p.top_k))
    _opt(mask, "mask", torch.uint8, (p.bs, p.top_k))
    _check_scales(smooth, quant_mode, p.num_instances, H)
    if not isinstance(route, dict):
        raise TypeError("route must be dispatch_route's output dict")
    _req(route.get("expand_idx"), "route['expand_idx']", torch.int32, (p.bs, p.top_k))
    _req(route.get("offsets"), "route['offsets']", torch.int32, (p.num_instances + 1,))
    _req(global_idx, "global_idx", torch.int32, (p.bs, p.top_k))
    _ptr_table(peer_rows, "peer_rows")
    if p.scale_bytes:
        _ptr_table(peer_scales, "peer_scales")
    if peer_src is not None:
        _ptr_table(peer_src, "peer_src")
    _req(workspace, "workspace", torch.uint8)
    sl = 0 if smooth is None else smooth.numel()
    dp = DispatchParams(p.bs, H, p.top_k, int(ep_world_size), p.num_instances, int(quant_mode), sl, 1)
    _same_device(dev, ("instance_ids", instance_ids), ("mask", mask), ("smooth", smooth),
                 ("route['expand_idx']", route["expand_idx"]), ("route['offsets']", route["offsets"]),
                 ("global_idx", global_idx), ("peer_rows", peer_rows), ("peer_scales", peer_scales),
                 ("peer_src", peer_src), ("workspace", workspace))
    with torch.cuda.device(dev):
        _check("moe_ep_dispatch", lib.moe_ep_dispatch(
            ctypes.byref(dp), ctypes.byref(p), _ptr(x), _ptr(instance_ids), _ptr(mask), _ptr(smooth),
            _ptr(route["expand_idx"]), _ptr(route["offsets"]), _ptr(peer_rows),
            _ptr(peer_scales if p.scale_bytes else None), _ptr(peer_src), _ptr(global_idx), _ptr(workspace),
            workspace.numel(), _stream(stream)))


def ep_combine_add_rmsnorm(p: EpParams, peer_rows, global_idx, expert_scales, residual_x, gamma, norm_eps,
                           workspace, shared_x=None, want_x_out=False, want_rstd=False, out=None, stream=None):
    """moe_ep_combine_add_rmsnorm: the combine reading each copy's expert
    output from the GPU that owns its row.  Returns a dict like
    combine_add_rmsnorm."""
    _ptr_table(peer_rows, "peer_rows")
    _req(global_idx, "global_idx", torch.int32, (p.bs, p.top_k))
    _req(residual_x, "residual_x", torch.bfloat16)
    H = residual_x.shape[1]
    _req(residual_x, "residual_x", torch.bfloat16, (p.bs, H))
    dev = residual_x.device
    _req(expert_scales, "expert_scales", torch.float32, (p.bs, p.top_k))
    _req(gamma, "gamma", torch.bfloat16, (H,))
    _opt(shared_x, "shared_x", torch.bfloat16, (p.bs, H))
    _req(workspace, "workspace", torch.uint8)
    if out is None:
        out = dict(y=torch.empty((p.bs, H), dtype=torch.bfloat16, device=dev),
                   x_out=torch.empty((p.bs, H), dtype=torch.bfloat16, device=dev) if want_x_out else None,
                   rstd=torch.empty((p.bs,), dtype=torch.float32, device=dev) if want_rstd else None)
    _check_combine_out(out, p.bs, H)
    cp = CombineParams(p.bs, H, p.top_k, max(p.recv_rows, 1), float(norm_eps), 1)
    _same_device(dev, ("peer_rows", peer_rows), ("global_idx", global_idx), ("expert_scales", expert_scales),
                 ("gamma", gamma), ("shared_x", shared_x), ("workspace", workspace),
                 *((f"out['{n}']", t) for n, t in out.items()))
    with torch.cuda.device(dev):
        _check("moe_ep_combine_add_rmsnorm", lib.moe_ep_combine_add_rmsnorm(
            ctypes.byref(cp), ctypes.byref(p), _ptr(peer_rows), _ptr(global_idx), _ptr(expert_scales),
            _ptr(shared_x), _ptr(residual_x), _ptr(gamma), _ptr(out["y"]), _ptr(out.get("x_out")),
            _ptr(out.get("rstd")), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def ipc_export(t: torch.Tensor):
    """(handle bytes, offset) for a CUDA tensor's memory, for moe_ipc_import in another process."""
    h = (ctypes.c_uint8 * IPC_HANDLE_BYTES)()
    off = ctypes.c_uint64(0)
    with torch.cuda.device(t.device):
        _check("moe_ipc_export", lib.moe_ipc_export(_ptr(t), h, ctypes.byref(off)))
    return bytes(h), int(off.value)


def ipc_import(handle: bytes, offset: int):
    """(base, device address) of a peer's exported memory, mapped on the current device."""
    h = (ctypes.c_uint8 * IPC_HANDLE_BYTES).from_buffer_copy(handle)
    base, ptr = ctypes.c_void_p(), ctypes.c_void_p()
    _check("moe_ipc_import", lib.moe_ipc_import(h, ctypes.c_uint64(offset), ctypes.byref(base), ctypes.byref(ptr)))
    return base.value, ptr.value


def ipc_close(base: int):
    _check("moe_ipc_close", lib.moe_ipc_close(ctypes.c_void_p(base)))
