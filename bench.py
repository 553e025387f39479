#!/usr/bin/env python
"""MoE dispatch+combine throughput on B200: tokens/s and achieved HBM GB/s.

One step = one MoE layer's hot path on one batch of seeded synthetic input:
moe_update_expert -> moe_dispatch -> moe_combine_add_rmsnorm (the expert FFN
between dispatch and combine is stood in for by a resident buffer of bf16
expert-output rows).  The step's inputs are cold in L2 when it starts: where
a few input sets (activations and the layer's parameters) together exceed
twice L2, the timed steps cycle through them back to back with events only
at the ends of each graph; smaller workloads flush L2 (512 MiB written, then
256 MiB read) before every step, outside the timed events.  `config.l2` says
which.  The line also carries the gate figure -- dispatch + combine alone,
pairs back to back over the cold sets -- and each kernel's roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl b200|reference]

`--workload layer_stack` times 32 chained layers captured in one CUDA graph.

With N > 1 it runs under torch.distributed.run, one process per GPU; the
path has no exchange step on one GPU, so every rank runs an independent
replica on its own batch (weak scaling, no data-path collective) and the
reported value is the tokens of all ranks over the slowest rank's time.
`--impl reference` times the plain CPU oracle on this host instead.
"""
from __future__ import annotations

import argparse
import functools
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "deepseek_decode_bs512"
METRIC = "MoE dispatch+combine tokens/s (1 B200; HBM GB/s vs peak in roofline)"
L2_FLUSH_BYTES = 512 << 20
L2_BYTES = 126 * 2**20  # B200 L2
FALLBACK_HBM_GBS = 6650.0


# --------------------------------------------------------------------------
# algorithmic bytes: what each operation must move at minimum
# --------------------------------------------------------------------------

def algorithmic_bytes(w, n, x_out=False, rstd=False):
    """Bytes each op must read + write for workload `w` with `n` kept copies.
    Pruned copies are not counted (the method skips them)."""
    bs, H, K, E = w.bs, w.hidden, w.top_k, w.num_instances
    items = bs * K
    upd = items * (4 + 4 + 4 + 1) + (4 if w.prune_threshold > 0 else 0) + 2 * 4 * w.num_logical
    code = 2 if w.quant_mode == 0 else 1
    sc = {0: 0, 1: 0, 2: 4, 3: 4 * ((H + 127) // 128), 4: H // 32}[w.quant_mode]
    scale_bytes = 0  # smooth rows of the instances hit, or the static scales
    if w.smooth is not None:
        if w.smooth.size in (1, H):
            scale_bytes = 4 * w.smooth.size
        else:
            scale_bytes = 4 * H * len(set(map(int, w.meta.get("distinct_instances", []))))
    disp = (2 * bs * H                      # x
            + scale_bytes                   # smooth / static scales read
            + n * (H * code + sc)           # codes + scales of every kept copy
            + items * (4 + 1)               # instance ids + mask
            + items * 4 + n * 4             # expand_idx + src_of_row
            + 4 * E + 4 * (E + 1))          # counts + offsets
    if int(w.meta.get("tp", 1)) == 2:       # the per-(rank, domain) counts
        disp += 4 * (E + 1) + 8 * E
    comb = (n * 2 * H * int(w.meta.get("tp", 1))  # expert rows gathered back (both TP partials)
            + 2 * bs * H                    # residual
            + (2 * bs * H if w.shared_x is not None else 0)
            + 2 * H                         # gamma
            + 2 * bs * H                    # y
            + (2 * bs * H if x_out else 0) + (4 * bs if rstd else 0)
            + items * (4 + 4))              # expand_idx + scales
    return dict(update=upd, dispatch=disp, combine=comb)


def kernels_per_step(w):
    """Kernels of this library one step launches: update_expert, the
    dispatch's kernels, the combine.  Up to 1024 copies the scatter blocks
    route themselves, up to 8192 one route kernel runs first, and beyond that
    the three-pass route."""
    copies = w.bs * w.top_k
    if copies > 8192:
        disp = 4
    elif copies <= 1024:
        disp = 1
    else:
        disp = 2
    if int(w.meta.get("tp", 1)) == 2:
        disp += 1  # the per-(rank, domain) counts
    return 1 + disp + 1


# The sources a kernel is compiled from: stored ncu counters are kept while
# these files are unchanged.
KERNEL_SOURCES = {
    "combine_token_kernel": ("combine.cuh", "common.cuh"),
    "dispatch_token_smooth_kernel": ("dispatch.cuh", "common.cuh"),
    "dispatch_token_kernel": ("dispatch.cuh", "common.cuh"),
    "gmm_kernel": ("grouped_matmul.cuh", "common.cuh"),
    "gmm_mx_kernel": ("grouped_matmul.cuh", "common.cuh"),
    # the EP instantiations (rows stored to / read from their owners), one-GPU group
    "dispatch_token_smooth_kernel_ep": ("dispatch.cuh", "common.cuh"),
    "combine_token_kernel_ep": ("combine.cuh", "common.cuh"),
}


def source_hash(kernel):
    """Hash of the CUDA sources of `kernel`, to tell whether stored ncu
    counters still describe the kernel being timed."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "combine_moe_update_b200", "csrc")
    for fn in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current sources of the kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(p))[f"{kernel}@{workload}"]
    except (OSError, KeyError, ValueError):
        return None
    return rec.get("dram_bytes_per_launch") if rec.get("source_hash") == source_hash(kernel) else None


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return float(json.load(open(p))["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# --------------------------------------------------------------------------
# clocks during the timed region (read-only NVML queries)
# --------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, device_index, period_s=0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report no samples
            self.nv = None

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_r(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr is not None:
            self._thr.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------
# distributed plumbing (host side; covered by gloo tests)
# --------------------------------------------------------------------------

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def reduce_over_ranks(values, op):
    """Element-wise max / sum of a list of floats over all ranks (identity
    when torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor(list(values), dtype=torch.float64, device=dev)
    dist.all_reduce(t, op={"max": dist.ReduceOp.MAX, "sum": dist.ReduceOp.SUM}[op])
    return t.cpu().tolist()


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# --------------------------------------------------------------------------
# the B200 arm
# --------------------------------------------------------------------------

def run_b200(args, rank, world, local_rank):
    import numpy as np
    import torch
    from combine_moe_update_b200 import binding as B
    from combine_moe_update_b200 import inputs as gen

    torch.cuda.set_device(local_rank)
    w = gen.make(args.workload, seed=None if rank == 0 else 1000 + rank)
    if "expert_out_dim" in w.meta:
        return run_b200_expert(args, rank, world, local_rank, w)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    bf = lambda a: dev(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(torch.bfloat16)

    # resident parameters of the layer
    table = dev(w.table)
    smooth = None if w.smooth is None else dev(w.smooth)
    gamma = bf(w.gamma)
    # this batch's activations
    ids, scales = dev(w.expert_ids), dev(w.expert_scales)
    # several source ranks (every simulated rank sends its own tokens); a TP
    # pair's two partial expert outputs of every row as one [2, rows, H] tensor
    S = int(w.meta.get("sources", 1))
    TP = int(w.meta.get("tp", 1))
    x, residual = bf(w.x), bf(w.residual)
    expert_out = bf(w.expert_out) if TP == 1 else bf(np.stack([w.expert_out, w.meta["expert_out_tp1"]]))
    shared = None if w.shared_x is None else bf(w.shared_x)
    upd = functools.partial(B.update_expert, sources=S)
    if TP == 1:
        disp = functools.partial(B.dispatch, sources=S)
        comb = functools.partial(B.combine_add_rmsnorm, sources=S)
    else:
        tpc = torch.empty((w.num_instances, 2), dtype=torch.int32, device="cuda")
        tp_sl = 0 if w.smooth is None else w.smooth.size

        def disp(xx, *a, **k):  # the dispatch over the TP-major sources, then the per-(rank, domain) counts
            o = B.dispatch(xx, *a, sources=S, **k)
            B.dispatch_tp_counts(o, w.bs // S, w.hidden, w.top_k, w.ep_world_size, w.quant_mode, scales_len=tp_sl,
                                 workspace=k.get("workspace"), out=tpc)
            return o

        def comb(ee, *a, **k):  # the ReduceScatterV of the two partials fused into the gather
            return B.combine_add_rmsnorm_tp2(ee[0], ee[1], *a, sources=S, **k)
    ws = B.new_workspace(nbytes=B.dispatch_workspace_bytes(
        w.bs // S, w.hidden, w.top_k, w.ep_world_size, w.num_instances, w.quant_mode,
        0 if w.smooth is None else w.smooth.size, S))
    bal = torch.empty_like(ids)
    bm = torch.empty(ids.shape, dtype=torch.uint8, device="cuda")
    d = B.alloc_dispatch_outputs(w.bs, w.hidden, w.top_k, w.num_instances, w.quant_mode)
    c = dict(y=torch.empty_like(x), x_out=None, rstd=None)

    def step(xx=x, ii=ids, ss=scales, rr=residual, ee=expert_out, sh=shared):
        upd(ii, table, w.ep_world_size, expert_scales=ss, prune_threshold=w.prune_threshold,
                        workspace=ws, out=(bal, bm))
        disp(xx, bal, w.num_instances, w.ep_world_size, w.quant_mode, mask=bm, smooth=smooth,
                   workspace=ws, out=d)
        comb(ee, d["expand_idx"], ss, rr, gamma, w.norm_eps, shared_x=sh, workspace=ws, out=c)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    clean = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.float32, device="cuda")  # 256 MiB

    def flush_l2():
        # overwrite 512 MiB, then read 256 MiB: L2 then holds neither the step's
        # inputs nor dirty lines whose write-back would land in the timed step
        flush.zero_()
        clean.sum()

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()
    assert B.read_device_error(ws) == 0, "device error during warm-up"
    n = int(d["offsets"][-1].item())
    w.meta["distinct_instances"] = torch.unique(bal[bm.bool()]).cpu().tolist() if smooth is not None else []
    alg = algorithmic_bytes(w, n)

    # Timed region: CUDA graphs of G steps each, every step = [L2 flush] then
    # update_expert, dispatch and combine between two timing events recorded
    # as graph nodes; the flush sits outside the bracket.  Nothing separates
    # the three calls, so each kernel's launch overlaps its predecessor's
    # tail (programmatic dependent launch), as in a real layer.
    # A second graph brackets every call with its own events for the per-call
    # breakdown and the combine kernel's roofline; an event between two calls
    # ends that overlap, so the three call times add up to more than a step.
    K = args.steps
    G = max(g for g in range(1, 17) if K % g == 0)
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())

    def capture(per_call):
        evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4 if per_call else 2)]
               for _ in range(G)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for e in evs:
                flush_l2()
                e[0].record()
                upd(ids, table, w.ep_world_size, expert_scales=scales,
                                prune_threshold=w.prune_threshold, workspace=ws, out=(bal, bm))
                if per_call:
                    e[1].record()
                disp(x, bal, w.num_instances, w.ep_world_size, w.quant_mode, mask=bm, smooth=smooth,
                           workspace=ws, out=d)
                if per_call:
                    e[2].record()
                comb(expert_out, d["expand_idx"], scales, residual, gamma, w.norm_eps,
                                      shared_x=shared, workspace=ws, out=c)
                e[-1].record()
        return g, evs

    # The timed steps: when a handful of input sets (activations and the
    # layer's own parameters: table, smooth scales, gamma) together exceed
    # twice L2, the G steps of a graph cycle through them back to back -- the
    # next step's inputs are always cold, as for consecutive layers -- with
    # events only at the graph's ends, so no event or flush sits between
    # steps.  Otherwise every step gets the L2 flush and its own events.
    act = [x, ids, scales, residual, expert_out, shared, table, smooth, gamma]
    per_set = sum(t.numel() * t.element_size() for t in act if t is not None)
    R = -(-(2 * L2_BYTES) // per_set) + 1
    cold_sets = R <= 16 and G >= R
    if cold_sets:
        sets = [[None if t is None else t.clone() for t in act] for _ in range(R)]
        ev_cold = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=cap):
            ev_cold[0].record()
            for s_ in range(G):
                xx, ii, ss, rr, ee, sh, tb, sm, gm = sets[s_ % R]
                upd(ii, tb, w.ep_world_size, expert_scales=ss, prune_threshold=w.prune_threshold,
                                workspace=ws, out=(bal, bm))
                disp(xx, bal, w.num_instances, w.ep_world_size, w.quant_mode, mask=bm, smooth=sm,
                           workspace=ws, out=d)
                comb(ee, d["expand_idx"], ss, rr, gm, w.norm_eps, shared_x=sh, workspace=ws,
                                      out=c)
            ev_cold[1].record()
        l2_note = (f"not flushed: {R} input sets of {per_set / 2**20:.0f} MiB (activations and layer parameters) "
                   f"cycled back to back, {R * per_set / 2**20:.0f} MiB > 2 x L2; events only at each "
                   f"{G}-step graph's ends")
    else:
        graph, ev_step = capture(False)
        l2_note = "flushed before every timed step: 512 MiB written, then 256 MiB read; events around each step"
    graph_ops, ev_ops = capture(True)
    for g in (graph, graph_ops):
        g.replay()  # one untimed replay after capture
    torch.cuda.synchronize()
    sums = [0.0, 0.0, 0.0, 0.0]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for _ in range(K // G):
            graph.replay()
            torch.cuda.synchronize()
            if cold_sets:
                sums[0] += ev_cold[0].elapsed_time(ev_cold[1])
            else:
                for e in ev_step:
                    sums[0] += e[0].elapsed_time(e[1])
        barrier()
        torch.cuda.synchronize()
        for _ in range(K // G):
            graph_ops.replay()
            torch.cuda.synchronize()
            for e in ev_ops:
                sums[1] += e[0].elapsed_time(e[1])
                sums[2] += e[1].elapsed_time(e[2])
                sums[3] += e[2].elapsed_time(e[3])
    barrier()
    del graph, graph_ops
    assert B.read_device_error(ws) == 0, "device error during the timed steps"

    def time_graph(body, count):
        """Per-body time (ms): `body` captured `count` times in one graph with
        events only at its ends, replayed a few times."""
        eb = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            eb[0].record()
            for n_ in range(count):
                body(n_)
            eb[1].record()
        g.replay()
        torch.cuda.synchronize()
        reps = max(3, min(50, K // 4))
        tot = 0.0
        for _ in range(reps):
            g.replay()
            torch.cuda.synchronize()
            tot += eb[0].elapsed_time(eb[1]) / count
        del g
        return tot / reps

    # The gate (dispatch + combine alone): pairs back to back over the cold
    # input sets, each set's routing (update_expert's output) computed once
    # beforehand, events only at the graph's ends, so each pair overlaps its
    # predecessor's tail as consecutive layers would.
    t_pair = None
    if cold_sets:
        routes = []
        for xx, ii, ss, rr, ee, sh, tb, sm, gm in sets:
            rb, rm = torch.empty_like(bal), torch.empty_like(bm)
            upd(ii, tb, w.ep_world_size, expert_scales=ss, prune_threshold=w.prune_threshold, workspace=ws,
                out=(rb, rm))
            routes.append((rb, rm))

        def pair(n_):
            (xx, ii, ss, rr, ee, sh, tb, sm, gm), (rb, rm) = sets[n_ % R], routes[n_ % R]
            disp(xx, rb, w.num_instances, w.ep_world_size, w.quant_mode, mask=rm, smooth=sm, workspace=ws, out=d)
            comb(ee, d["expand_idx"], ss, rr, gm, w.norm_eps, shared_x=sh, workspace=ws, out=c)

        t_pair = time_graph(pair, R * max(1, 16 // R))
        del routes
        assert B.read_device_error(ws) == 0, "device error during the gate pairs"
        gate_timing = (f"{R * max(1, 16 // R)} dispatch+combine pairs back to back over {R} input sets "
                       f"({R * per_set / 2**20:.0f} MiB > 2 x L2), routing computed beforehand, CUDA events around "
                       "the whole run")
    if cold_sets:
        del sets

    # Each kernel on its own for the roofline: launches back to back (each a
    # programmatic dependent of the one before, as in consecutive layers)
    # over input sets whose total exceeds twice L2, so every launch reads
    # cold inputs and no event sits between launches; time per launch = the
    # span / count.  Workloads too small for that use the event-bracketed
    # call of the breakdown graph instead, and say so.
    def cold_copies(tensors):
        per = sum(t.numel() * t.element_size() for t in tensors if t is not None)
        n_ = -(-(2 * L2_BYTES) // per) + 1
        return n_, per

    R_c, per_c = cold_copies((expert_out, residual, shared))
    if R_c <= 16:
        csets = [[None if t is None else t.clone() for t in (expert_out, residual, shared)] for _ in range(R_c)]
        t_comb_kernel = time_graph(
            lambda n_: comb(csets[n_ % R_c][0], d["expand_idx"], scales, csets[n_ % R_c][1], gamma, w.norm_eps,
                            shared_x=csets[n_ % R_c][2], workspace=ws, out=c), R_c * max(1, 16 // R_c))
        del csets
        comb_timing = (f"{R_c * max(1, 16 // R_c)} back-to-back launches over {R_c} input sets "
                       f"({R_c * per_c / 2**20:.0f} MiB > 2 x L2), CUDA events around the whole run")
    else:
        t_comb_kernel = sums[3] / K
        comb_timing = "per-call CUDA events in the breakdown graph (inputs too small to exceed L2 in a few sets)"

    R_d, per_d = cold_copies((x, smooth, bal, bm))
    if R_d <= 32:
        # copies of x, the scale rows and the routing (bal, bm hold this batch's)
        dsets = [[None if t is None else t.clone() for t in (x, smooth, bal, bm)] for _ in range(R_d)]
        t_disp_kernel = time_graph(
            lambda n_: disp(dsets[n_ % R_d][0], dsets[n_ % R_d][2], w.num_instances, w.ep_world_size, w.quant_mode,
                            mask=dsets[n_ % R_d][3], smooth=dsets[n_ % R_d][1], workspace=ws, out=d),
            R_d * max(1, 32 // R_d))
        del dsets
        disp_timing = (f"{R_d * max(1, 32 // R_d)} back-to-back calls over {R_d} input sets "
                       f"({R_d * per_d / 2**20:.0f} MiB > 2 x L2), CUDA events around the whole run")
    else:
        t_disp_kernel = sums[2] / K
        disp_timing = "per-call CUDA events in the breakdown graph (inputs too small to exceed L2 in a few sets)"
    assert B.read_device_error(ws) == 0, "device error during the roofline launches"

    t_step, t_upd, t_disp, t_comb, t_comb_kernel, t_disp_kernel, t_pair = reduce_over_ranks(
        [v / K for v in sums] + [t_comb_kernel, t_disp_kernel, t_pair if t_pair is not None else 0.0], "max")
    value = world * w.bs / (t_step * 1e-3)

    # ---- end to end through the public API with host buffers ----
    pin = lambda t: t.cpu().pin_memory()
    h_in = dict(x=pin(x), ids=pin(ids), scales=pin(scales), residual=pin(residual), expert_out=pin(expert_out))
    if shared is not None:
        h_in["shared"] = pin(shared)
    d_in = dict(x=torch.empty_like(x), ids=torch.empty_like(ids), scales=torch.empty_like(scales),
                residual=torch.empty_like(residual), expert_out=torch.empty_like(expert_out),
                shared=None if shared is None else torch.empty_like(shared))
    h_y = torch.empty(c["y"].shape, dtype=c["y"].dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in h_in.values())
    d2h = h_y.numel() * h_y.element_size()

    def e2e_step():
        for k_, t in h_in.items():
            d_in[k_].copy_(t, non_blocking=True)
        step(d_in["x"], d_in["ids"], d_in["scales"], d_in["residual"], d_in["expert_out"], d_in["shared"])
        h_y.copy_(c["y"], non_blocking=True)

    for _ in range(max(3, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ke = max(10, min(K, 200))
    e0.record()
    for _ in range(ke):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    (t_e2e,) = reduce_over_ranks([e0.elapsed_time(e1) / ke], "max")

    peak, peak_kind = measured_peak()
    per_instance = w.smooth is not None and w.smooth.size > w.hidden
    disp_name = "dispatch_token_smooth_kernel" if per_instance else "dispatch_token_kernel"

    def roof(kernel, nbytes, t_ms, timing, traffic_key):
        a = nbytes / (t_ms * 1e-3) / 1e9
        return {"bound": "hbm", "kernel": kernel, "achieved": round(a, 1), "peak": peak, "peak_kind": peak_kind,
                "unit": "GB/s", "frac": round(a / peak, 4), "launch_us": round(t_ms * 1e3, 2), "timing": timing,
                "traffic": stored_traffic(traffic_key, args.workload) if traffic_key else None,
                "algorithmic_bytes": nbytes}

    r_comb = roof("combine_token_kernel", alg["combine"], t_comb_kernel, comb_timing, "combine_token_kernel")
    r_disp = roof(disp_name, alg["dispatch"], t_disp_kernel, disp_timing,
                  disp_name if disp_name in KERNEL_SOURCES else None)
    r_disp["note"] = ("the whole moe_dispatch call: one kernel that routes its own copies"
                      if kernels_per_step(w) == 3 else "the whole moe_dispatch call (route and scatter kernels)")
    # the dominant kernel by time carries the line's roofline
    roofline, other = (r_comb, r_disp) if t_comb_kernel >= t_disp_kernel else (r_disp, r_comb)
    step_gbs = (alg["update"] + alg["dispatch"] + alg["combine"]) / (t_step * 1e-3) / 1e9
    gate = None
    if t_pair:
        gb = (alg["dispatch"] + alg["combine"]) / (t_pair * 1e-3) / 1e9
        gate = {"us": round(t_pair * 1e3, 2), "tokens_per_s": round(world * w.bs / (t_pair * 1e-3), 1),
                "hbm_gbs": round(gb, 1), "frac_of_peak": round(gb / peak, 4),
                "algorithmic_bytes": alg["dispatch"] + alg["combine"], "timing": gate_timing}
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(t_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": {0: "bf16", 1: "int8", 2: "int8", 3: "int8", 4: "fp8e4m3"}[w.quant_mode] + "+fp32",
        "data": "synthetic (seeded; pages' shapes)",
        "config": {"workload": args.workload, "bs": w.bs, "hidden": w.hidden, "top_k": w.top_k,
                   "num_instances": w.num_instances, "ep_world_size_simulated": w.ep_world_size,
                   "quant_mode": w.quant_mode, "smooth_scales": w.smooth is not None,
                   "shared_expert": w.shared_x is not None, "kept_copies": n, "source_ranks": S,
                   "tp_world_size": TP, "l2": l2_note, "parallelism": f"replicas x{world}"},
        "gate": gate,
        "breakdown_us": {"update_expert": round(t_upd * 1e3, 2), "dispatch": round(t_disp * 1e3, 2),
                         "combine": round(t_comb * 1e3, 2),
                         "note": "each call bracketed by its own events (about 4.5 us each, no launch overlap)"},
        "achieved_gbs": {"step": round(step_gbs, 1), "dispatch": r_disp["achieved"], "combine": r_comb["achieved"]},
        "roofline": roofline,
        "roofline_other": other,
        "e2e": {"value": round(world * w.bs / (t_e2e * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "pinned host activations -> device, the three calls, y -> host; layer parameters resident"},
        "gpu_launches": kernels_per_step(w) * K,
        "timing": (f"CUDA graphs of {G} steps; breakdown_us from a second graph with the L2 flush before each step "
                   "and events between the calls (no launch overlap there, so its parts sum above a step)"),
        "clocks": clk.summary(),
    }
    return out, w


def run_b200_layer_stack(args, rank, world, local_rank):
    """32 chained MoE layers captured in one CUDA graph: each layer is
    update_expert -> dispatch (bf16 rows) -> identity expert (the combine
    reads the dispatch's rows) -> combine+Add+RMSNorm, with X_{l+1} = y_l and
    residual_{l+1} = x_out_l.  A timed iteration is one replay of the whole
    stack, with L2 flushed before it outside the events; per-layer time =
    replay time / 32."""
    import numpy as np
    import torch
    from combine_moe_update_b200 import binding as B
    from combine_moe_update_b200 import inputs as gen

    torch.cuda.set_device(local_rank)
    st = gen.make_layer_stack(seed=4 if rank == 0 else 1000 + rank)
    L, bs, H, K, E = st.layers, st.bs, st.hidden, st.top_k, st.num_experts
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    bf = lambda a: dev(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(torch.bfloat16)
    ids = [dev(a) for a in st.expert_ids]
    scs = [dev(a) for a in st.expert_scales]
    gms = [bf(a) for a in st.gammas]
    table = dev(st.table)
    x0, r0 = bf(st.x0), bf(st.residual0)
    wsp = B.new_workspace()
    bal = [torch.empty((bs, K), dtype=torch.int32, device="cuda") for _ in range(L)]
    bm = [torch.empty((bs, K), dtype=torch.uint8, device="cuda") for _ in range(L)]
    dsp = [B.alloc_dispatch_outputs(bs, H, K, E, 0) for _ in range(L)]
    outs = [dict(y=torch.empty((bs, H), dtype=torch.bfloat16, device="cuda"),
                 x_out=torch.empty((bs, H), dtype=torch.bfloat16, device="cuda"), rstd=None) for _ in range(L)]

    def stack():
        x, r = x0, r0
        for l in range(L):
            B.update_expert(ids[l], table, st.ep_world_size, expert_scales=scs[l], workspace=wsp, out=(bal[l], bm[l]))
            B.dispatch(x, bal[l], E, st.ep_world_size, 0, mask=bm[l], workspace=wsp, out=dsp[l])
            B.combine_add_rmsnorm(dsp[l]["expand_x"], dsp[l]["expand_idx"], scs[l], r, gms[l], st.norm_eps,
                                  workspace=wsp, out=outs[l])
            x, r = outs[l]["y"], outs[l]["x_out"]

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    clean = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.float32, device="cuda")

    def flush_l2():
        flush.zero_()
        clean.sum()

    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        for _ in range(args.warmup):
            stack()
    torch.cuda.current_stream().wait_stream(cap)
    torch.cuda.synchronize()
    assert B.read_device_error(wsp) == 0, "device error during warm-up"
    n = int(dsp[0]["offsets"][-1].item())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        stack()
    g.replay()
    torch.cuda.synchronize()

    K_ = args.steps
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K_)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K_)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for k_ in range(K_):
            flush_l2()
            e0[k_].record()
            g.replay()
            e1[k_].record()
        torch.cuda.synchronize()
    barrier()
    t_stack = sum(a.elapsed_time(b) for a, b in zip(e0, e1)) / K_
    assert B.read_device_error(wsp) == 0, "device error during the timed stacks"

    # end to end: the stack's inputs (x0, residual0 and every layer's routing)
    # from pinned host memory, the graph, the last y back to the host
    pin = lambda t: t.cpu().pin_memory()
    h_in = [(pin(x0), x0), (pin(r0), r0)] + [(pin(t), t) for t in ids + scs]
    h_y = torch.empty((bs, H), dtype=torch.bfloat16).pin_memory()
    h2d = sum(h.numel() * h.element_size() for h, _ in h_in)
    d2h = h_y.numel() * h_y.element_size()

    def e2e_step():
        for h, d_ in h_in:
            d_.copy_(h, non_blocking=True)
        g.replay()
        h_y.copy_(outs[-1]["y"], non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    ke = max(5, min(K_, 100))
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for _ in range(ke):
        e2e_step()
    a1.record()
    torch.cuda.synchronize()
    t_stack, t_e2e = reduce_over_ranks([t_stack, a0.elapsed_time(a1) / ke], "max")
    del g

    class _W:  # the per-layer shape, for the byte count
        pass
    lw = _W()
    lw.bs, lw.hidden, lw.top_k, lw.num_instances, lw.num_logical = bs, H, K, E, E
    lw.quant_mode, lw.prune_threshold, lw.smooth, lw.shared_x, lw.meta = 0, 0.0, None, None, {}
    alg = algorithmic_bytes(lw, n, x_out=True)
    per_layer = t_stack / L
    peak, peak_kind = measured_peak()
    layer_bytes = alg["update"] + alg["dispatch"] + alg["combine"]
    achieved = layer_bytes / (per_layer * 1e-3) / 1e9
    out = {
        "metric": METRIC, "value": round(world * bs / (per_layer * 1e-3), 1), "unit": "tokens/s", "n_gpus": world,
        "steps": K_, "warmup": args.warmup, "ms_per_step": round(t_stack, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16+fp32", "data": "synthetic (seeded; pages' shapes)",
        "config": {"workload": "layer_stack", "layers": L, "bs": bs, "hidden": H, "top_k": K, "num_instances": E,
                   "ep_world_size_simulated": st.ep_world_size, "quant_mode": 0, "kept_copies_per_layer": n,
                   "l2": "flushed before every timed stack (512 MiB written, then 256 MiB read), outside the events",
                   "parallelism": f"replicas x{world}"},
        "per_layer_us": round(per_layer * 1e3, 3),
        "step": "one replay of the 32-layer graph; value = tokens through one layer per second (Bs / per-layer time)",
        "roofline": {"bound": "hbm", "kernel": "whole layer (update, dispatch, combine)", "achieved": round(achieved, 1),
                     "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": None, "algorithmic_bytes": layer_bytes,
                     "note": "latency-bound: 7.9 MB per layer, three dependent launches"},
        "e2e": {"value": round(world * bs * L / (t_e2e * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "per step: x0, residual0 and all 32 layers' routing host -> device, the graph, the last y "
                        "device -> host; value = Bs / (step time / 32)"},
        "gpu_launches": 3 * L * K_,
        "timing": "CUDA events around each replay of the 32-layer graph, L2 flushed before each replay",
        "clocks": clk.summary(),
    }
    return out, st


def graph_time(body, sets, steps):
    """Per-call time (ms) of `body(n)` captured for n < count (count = sets
    rounded up to at least 16 calls) in one CUDA graph with events only at
    its ends, averaged over a few replays."""
    import torch
    count = sets * max(1, -(-16 // sets))
    eb = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        eb[0].record()
        for n_ in range(count):
            body(n_)
        eb[1].record()
    g.replay()
    torch.cuda.synchronize()
    reps = max(3, min(50, steps // 4))
    tot = 0.0
    for _ in range(reps):
        g.replay()
        torch.cuda.synchronize()
        tot += eb[0].elapsed_time(eb[1]) / count
    del g
    return tot / reps


def ep_kernel_roofline(kernel, alg_bytes, t_ms, peak, peak_kind, traffic_key=None, workload=None):
    ach = alg_bytes / (t_ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": kernel, "achieved": round(ach, 1), "peak": peak, "peak_kind": peak_kind,
            "unit": "GB/s", "frac": round(ach / peak, 4), "launch_us": round(t_ms * 1e3, 2),
            "traffic": stored_traffic(traffic_key, workload) if traffic_key else None,
            "algorithmic_bytes": alg_bytes,
            "timing": "launches back to back over input sets larger than twice L2, CUDA events at the graph's ends; "
                      "the dispatch's bytes include the route's outputs (about 0.1 %)"}


def run_b200_ep(args, rank, world, local_rank):
    """Expert parallelism across the GPUs of the job: GPU g owns instances
    [g E / N, (g + 1) E / N) and dispatches its own batch; every step is
    update + routing of its tokens, the gather of every GPU's counts, the
    plan, the EP dispatch storing each quantized copy into its owner's
    receive buffer (peer memory), a barrier, the expert step (the owner's
    output buffer, resident), a barrier, and the EP combine+Add+RMSNorm
    reading every copy's output from its owner.  The two-step form
    dispatches locally, pushes the rows, and pulls the outputs back before a
    local combine.  Timed with events on each rank, max over ranks."""
    import numpy as np
    import torch
    from combine_moe_update_b200 import binding as B
    from combine_moe_update_b200 import ep as EP
    from combine_moe_update_b200 import inputs as gen

    torch.cuda.set_device(local_rank)
    w = gen.make(args.workload, seed=None if rank == 0 else 1000 + rank)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    bf = lambda a: dev(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(torch.bfloat16)
    fused = not args.ep_two_step
    grp = EP.ProcessGroupEP(fused=fused, bs=w.bs, hidden=w.hidden, top_k=w.top_k, num_instances=w.num_instances,
                            ep_world_size=w.ep_world_size, quant_mode=w.quant_mode)
    r = grp.r
    table, smooth, gamma = dev(w.table), None if w.smooth is None else dev(w.smooth), bf(w.gamma)
    ids, scales, x, residual = dev(w.expert_ids), dev(w.expert_scales), bf(w.x), bf(w.residual)
    shared = None if w.shared_x is None else bf(w.shared_x)
    r.expert_out.copy_(bf(np.resize(w.expert_out, (r.cap, w.hidden))))  # the expert step's output, resident
    out = dict(y=torch.empty_like(x), x_out=None, rstd=None)

    def step():
        grp.dispatch(expert_ids=ids, table=table, x=x, expert_scales=scales, smooth=smooth,
                     prune_threshold=w.prune_threshold)
        grp.combine(expert_scales=scales, residual=residual, gamma=gamma, norm_eps=w.norm_eps, shared_x=shared,
                    out=out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert r.device_errors() == 0, "device error during warm-up"
    K = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        e0.record()
        for _ in range(K):
            step()
        e1.record()
        torch.cuda.synchronize()
    (t_step,) = reduce_over_ranks([e0.elapsed_time(e1) / K], "max")
    recv = r.received()
    assert r.device_errors() == 0, "device error during the timed steps"
    n = int(r.d["offsets"][-1].item())
    # The two EP kernels on their own (one GPU: every owner is this GPU): launches back to back over input sets
    # larger than twice L2 (x for the dispatch; expert outputs, residual and shared rows for the combine, each
    # set behind its own pointer table), events only at the graph's ends.
    t_epd = t_epc = None
    if fused and world == 1:
        per_x = x.numel() * x.element_size()
        Rd = -(-(2 * L2_BYTES) // per_x) + 1
        xs = [x.clone() for _ in range(Rd)]
        t_epd = graph_time(lambda n_: r.ep_dispatch(xs[n_ % Rd], grp.tables, smooth=smooth), Rd, K)
        del xs
        cset = (r.expert_out, residual, shared)
        per_c = sum(t.numel() * t.element_size() for t in cset if t is not None)
        Rc = -(-(2 * L2_BYTES) // per_c) + 1
        cl = [[None if t is None else t.clone() for t in cset] for _ in range(Rc)]
        tabs = [EP.PeerTables(None, None, None, [c[0].data_ptr()], r.device) for c in cl]
        t_epc = graph_time(lambda n_: B.ep_combine_add_rmsnorm(r.p_pull, tabs[n_ % Rc].expert_out, r.global_idx,
                                                               scales, cl[n_ % Rc][1], gamma, w.norm_eps, r.ep_ws,
                                                               shared_x=cl[n_ % Rc][2], out=out),
                           Rc * max(1, 16 // Rc), K)
        del cl, tabs
        assert r.device_errors() == 0, "device error in the EP kernel timing"
    grp.close()
    copies = w.bs * w.top_k
    route = 3 if copies > 8192 else 1
    # fused: update, route, plan, EP dispatch, EP combine; two-step: the one-GPU step + plan, push, pull
    n_kernels = 1 + route + 3 if fused else kernels_per_step(w) + 3
    # the whole step against HBM: the single-GPU path's bytes, plus for the two-step form the exchange (each
    # row read locally and written to its owner; each output read from its owner and written locally).  The
    # fused form writes each row once, at its owner, and reads each output once, from its owner.
    w.meta["distinct_instances"] = list(range(w.num_instances)) if w.smooth is not None else []
    alg = algorithmic_bytes(w, n)
    rb, sb = B.ep_row_bytes(w.quant_mode, w.hidden)
    exch = 0 if fused else 2 * n * (rb + sb) + 2 * n * 2 * w.hidden
    peak, peak_kind = measured_peak()
    step_bytes = alg["update"] + alg["dispatch"] + alg["combine"] + exch
    ach = step_bytes / (t_step * 1e-3) / 1e9
    return {
        "metric": METRIC, "value": round(world * w.bs / (t_step * 1e-3), 1), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(t_step, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": {0: "bf16", 1: "int8", 2: "int8", 3: "int8", 4: "fp8e4m3"}[w.quant_mode] + "+fp32",
        "data": "synthetic (seeded; pages' shapes; every GPU its own batch)",
        "config": {"workload": args.workload, "bs_per_gpu": w.bs, "hidden": w.hidden, "top_k": w.top_k,
                   "num_instances": w.num_instances, "ep_world_size_simulated": w.ep_world_size,
                   "quant_mode": w.quant_mode, "parallelism": f"ep{world}: instances split over the GPUs",
                   "exchange": "fused into dispatch and combine" if fused else "push and pull",
                   "rows_received_rank0": recv,
                   "l2": "not flushed: each step's exchange and gathers touch more than L2 across the group"},
        "roofline": ep_kernel_roofline("combine_token_kernel (EP)", alg["combine"], t_epc, peak, peak_kind,
                                       "combine_token_kernel_ep", args.workload) if t_epc else None,
        "roofline_other": ep_kernel_roofline("dispatch_token_smooth_kernel (EP)" if w.smooth is not None
                                             else "dispatch_token_kernel (EP)", alg["dispatch"], t_epd, peak,
                                             peak_kind, "dispatch_token_smooth_kernel_ep" if w.smooth is not None
                                             else None, args.workload) if t_epd else None,
        "step_roofline": {"bound": "hbm", "kernel": ("whole step (update, route, plan, EP dispatch, EP combine)"
                                                     if fused else
                                                     "whole step (update, dispatch, plan, push, pull, combine)"),
                          "achieved": round(ach, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                          "frac": round(ach / peak, 4), "traffic": None, "algorithmic_bytes": step_bytes,
                          "note": "eager launches with two NCCL barriers and a count gather per step"},
        "e2e": None,
        "gpu_launches": n_kernels * K,
        "timing": "CUDA events around K eager steps (each with two barriers), max over ranks",
        "clocks": clk.summary(),
    }, w


def oracle_stack(orc, st, lo, hi):
    """The oracle's 32 chained layers on tokens [lo, hi) of the stack."""
    x, r = st.x0[lo:hi], st.residual0[lo:hi]
    for l in range(st.layers):
        bal, bm, _ = orc.update_expert(st.expert_ids[l][lo:hi], st.table, st.ep_world_size,
                                       expert_scales=st.expert_scales[l][lo:hi])
        d = orc.dispatch(x, bal, st.num_experts, 0, mask=bm)
        c = orc.combine_add_rmsnorm(d["expand_x"], d["expand_idx"], st.expert_scales[l][lo:hi], r, st.gammas[l],
                                    st.norm_eps)
        x, r = c["y"], c["x_out"]


def layer_stack_oracle_rate(st, workers, budget_s):
    """Per-layer tokens/s of `workers` threads each running the oracle's
    chained layers on its own slice of tokens.  Returns (tokens/s, slice)."""
    from concurrent.futures import ThreadPoolExecutor
    from oracle import oracle as orc
    per = st.bs if workers == 1 else max(1, st.bs // workers)
    span = max(1, st.bs - per + 1)
    oracle_stack(orc, st, 0, 1)  # build and warm

    def work(k):
        lo = (k * per) % span
        done, t0 = 0, time.perf_counter()
        while True:
            oracle_stack(orc, st, lo, lo + per)
            done += per
            if time.perf_counter() - t0 >= budget_s:
                return done, time.perf_counter() - t0

    with ThreadPoolExecutor(max_workers=workers) as ex:
        res = list(ex.map(work, range(workers)))
    # tokens through one layer per second: every pass moves `per` tokens through all the layers
    return st.layers * sum(r[0] for r in res) / max(r[1] for r in res), per


def layer_stack_cpu_baseline(st, budget_s):
    cores, model = host_cpu()
    one, _ = layer_stack_oracle_rate(st, 1, budget_s / 2)
    many, per = layer_stack_oracle_rate(st, cores, budget_s / 2)
    return {"value": round(many, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle", "cpu_model": model,
            "single_thread": round(one, 2),
            "sample": (f"{cores} threads, each repeating the 32 chained oracle layers on its own slice of {per} of the "
                       f"{st.bs} tokens for {budget_s / 2:.0f} s; value = tokens through one layer per second")}


def layer_stack_reference(args):
    from combine_moe_update_b200 import inputs as gen
    st = gen.make_layer_stack()
    cores, model = host_cpu()
    budget = max(2.0, 100.0 / max(1, args.steps + args.warmup))
    value, per = layer_stack_oracle_rate(st, cores, budget)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32 quant / f64 combine",
        "data": "synthetic (seeded; pages' shapes)",
        "config": {"workload": "layer_stack", "layers": st.layers, "bs": st.bs, "hidden": st.hidden,
                   "top_k": st.top_k, "num_instances": st.num_experts, "quant_mode": 0},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "cpu_model": model,
                         "sample": f"{cores} threads x {per} tokens through 32 chained layers, {budget:.0f} s"},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def gmm_bytes(offsets, hidden, out_dim, mx=False):
    """Algorithmic bytes of one grouped matmul: the weights of every instance
    that received rows (read once), the rows (one byte per element) and their
    factors, the weights' factors, the offsets, and the bf16 output rows.
    Factors: int8 one f32 per row and per channel; mxfp8 one byte per
    32-element block of every row and weight row."""
    import numpy as np
    off = np.asarray(offsets, np.int64)
    used = int(np.count_nonzero(np.diff(off)))
    n = int(off[-1] - off[0])
    f_w, f_x = (out_dim * (hidden // 32), hidden // 32) if mx else (out_dim * 4, 4)
    return used * out_dim * hidden + used * f_w + n * hidden + n * f_x + n * out_dim * 2 + off.size * 4


def run_b200_expert(args, rank, world, local_rank, w):
    """The layer with the instances' grouped int8 matmul in the step:
    moe_update_expert -> moe_dispatch (int8 rows) -> moe_grouped_matmul
    (N = H, every instance's weight resident in HBM) -> moe_combine_add_rmsnorm
    reading the matmul's output rows.  The weights (13 GB at 256 instances)
    dwarf L2, and the activations are flushed out of L2 before every step."""
    import numpy as np
    import torch
    from combine_moe_update_b200 import binding as B
    from combine_moe_update_b200 import inputs as gen

    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    bf = lambda a: dev(np.ascontiguousarray(a, np.uint16).view(np.int16)).view(torch.bfloat16)
    H, E, N = w.hidden, w.num_instances, int(w.meta["expert_out_dim"])
    assert N == H, "the combine gathers rows of width H"
    table = dev(w.table)
    smooth = None if w.smooth is None else dev(w.smooth)
    gamma = bf(w.gamma)
    mx = w.quant_mode == 4  # mxfp8 rows: mxfp8 weights on the block-scaled path
    if mx:
        weight, wscale = gen.gmm_weights_device_mx(w.meta["weight_seed"], E, N, H, "cuda")
        gmm = functools.partial(B.grouped_matmul_mx, weight=weight, weight_sf=wscale)
    else:
        weight, wscale = gen.gmm_weights_device(w.meta["weight_seed"], E, N, H, "cuda")
        gmm = functools.partial(B.grouped_matmul, weight=weight, weight_scales=wscale)
    ids, scales = dev(w.expert_ids), dev(w.expert_scales)
    x, residual = bf(w.x), bf(w.residual)
    shared = None if w.shared_x is None else bf(w.shared_x)
    ws = B.new_workspace(nbytes=B.dispatch_workspace_bytes(
        w.bs, H, w.top_k, w.ep_world_size, E, w.quant_mode, 0 if w.smooth is None else w.smooth.size))
    rows = w.bs * w.top_k
    gws = B.new_workspace(nbytes=B.grouped_matmul_workspace_bytes(rows, H, N, E))
    bal = torch.empty_like(ids)
    bm = torch.empty(ids.shape, dtype=torch.uint8, device="cuda")
    d = B.alloc_dispatch_outputs(w.bs, H, w.top_k, E, w.quant_mode)
    ex = torch.zeros((rows, N), dtype=torch.bfloat16, device="cuda")
    c = dict(y=torch.empty_like(x), x_out=None, rstd=None)

    def calls(xx=x, ii=ids, ss=scales, rr=residual, sh=shared, ev=None):
        mark = (lambda j: ev[j].record()) if ev is not None else (lambda j: None)
        B.update_expert(ii, table, w.ep_world_size, expert_scales=ss, prune_threshold=w.prune_threshold,
                        workspace=ws, out=(bal, bm))
        mark(1)
        B.dispatch(xx, bal, E, w.ep_world_size, w.quant_mode, mask=bm, smooth=smooth, workspace=ws, out=d)
        mark(2)
        gmm(d["expand_x"], d["dyn_scales"], d["offsets"], out=ex, workspace=gws)
        mark(3)
        B.combine_add_rmsnorm(ex, d["expand_idx"], ss, rr, gamma, w.norm_eps, shared_x=sh, workspace=ws, out=c)

    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    clean = torch.zeros(L2_FLUSH_BYTES // 8, dtype=torch.float32, device="cuda")

    def flush_l2():
        flush.zero_()
        clean.sum()

    for _ in range(args.warmup):
        flush_l2()
        calls()
    torch.cuda.synchronize()
    assert B.read_device_error(ws) == 0 and B.read_device_error(gws) == 0, "device error during warm-up"
    off = d["offsets"].cpu().numpy()
    n = int(off[-1])
    alg = algorithmic_bytes(w, n)
    alg["grouped_matmul"] = gmm_bytes(off, H, N, mx)
    # the combine reads the matmul's rows instead of the stand-in rows: same byte count

    K = args.steps
    G = max(g for g in range(1, 9) if K % g == 0)
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())

    def capture(per_call):
        evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)] for _ in range(G)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            for e in evs:
                flush_l2()
                e[0].record()
                calls(ev=e if per_call else None)
                e[4].record()
        return g, evs

    graph, ev_step = capture(False)
    graph_ops, ev_ops = capture(True)
    for g in (graph, graph_ops):
        g.replay()
    torch.cuda.synchronize()
    sums = [0.0] * 5
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for _ in range(K // G):
            graph.replay()
            torch.cuda.synchronize()
            for e in ev_step:
                sums[0] += e[0].elapsed_time(e[4])
        barrier()
        torch.cuda.synchronize()
        for _ in range(K // G):
            graph_ops.replay()
            torch.cuda.synchronize()
            for e in ev_ops:
                for j in range(4):
                    sums[1 + j] += e[j].elapsed_time(e[j + 1])
    barrier()
    del graph, graph_ops
    assert B.read_device_error(ws) == 0 and B.read_device_error(gws) == 0, "device error during the timed steps"

    # The matmul on its own for the roofline: calls back to back (each kernel a
    # programmatic dependent of the one before) in one graph; the weights are
    # far larger than L2, so every call streams them from HBM.  Time per call =
    # the span / count; a call is the planning kernel plus the matmul kernel.
    M = 8
    eb = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    graph_g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_g, stream=cap):
        eb[0].record()
        for _ in range(M):
            gmm(d["expand_x"], d["dyn_scales"], d["offsets"], out=ex, workspace=gws)
        eb[1].record()
    graph_g.replay()
    torch.cuda.synchronize()
    reps = max(3, min(20, K // 4))
    t_gmm = 0.0
    for _ in range(reps):
        graph_g.replay()
        torch.cuda.synchronize()
        t_gmm += eb[0].elapsed_time(eb[1]) / M
    t_gmm /= reps
    del graph_g
    assert B.read_device_error(gws) == 0, "device error during the matmul roofline calls"

    t_step, t_upd, t_disp, t_gm, t_comb, t_gmm = reduce_over_ranks([v / K for v in sums] + [t_gmm], "max")
    value = world * w.bs / (t_step * 1e-3)

    # end to end through the public API with host buffers (weights and layer parameters resident)
    pin = lambda t: t.cpu().pin_memory()
    h_in = dict(x=pin(x), ids=pin(ids), scales=pin(scales), residual=pin(residual))
    if shared is not None:
        h_in["shared"] = pin(shared)
    d_in = {k_: torch.empty_like(v) for k_, v in (("x", x), ("ids", ids), ("scales", scales), ("residual", residual))}
    d_in["shared"] = None if shared is None else torch.empty_like(shared)
    h_y = torch.empty(c["y"].shape, dtype=c["y"].dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in h_in.values())
    d2h = h_y.numel() * h_y.element_size()

    def e2e_step():
        for k_, t in h_in.items():
            d_in[k_].copy_(t, non_blocking=True)
        calls(d_in["x"], d_in["ids"], d_in["scales"], d_in["residual"], d_in["shared"])
        h_y.copy_(c["y"], non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ke = max(5, min(K, 50))
    e0.record()
    for _ in range(ke):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    (t_e2e,) = reduce_over_ranks([e0.elapsed_time(e1) / ke], "max")

    peak, peak_kind = measured_peak()
    achieved = alg["grouped_matmul"] / (t_gmm * 1e-3) / 1e9
    step_bytes = alg["update"] + alg["dispatch"] + alg["grouped_matmul"] + alg["combine"]
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(t_step, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "fp8e4m3 with E8M0 blocks (matmul fp32 accumulate)" if mx else "int8+int32 (matmul), fp32",
        "data": "synthetic (seeded; pages' shapes; instance weights drawn on the device)",
        "config": {"workload": args.workload, "bs": w.bs, "hidden": H, "top_k": w.top_k, "num_instances": E,
                   "ep_world_size_simulated": w.ep_world_size, "quant_mode": w.quant_mode,
                   "smooth_scales": w.smooth is not None, "shared_expert": w.shared_x is not None,
                   "kept_copies": n, "expert_out_dim": N, "weight_bytes": E * N * H,
                   "l2": "flushed before every timed step (512 MiB written, 256 MiB read); weights >> L2",
                   "parallelism": f"replicas x{world}"},
        "breakdown_us": {"update_expert": round(t_upd * 1e3, 2), "dispatch": round(t_disp * 1e3, 2),
                         "grouped_matmul": round(t_gm * 1e3, 2), "combine": round(t_comb * 1e3, 2)},
        "achieved_gbs": {"step": round(step_bytes / (t_step * 1e-3) / 1e9, 1), "grouped_matmul": round(achieved, 1)},
        "roofline": {"bound": "hbm", "kernel": "gmm_mx_kernel" if mx else "gmm_kernel", "achieved": round(achieved, 1), "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "launch_us": round(t_gmm * 1e3, 2),
                     "timing": f"{M} back-to-back calls (planning + matmul kernel) in a graph, CUDA events around them",
                     "traffic": stored_traffic("gmm_mx_kernel" if mx else "gmm_kernel", args.workload),
                     "algorithmic_bytes": alg["grouped_matmul"],
                     "tensor_tops": round(2.0 * n * N * H / (t_gmm * 1e-3) / 1e12, 1)},
        "e2e": {"value": round(world * w.bs / (t_e2e * 1e-3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "pinned host activations -> device, the four calls, y -> host; weights resident"},
        "gpu_launches": 6 * K,  # update_expert, route, scatter, matmul planning, matmul, combine
        "timing": f"CUDA graphs of {G} steps, L2 flushed before each step outside the events",
        "clocks": clk.summary(),
    }
    return out, w


# --------------------------------------------------------------------------
# the CPU oracle, as a reported baseline and as the reference arm
# --------------------------------------------------------------------------

def oracle_step(orc, w):
    bal, bm, _ = orc.update_expert(w.expert_ids, w.table, w.ep_world_size, expert_scales=w.expert_scales,
                                   prune_threshold=w.prune_threshold)
    d = orc.dispatch(w.x, bal, w.num_instances, w.quant_mode, mask=bm, smooth=w.smooth)
    rows = w.expert_out
    if "expert_out_dim" in w.meta:
        rows = _oracle_expert_rows(orc, w, d)
    if int(w.meta.get("tp", 1)) == 2:  # a slice of the TP-major tokens: its rows are the pair's gathered order
        orc.combine_add_rmsnorm_tp(rows, w.meta["expert_out_tp1"], d["expand_idx"], w.expert_scales, w.residual,
                                   w.gamma, w.norm_eps, shared_x=w.shared_x)
        return
    orc.combine_add_rmsnorm(rows, d["expand_idx"], w.expert_scales, w.residual, w.gamma, w.norm_eps,
                            shared_x=w.shared_x)


def _oracle_expert_rows(orc, w, d):
    """The oracle's grouped matmul over the instances this sample reaches (the
    others have no rows, so dropping them from the offsets changes nothing);
    their host weights are drawn once per sample and cached on it."""
    import numpy as np
    from combine_moe_update_b200 import inputs as gen
    off = d["offsets"]
    used = [e for e in range(w.num_instances) if off[e + 1] > off[e]]
    cache = w.meta.setdefault("_host_weights", {})
    key = tuple(used)
    mx = w.quant_mode == 4
    if key not in cache:
        draw = gen.gmm_weights_host_mx if mx else gen.gmm_weights_host
        hw = draw(w.meta["weight_seed"], used, w.meta["expert_out_dim"], w.hidden)
        cache.clear()
        cache[key] = (np.stack([hw[e][0] for e in used]), np.stack([hw[e][1] for e in used]))
    wts, wss = cache[key]
    off_c = np.array([off[e] for e in used] + [off[-1]], np.int32)
    out = np.zeros((d["expand_x"].shape[0], w.meta["expert_out_dim"]), np.uint16)
    if mx:
        g = orc.grouped_matmul_mx(d["expand_x"], d["dyn_scales"], off_c, wts, wss, out=out)
    else:
        g = orc.grouped_matmul(d["expand_x"], d["dyn_scales"], off_c, wts, wss, out=out)
    return g["out"]


def subsample(w, tokens, start=0):
    """Tokens [start, start + tokens) of the workload (same parameters)."""
    import copy
    s = copy.copy(w)
    s.bs = tokens
    for k in ("x", "expert_ids", "expert_scales", "residual", "shared_x", "active_mask"):
        v = getattr(w, k)
        if v is not None:
            setattr(s, k, v[start:start + tokens].copy())
    s.expert_out = w.expert_out[start * w.top_k:(start + tokens) * w.top_k].copy()
    s.meta = {k: v for k, v in w.meta.items() if not k.startswith("_")}
    if "expert_out_tp1" in w.meta:
        s.meta["expert_out_tp1"] = w.meta["expert_out_tp1"][start * w.top_k:(start + tokens) * w.top_k].copy()
    return s


def host_cpu():
    """Cores this process may run on, and the CPU model."""
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return cores, model


def oracle_rate(orc, w, workers, budget_s):
    """Tokens per second of `workers` threads, each running the oracle step on
    its own slice of the workload's tokens (data parallel over tokens) for
    about `budget_s` seconds.  The oracle's C calls release the GIL, so the
    threads run on separate cores.  Returns (tokens/s, tokens per slice)."""
    from concurrent.futures import ThreadPoolExecutor
    per = w.bs if workers == 1 else max(1, w.bs // workers)
    span = max(1, w.bs - per + 1)
    subs = [subsample(w, per, start=(k * per) % span) for k in range(workers)]
    oracle_step(orc, subs[0])  # build and warm the oracle

    def work(sub):
        done, t0 = 0, time.perf_counter()
        while True:
            oracle_step(orc, sub)
            done += sub.bs
            if time.perf_counter() - t0 >= budget_s:
                return done, time.perf_counter() - t0

    with ThreadPoolExecutor(max_workers=workers) as ex:
        res = list(ex.map(work, subs))
    return sum(r[0] for r in res) / max(r[1] for r in res), per


def cpu_baseline(w, budget_s=10.0):
    """The oracle on this host: single-threaded, and on every core with one
    token slice per core.  `value` is the all-cores figure."""
    from oracle import oracle as orc
    cores, model = host_cpu()
    if "expert_out_dim" in w.meta:
        # a full step of the matmul layer takes minutes on one core: time a
        # sample of tokens sized from a one-token calibration run
        one = subsample(w, 1)
        t0 = time.perf_counter()
        oracle_step(orc, one)
        per_tok = time.perf_counter() - t0
        # at most 4 tokens: each reaches up to K instances, whose weights (H * H
        # bytes each) are drawn into host memory
        tokens = int(max(1, min(4, budget_s / max(per_tok, 1e-9))))
        sample = subsample(w, tokens)
        oracle_step(orc, sample)  # draw and cache this sample's weights outside the timing
        t0 = time.perf_counter()
        oracle_step(orc, sample)
        dt = time.perf_counter() - t0
        return {"value": round(tokens / dt, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                "host_cores": cores, "cpu_model": model,
                "sample": f"one step of the first {tokens} of {w.bs} tokens ({dt:.1f} s, single-threaded C "
                          "oracle; the weights of the instances they reach drawn on the host)"}
    half = budget_s / 2
    one, _ = oracle_rate(orc, w, 1, half)
    many, per = oracle_rate(orc, w, cores, half)
    return {"value": round(many, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "cpu_model": model, "single_thread": round(one, 2),
            "sample": (f"{cores} threads, each repeating the oracle step on its own slice of {per} of the "
                       f"{w.bs} tokens for {half:.0f} s (data parallel over tokens); single_thread: full "
                       f"{w.bs}-token steps on one core for {half:.0f} s")}


def run_reference(args, rank):
    """Reference arm: the plain CPU oracle on this host's cores."""
    if rank != 0:
        return None
    from combine_moe_update_b200 import inputs as gen
    from oracle import oracle as orc
    w = gen.make(args.workload) if args.workload != "layer_stack" else None
    if w is None:
        return layer_stack_reference(args)
    orc.build()
    cores, model = host_cpu()
    expert = "expert_out_dim" in w.meta
    workers = 1 if expert else cores
    # calibrate: seconds per token, then size each step so the run stays within ~2 minutes
    cal = 1 if expert else 16
    t0 = time.perf_counter()
    oracle_step(orc, subsample(w, cal))
    per_tok = (time.perf_counter() - t0) / cal
    budget = 120.0 / max(1, args.steps + args.warmup)
    # a step is one oracle step on a slice of the batch per thread; the matmul
    # layer: at most 4 tokens, whose instances' weights are drawn on the host
    tokens = int(max(1, min(4 if expert else max(1, w.bs // workers), budget / max(per_tok, 1e-9))))
    span = max(1, w.bs - tokens + 1)
    subs = [subsample(w, tokens, start=(k * tokens) % span) for k in range(workers)]
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=workers) as ex:
        for _ in range(args.warmup):
            list(ex.map(lambda sb: oracle_step(orc, sb), subs))
        t0 = time.perf_counter()
        for _ in range(args.steps):
            list(ex.map(lambda sb: oracle_step(orc, sb), subs))
        dt = time.perf_counter() - t0
    value = args.steps * tokens * workers / dt
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32 quant / f64 combine",
        "data": "synthetic (seeded; pages' shapes)",
        "config": {"workload": args.workload, "bs": w.bs, "hidden": w.hidden, "top_k": w.top_k,
                   "num_instances": w.num_instances, "quant_mode": w.quant_mode,
                   "tokens_per_step": tokens * workers},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": workers, "kind": "oracle",
                         "cpu_model": model,
                         "sample": f"{workers} threads x {tokens} of the {w.bs} tokens per step, {args.steps} steps"},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--cpu-baseline-seconds", type=float, default=10.0)
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism across the job's GPUs (real exchange through peer memory) "
                         "instead of independent replicas")
    ap.add_argument("--ep-two-step", action="store_true",
                    help="with --ep: dispatch locally, then push / pull the rows (instead of the fused "
                         "EP dispatch and combine that read and write the owners' buffers directly)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local_rank = dist_env()

    if args.impl == "reference":
        line = run_reference(args, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0

    import datetime
    import torch.distributed as dist
    if world > 1 or args.ep:
        if world == 1:  # a one-GPU group, so --ep runs the same code path alone
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", "29511")
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        import torch
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.ep:
            out, w = run_b200_ep(args, rank, world, local_rank)
            if rank == 0:
                out["cpu_baseline"] = None
                print(json.dumps(out), flush=True)
            return 0
        if args.workload == "layer_stack":
            out, st = run_b200_layer_stack(args, rank, world, local_rank)
            if rank == 0:
                out["cpu_baseline"] = layer_stack_cpu_baseline(st, args.cpu_baseline_seconds) if world == 1 else None
                print(json.dumps(out), flush=True)
            return 0
        out, w = run_b200(args, rank, world, local_rank)
        if rank == 0:
            out["cpu_baseline"] = cpu_baseline(w, args.cpu_baseline_seconds) if world == 1 else None
            print(json.dumps(out), flush=True)
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
