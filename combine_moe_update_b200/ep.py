"""Expert parallelism across GPUs: one MoE layer over the GPUs of a group.

The pages' EP AllToAllV sends every quantized (token, k) copy to the rank
that hosts its instance (aclnnMoeDistributeDispatchV2, 功能说明 and 计算公式)
and brings the expert outputs back before the weighted sum
(aclnnMoeDistributeCombineAddRmsNorm, 计算公式: ataOut = AllToAllV).  Over G
GPUs, GPU q owns instances [q * E / G, (q + 1) * E / G) -- the simulated
ranks that host them -- and every GPU is one source of its own Bs tokens, so
the group's rows are those of the multi-source dispatch on one GPU (ordered
by instance, source GPU, token, k) and GPU q's receive buffer is the stretch
of that order its instances own.

A layer on every GPU g (fused, the default):
  route            update_expert + the routing half of the dispatch
                   (moe_dispatch_route) of its own tokens over all E
                   instances;
  gather counts    every GPU's per-instance counts into counts_all [G, E];
  plan, dispatch   moe_ep_plan, then moe_ep_dispatch: each token is
                   quantized once and its copies stored straight into their
                   owners' receive buffers through peer memory; a barrier;
  expert step      on the receive buffer (the caller's), then a barrier;
  combine          moe_ep_combine_add_rmsnorm: the weighted sum reads each
                   copy's expert output from its owner's buffer.
The two-step form (fused=False) dispatches into a local buffer first and
moves the rows with moe_ep_push, and brings the outputs back with
moe_ep_pull before the one-GPU combine; it computes the same rows.
The barriers are one-element all-reduces on the stream, so every kernel
before them has finished on every GPU when the next step starts.

EmulatedGroup runs the G GPUs of a group on one device (G sets of buffers in
this GPU's memory, the steps in order, no kernel waiting on another);
ProcessGroupEP is one process's GPU in a torch.distributed group, with the
peer tables built from CUDA IPC mappings.  Every step of the computation
runs in the library's kernels; this module only allocates and sequences.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


class EPRank:
    """One GPU of the group: its dispatch outputs, receive and expert-output
    buffers, and the parameters of the library's EP calls."""

    def __init__(self, *, bs, hidden, top_k, num_instances, ep_world_size, quant_mode, gpus, rank,
                 recv_rows: Optional[int] = None, device="cuda"):
        if num_instances % gpus or ep_world_size % gpus:
            raise ValueError("the GPUs must split the instances and the simulated ranks evenly")
        self.bs, self.hidden, self.top_k, self.E = bs, hidden, top_k, num_instances
        self.ep_world_size, self.quant_mode, self.G, self.g = ep_world_size, quant_mode, gpus, rank
        self.device = torch.device(device)
        # a GPU can receive every copy of the group (all of them on its instances)
        self.cap = gpus * bs * top_k if recv_rows is None else int(recv_rows)
        row_bytes, scale_bytes = B.ep_row_bytes(quant_mode, hidden)
        self.p_push = B.ep_params(bs, top_k, num_instances, gpus, rank, row_bytes, scale_bytes, self.cap)
        self.p_pull = B.ep_params(bs, top_k, num_instances, gpus, rank, 2 * hidden, 0, self.cap)
        dev = self.device
        self.bal = torch.empty((bs, top_k), dtype=torch.int32, device=dev)
        self.bm = torch.empty((bs, top_k), dtype=torch.uint8, device=dev)
        self.d = B.alloc_dispatch_outputs(bs, hidden, top_k, num_instances, quant_mode, dev)
        self.route_out = {n: self.d[n] for n in ("expand_idx", "src_of_row", "counts", "offsets")}
        self.recv_x = torch.empty((self.cap, hidden), dtype=B.expand_dtype(quant_mode), device=dev)
        self.recv_scales = (torch.empty((self.cap, scale_bytes), dtype=torch.uint8, device=dev)
                            if scale_bytes else None)
        self.recv_src = torch.empty((self.cap,), dtype=torch.int32, device=dev)
        self.expert_out = torch.empty((self.cap, hidden), dtype=torch.bfloat16, device=dev)
        self.ret = torch.empty((bs * top_k, hidden), dtype=torch.bfloat16, device=dev)
        self.counts_all = torch.empty((gpus, num_instances), dtype=torch.int32, device=dev)
        self.recv_counts = torch.empty((num_instances // gpus,), dtype=torch.int32, device=dev)
        self.recv_offsets = torch.empty((num_instances // gpus + 1,), dtype=torch.int32, device=dev)
        self.global_idx = torch.empty((bs, top_k), dtype=torch.int32, device=dev)
        self.ws = B.new_workspace(dev)
        self.ep_ws = B.new_workspace(dev, nbytes=B.ep_workspace_bytes(self.p_push))

    def local_dispatch(self, expert_ids, table, x, expert_scales=None, smooth=None, prune_threshold=0.0,
                       active_mask=None, stream=None):
        """update_expert + dispatch of this GPU's own tokens over all E instances."""
        B.update_expert(expert_ids, table, self.ep_world_size, expert_scales=expert_scales, active_mask=active_mask,
                        prune_threshold=prune_threshold, workspace=self.ws, out=(self.bal, self.bm), stream=stream)
        B.dispatch(x, self.bal, self.E, self.ep_world_size, self.quant_mode, mask=self.bm, smooth=smooth,
                   workspace=self.ws, out=self.d, stream=stream)

    def route(self, expert_ids, table, expert_scales=None, prune_threshold=0.0, active_mask=None, scales_len=0,
              stream=None):
        """update_expert + moe_dispatch_route of this GPU's own tokens (fused form)."""
        B.update_expert(expert_ids, table, self.ep_world_size, expert_scales=expert_scales, active_mask=active_mask,
                        prune_threshold=prune_threshold, workspace=self.ws, out=(self.bal, self.bm), stream=stream)
        B.dispatch_route(self.bal, self.E, self.ep_world_size, self.hidden, self.quant_mode, mask=self.bm,
                         scales_len=scales_len, workspace=self.ws, out=self.route_out, stream=stream)

    def ep_dispatch(self, x, tables: "PeerTables", smooth=None, stream=None):
        """moe_ep_dispatch: this GPU's copies into their owners' receive buffers."""
        B.ep_dispatch(self.p_push, x, self.bal, self.ep_world_size, self.quant_mode, self.route_out, tables.recv_x,
                      tables.recv_scales, tables.recv_src, self.global_idx, self.ep_ws, mask=self.bm, smooth=smooth,
                      stream=stream)

    def ep_combine(self, tables: "PeerTables", expert_scales, residual, gamma, norm_eps, shared_x=None, out=None,
                   stream=None):
        """moe_ep_combine_add_rmsnorm: combine+Add+RMSNorm reading the owners' expert outputs."""
        return B.ep_combine_add_rmsnorm(self.p_pull, tables.expert_out, self.global_idx, expert_scales, residual,
                                        gamma, norm_eps, self.ep_ws, shared_x=shared_x, out=out, stream=stream)

    def plan(self, stream=None):
        B.ep_plan(self.p_push, self.counts_all, self.recv_counts, self.recv_offsets, self.ep_ws, stream=stream)

    def push(self, tables: "PeerTables", stream=None):
        B.ep_push(self.p_push, self.d, self.bal, tables.recv_x, tables.recv_scales, tables.recv_src,
                  self.global_idx, self.ep_ws, stream=stream)

    def pull(self, tables: "PeerTables", stream=None):
        B.ep_pull(self.p_pull, tables.expert_out, self.d["offsets"], self.ret, self.ep_ws, stream=stream)

    def combine(self, expert_scales, residual, gamma, norm_eps, shared_x=None, out=None, stream=None):
        """combine+Add+RMSNorm of this GPU's tokens from the pulled outputs."""
        return B.combine_add_rmsnorm(self.ret, self.d["expand_idx"], expert_scales, residual, gamma, norm_eps,
                                     shared_x=shared_x, workspace=self.ws, out=out, stream=stream)

    def received(self):
        """Rows this GPU received (reads the count back to the host)."""
        return int(self.recv_offsets[-1].item())

    def device_errors(self):
        return B.read_device_error(self.ws) | B.read_device_error(self.ep_ws)

    def buffers(self):
        return [self.recv_x, self.recv_scales, self.recv_src, self.expert_out]


class PeerTables:
    """Every GPU's buffer addresses as this GPU dereferences them: [G] int64
    device tensors (receive rows, their scales, their copy ids, expert
    outputs)."""

    def __init__(self, recv_x, recv_scales, recv_src, expert_out, device):
        t = lambda a: None if a is None else torch.tensor(a, dtype=torch.int64, device=device)
        self.recv_x, self.recv_scales, self.recv_src, self.expert_out = (t(recv_x), t(recv_scales), t(recv_src),
                                                                         t(expert_out))


class EmulatedGroup:
    """The G GPUs of a group emulated on one device: G sets of buffers in this
    GPU's memory, each step run for every GPU in turn.  No kernel waits on
    another, so the order on one stream is enough."""

    def __init__(self, gpus, fused=True, **kw):
        self.fused = fused
        self.ranks = [EPRank(gpus=gpus, rank=g, **kw) for g in range(gpus)]
        addr = lambda ts: None if ts[0] is None else [t.data_ptr() for t in ts]
        rs = self.ranks
        self.tables = PeerTables(addr([r.recv_x for r in rs]), addr([r.recv_scales for r in rs]),
                                 addr([r.recv_src for r in rs]), addr([r.expert_out for r in rs]), rs[0].device)

    def dispatch(self, inputs):
        """inputs[g]: the keyword arguments of EPRank.local_dispatch for GPU g."""
        for r, kw in zip(self.ranks, inputs):
            if self.fused:
                kw = dict(kw)
                x, smooth = kw.pop("x"), kw.pop("smooth", None)
                r.route(scales_len=0 if smooth is None else smooth.numel(), **kw)
            else:
                r.local_dispatch(**kw)
        counts_all = torch.stack([r.d["counts"] for r in self.ranks])  # the gather
        for r in self.ranks:
            r.counts_all.copy_(counts_all)
            r.plan()
        for r, kw in zip(self.ranks, inputs):
            if self.fused:
                r.ep_dispatch(kw["x"], self.tables, smooth=kw.get("smooth"))
            else:
                r.push(self.tables)

    def combine(self, inputs):
        """inputs[g]: the keyword arguments of EPRank.combine for GPU g."""
        if self.fused:
            return [r.ep_combine(self.tables, **kw) for r, kw in zip(self.ranks, inputs)]
        for r in self.ranks:
            r.pull(self.tables)
        return [r.combine(**kw) for r, kw in zip(self.ranks, inputs)]


def gather_counts(counts: torch.Tensor, counts_all: torch.Tensor, group=None):
    """Every GPU's per-instance counts into counts_all [G, E] on every GPU."""
    import torch.distributed as dist
    dist.all_gather_into_tensor(counts_all.view(-1), counts.view(-1), group=group)


def group_barrier(flag: torch.Tensor, group=None):
    """A one-element all-reduce on the current stream: the work enqueued after
    it starts once every GPU's earlier kernels have finished."""
    import torch.distributed as dist
    dist.all_reduce(flag, group=group)


class ProcessGroupEP:
    """This process's GPU in a torch.distributed group (one process per GPU).
    The peer tables hold CUDA IPC mappings of the other GPUs' buffers (plain
    peer mappings, no multicast object); call close() before the process
    group is destroyed."""

    def __init__(self, group=None, fused=True, **kw):
        import torch.distributed as dist
        self.group, self.fused = group, fused
        G, g = dist.get_world_size(group), dist.get_rank(group)
        self.r = EPRank(gpus=G, rank=g, **kw)
        self.flag = torch.zeros(1, dtype=torch.float32, device=self.r.device)
        mine = [None if t is None else B.ipc_export(t) for t in self.r.buffers()]
        everyone = [None] * G
        dist.all_gather_object(everyone, mine, group=group)
        self._bases = []
        cols = [[None] * G for _ in range(4)]
        for q in range(G):
            for b, t in enumerate(self.r.buffers()):
                if t is None:
                    continue
                if q == g:
                    cols[b][q] = t.data_ptr()
                else:
                    base, ptr = B.ipc_import(*everyone[q][b])
                    self._bases.append(base)
                    cols[b][q] = ptr
        self.tables = PeerTables(*(None if c[0] is None else c for c in cols), self.r.device)

    def dispatch(self, **kw):
        """route (or local dispatch), gather counts, plan, EP dispatch (or
        push), barrier: afterwards self.r.recv_x[:received] holds this GPU's
        rows."""
        if self.fused:
            x, smooth = kw.pop("x"), kw.pop("smooth", None)
            self.r.route(scales_len=0 if smooth is None else smooth.numel(), **kw)
        else:
            self.r.local_dispatch(**kw)
        gather_counts(self.r.d["counts"], self.r.counts_all, self.group)
        self.r.plan()
        if self.fused:
            self.r.ep_dispatch(x, self.tables, smooth=smooth)
        else:
            self.r.push(self.tables)
        group_barrier(self.flag, self.group)

    def combine(self, **kw):
        """barrier (every expert output written), then the EP combine (or
        pull and the one-GPU combine)."""
        group_barrier(self.flag, self.group)
        if self.fused:
            return self.r.ep_combine(self.tables, **kw)
        self.r.pull(self.tables)
        return self.r.combine(**kw)

    def close(self):
        import torch.distributed as dist
        torch.cuda.synchronize()
        dist.barrier(group=self.group)  # no GPU reads a mapping that is about to close
        for b in self._bases:
            B.ipc_close(b)
        self._bases = []
