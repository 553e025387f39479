"""A TP domain of two ranks across the two GPUs of a pair.

With tpWorldSize 2 the pages run every EP rank twice, once per TP domain,
with one instance per EP rank (aclnnMoeDistributeDispatchV2 and
aclnnMoeDistributeCombineAddRmsNorm, 计算公式): the dispatch is AllToAllV
within each domain followed by AllGatherV across the pair, so both TP ranks
of EP rank g hold the rows of instance g from all 2 * ws source devices
(domain 0's rows first); each TP rank computes a partial expert output of
every such row; the combine's ReduceScatterV sums the pair's partials and
hands each domain the rows of its own tokens, and AllToAllV brings them
back.  Numbering the 2 * ws devices TP-major (device t * ws + g is EP rank g
of domain t), those rows are exactly what moe_dispatch writes for the
devices' tokens as 2 * ws sources.

Here GPU t of the pair is TP domain t: it holds that domain's ws EP ranks
(simulated on it, as everywhere in this library) and their ws * bs tokens.
A layer on GPU t:
  gather inputs   the pair's token arrays (x, ids, routing weights, active
                  mask) in TP-major order on both GPUs.  The AllGatherV moves
                  each token's K quantized copies (K * H code bytes and their
                  scales); the bf16 token itself is 2 * H bytes, so for K > 2
                  it is cheaper to gather the tokens and let each GPU quantize
                  its peer's tokens too (the kernels are deterministic, so both
                  GPUs compute the same rows);
  update, dispatch, counts
                  moe_update_expert, moe_dispatch and moe_dispatch_tp_counts
                  over all 2 * ws * bs tokens: the receive buffer after
                  AllToAllV(EP) + AllGatherV(TP), identical on both GPUs;
  expert step     the caller writes this GPU's partial output of every row
                  into `partial`; then a barrier;
  combine         moe_combine_add_rmsnorm_tp2 for this GPU's own tokens, each
                  gathered row the bf16 sum of its own partial and the peer's,
                  read through a CUDA IPC mapping (plain loads over NVLink):
                  the ReduceScatterV and the AllToAllV back in one kernel.

EmulatedTPPair runs both GPUs of the pair on one device (two sets of
buffers, the steps in order); ProcessGroupTP is one process's GPU in a
torch.distributed group of two.  Every step of the computation runs in the
library's kernels; this module only allocates, gathers and sequences.
"""
from __future__ import annotations

import torch

from . import binding as B

# the per-token arrays a layer gathers, in the order they are exchanged
GATHERED = ("x", "expert_ids", "expert_scales", "active_mask")


class TPRank:
    """One GPU of the pair: the dispatch outputs of the pair's tokens, this
    GPU's partial expert outputs, and the calls' parameters.

    ws: EP ranks per TP domain (one instance each); bs: tokens per source
    device; rank: this GPU's TP domain (0 or 1)."""

    def __init__(self, *, ws, bs, hidden, top_k, quant_mode, rank, device="cuda", scales_len=0):
        """scales_len: the number of smooth (or static) scale values the
        dispatch calls will pass (0: none)."""
        if rank not in (0, 1):
            raise ValueError("a TP pair has ranks 0 and 1")
        self.ws, self.bs, self.hidden, self.top_k, self.quant_mode, self.t = ws, bs, hidden, top_k, quant_mode, rank
        self.E, self.S = ws, 2 * ws
        self.T = self.S * bs          # the pair's tokens
        self.mine = slice(rank * ws * bs, (rank + 1) * ws * bs)  # this GPU's tokens among them
        self.device = torch.device(device)
        dev, T, K = self.device, self.T, top_k
        self.bal = torch.empty((T, K), dtype=torch.int32, device=dev)
        self.bm = torch.empty((T, K), dtype=torch.uint8, device=dev)
        self.d = B.alloc_dispatch_outputs(T, hidden, K, self.E, quant_mode, dev)
        self.tp_counts = torch.empty((self.E, 2), dtype=torch.int32, device=dev)
        self.partial = torch.empty((T * K, hidden), dtype=torch.bfloat16, device=dev)
        self.scales_len = scales_len
        self.ws_buf = B.new_workspace(dev, nbytes=B.dispatch_workspace_bytes(bs, hidden, K, ws, self.E, quant_mode,
                                                                          scales_len, self.S))

    def dispatch(self, full: dict, table, smooth=None, prune_threshold=0.0, stream=None):
        """update_expert, dispatch and the per-(rank, domain) counts of the
        pair's tokens (full: the gathered arrays of GATHERED)."""
        if (0 if smooth is None else smooth.numel()) != self.scales_len:
            raise ValueError("smooth does not have the scales_len this rank was built for")
        B.update_expert(full["expert_ids"], table, self.ws, expert_scales=full.get("expert_scales"),
                        active_mask=full.get("active_mask"), prune_threshold=prune_threshold,
                        workspace=self.ws_buf, out=(self.bal, self.bm), stream=stream, sources=self.S)
        B.dispatch(full["x"], self.bal, self.E, self.ws, self.quant_mode, mask=self.bm, smooth=smooth,
                   workspace=self.ws_buf, out=self.d, stream=stream, sources=self.S)
        B.dispatch_tp_counts(self.d, self.bs, self.hidden, self.top_k, self.ws, self.quant_mode,
                             scales_len=self.scales_len, workspace=self.ws_buf, out=self.tp_counts, stream=stream)

    def combine(self, peer_partial, expert_scales, residual, gamma, norm_eps, shared_x=None, out=None,
                want_x_out=False, stream=None):
        """The combine of this GPU's tokens (expert_scales: the pair's [T, K]
        weights; residual, shared_x: this GPU's [ws * bs, H] rows), each row
        the bf16 sum of this GPU's partial and peer_partial (a tensor on this
        device or the address of the peer's buffer mapped here)."""
        p0, p1 = (self.partial, peer_partial) if self.t == 0 else (peer_partial, self.partial)
        return B.combine_add_rmsnorm_tp2(p0, p1, self.d["expand_idx"][self.mine], expert_scales[self.mine],
                                         residual, gamma, norm_eps, shared_x=shared_x, want_x_out=want_x_out,
                                         workspace=self.ws_buf, out=out, stream=stream, sources=self.ws)

    def device_errors(self):
        return B.read_device_error(self.ws_buf)


def concat_tp_major(parts):
    """The pair's arrays in TP-major order: domain 0's tokens, then domain 1's."""
    return torch.cat(parts, dim=0).contiguous()


class EmulatedTPPair:
    """Both GPUs of the pair on one device: two sets of buffers, the steps
    for each GPU in turn.  No kernel waits on another, so the order on one
    stream is enough; the peer's partial is read as a plain tensor."""

    def __init__(self, **kw):
        self.ranks = [TPRank(rank=t, **kw) for t in (0, 1)]

    def dispatch(self, local, table, smooth=None, prune_threshold=0.0):
        """local[t]: GPU t's own arrays (keys of GATHERED; None entries are
        absent on both GPUs)."""
        full = {n: None if local[0].get(n) is None else concat_tp_major([local[0][n], local[1][n]])
                for n in GATHERED}
        for r in self.ranks:
            r.dispatch(full, table, smooth=smooth, prune_threshold=prune_threshold)
        return full

    def combine(self, full, inputs, norm_eps, peer_by_address=False):
        """inputs[t]: GPU t's residual, gamma and optional shared_x.  With
        peer_by_address the peer's partial is passed as a raw address, the
        way a mapped peer buffer is."""
        outs = []
        for r in self.ranks:
            peer = self.ranks[1 - r.t].partial
            outs.append(r.combine(peer.data_ptr() if peer_by_address else peer, full["expert_scales"],
                                  norm_eps=norm_eps, want_x_out=True, **inputs[r.t]))
        return outs


def gather_tp_major(local: torch.Tensor, group=None) -> torch.Tensor:
    """The pair's arrays in TP-major order on every rank of a two-rank group
    (an all-gather; NCCL for CUDA tensors, gloo for CPU ones)."""
    import torch.distributed as dist
    parts = [torch.empty_like(local) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, local.contiguous(), group=group)
    return concat_tp_major(parts)


class ProcessGroupTP:
    """This process's GPU in a torch.distributed group of two (one process
    per GPU, rank t = TP domain t).  The peer's partial buffer is mapped by
    CUDA IPC (a plain peer mapping, no multicast object); call close() before
    the process group is destroyed."""

    def __init__(self, group=None, **kw):
        import torch.distributed as dist
        if dist.get_world_size(group) != 2:
            raise ValueError("a TP pair is a group of two ranks")
        self.group = group
        self.r = TPRank(rank=dist.get_rank(group), **kw)
        self.flag = torch.zeros(1, dtype=torch.float32, device=self.r.device)
        handles = [None, None]
        dist.all_gather_object(handles, B.ipc_export(self.r.partial), group=group)
        self._base, self.peer_partial = B.ipc_import(*handles[1 - self.r.t])

    def dispatch(self, local: dict, table, smooth=None, prune_threshold=0.0):
        """Gather the pair's tokens, then update, dispatch and counts."""
        full = {n: None if local.get(n) is None else gather_tp_major(local[n], self.group) for n in GATHERED}
        self.r.dispatch(full, table, smooth=smooth, prune_threshold=prune_threshold)
        return full

    def combine(self, full, norm_eps, **kw):
        """A barrier (both partials written), the combine of this GPU's
        tokens, then a barrier (the peer has read this GPU's partial before
        either GPU writes the next layer's)."""
        import torch.distributed as dist
        dist.all_reduce(self.flag, group=self.group)
        out = self.r.combine(self.peer_partial, full["expert_scales"], norm_eps=norm_eps, **kw)
        dist.all_reduce(self.flag, group=self.group)
        return out

    def close(self):
        import torch.distributed as dist
        torch.cuda.synchronize()
        dist.barrier(group=self.group)  # no GPU reads a mapping that is about to close
        if self._base is not None:
            B.ipc_close(self._base)
            self._base = None
