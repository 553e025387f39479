// ep.cuh -- expert parallelism across GPUs: the AllToAllV of dispatch and of
// combine as copies through peer memory (aclnnMoeDistributeDispatchV2,
// "功能说明" and "计算公式": quantize, then AllToAllV over the EP ranks;
// aclnnMoeDistributeCombineAddRmsNorm, "计算公式": ataOut = AllToAllV back).
//
// G GPUs share the E deployed instances evenly: GPU q owns instances
// [q * E / G, (q + 1) * E / G) and so the simulated ranks that host them
// (instances are rank-major).  Every GPU is one source of its own Bs tokens,
// so across the group the rows are exactly those of the multi-source
// dispatch on one GPU, ordered by (instance, source GPU, token, k); GPU q's
// receive buffer holds the contiguous stretch of that order that its
// instances own.
//
// Each GPU first dispatches its own tokens with moe_dispatch (local rows in
// (instance, token, k) order over all E instances, and per-instance counts).
// The counts of all GPUs, cnt[G][E], are gathered on every GPU (a collective
// of E ints per GPU).  Then, on GPU g:
//   ep_plan_kernel   per instance e: the global row where GPU g's copies of
//                    e start, gstart[e] = (rows of instances < e, all GPUs) +
//                    (rows of e from GPUs < g); minus base[owner(e)], it is
//                    the row in the owner's receive buffer.  Also this GPU's
//                    own receive counts and offsets.
//   ep_push_kernel   every local row r of instance e goes to the owner's
//                    receive buffer at row gstart[e] - base[owner] +
//                    (r - local_offsets[e]), through the owner's pointer
//                    (peer memory over NVLink, or this GPU's own memory), with
//                    its scales and its global copy id; every copy's global
//                    row goes to global_idx.
//   ep_pull_kernel   the reverse for the expert outputs: local row r reads
//                    its row back from the owner's output buffer, so the
//                    combine gathers with the local expand_idx as on one GPU.
// All copies are 16-byte loads and stores by the SM (no TMA and no multicast
// touches peer memory).  The group synchronizes between the steps (every
// push done before any GPU reads its receive buffer; every expert output
// written before any pull) outside these kernels.
#pragma once
#include "common.cuh"

namespace moe {

struct EpArgs {
    int bs, top_k, num_instances, gpus, rank;
    int row_bytes;    // bytes of one row (a multiple of 16)
    int scale_bytes;  // bytes of one row's scales (0, 4, 4 * tiles or H / 32)
    int recv_rows;    // rows each receive buffer holds
    const int32_t *counts_all;     // [G][E] rows per instance from every GPU
    const int32_t *local_offsets;  // [E + 1] this GPU's dispatch offsets
    int32_t *gstart;               // [E] workspace: global row of this GPU's first copy of e
    int32_t *base;                 // [G + 1] workspace: first global row of every GPU's instances
    uint32_t *err;
};

// One block of 1024 threads; thread e owns instance e (E <= 1024).
__global__ void __launch_bounds__(1024) ep_plan_kernel(EpArgs a, int32_t *recv_counts, int32_t *recv_offsets) {
    __shared__ int s_warp[32];
    __shared__ int s_excl[1024];  // rows of instances < e, all GPUs
    __shared__ int s_total;
    const int E = a.num_instances, G = a.gpus, El = E / G, e = threadIdx.x;
    pdl_wait();  // the gathered counts and the local offsets come from earlier work
    int tot = 0, before = 0;
    if (e < E) {
        for (int p = 0; p < G; ++p) {
            const int c = a.counts_all[(size_t)p * E + e];
            tot += c;
            if (p < a.rank) before += c;
        }
    }
    const int incl = block_inclusive_scan(tot, s_warp);
    if (e < E) {
        s_excl[e] = incl - tot;
        a.gstart[e] = incl - tot + before;
    }
    if (e == 1023) s_total = incl;
    __syncthreads();
    for (int q = e; q <= G; q += 1024) a.base[q] = q < G ? s_excl[q * El] : s_total;
    const int b = s_excl[a.rank * El];
    const int end = a.rank + 1 < G ? s_excl[(a.rank + 1) * El] : s_total;
    if (e < El) {
        recv_counts[e] = (e + 1 < El ? s_excl[a.rank * El + e + 1] : end) - s_excl[a.rank * El + e];
        recv_offsets[e] = s_excl[a.rank * El + e] - b;
    }
    if (e == 0) {
        recv_offsets[El] = end - b;
        if (end - b > a.recv_rows) raise_error(a.err, kDevCapacity);
    }
    pdl_launch_dependents();
}

// The instance of local row r: the largest e with local_offsets[e] <= r (a
// binary search over the offsets staged in shared memory).
__device__ __forceinline__ int ep_row_instance(const int *s_off, int E, int r) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_off[mid] <= r) lo = mid; else hi = mid - 1;
    }
    return lo;
}

constexpr int kEpThreads = 256;
constexpr int kEpRowsPerBlock = 8;  // one warp per row

// Push (PUSH = true): local row r -> owner's receive buffer.  Pull (false):
// owner's output buffer -> local row r.  Grid: ceil(bs * K / 8) blocks of 8
// warps, one row per warp; the push also writes every copy's global row.
template <bool PUSH>
__global__ void __launch_bounds__(kEpThreads) ep_copy_kernel(EpArgs a, const uint8_t *local_rows, uint8_t *local_out,
                                                             const uint8_t *local_scales,
                                                             uint8_t *const *peer_rows, uint8_t *const *peer_scales,
                                                             int32_t *const *peer_src, const int32_t *src_of_row,
                                                             const int32_t *local_idx, int32_t *global_idx,
                                                             const int32_t *instance_ids) {
    extern __shared__ int s_off[];  // [E + 1] local offsets, then [E] gstart, then [G + 1] base
    const int E = a.num_instances, G = a.gpus, El = E / G, t = threadIdx.x, lane = t & 31, w = t >> 5;
    int *s_gs = s_off + E + 1, *s_base = s_gs + E;
    pdl_wait();  // the local rows, the offsets and the plan come from earlier kernels
    for (int q = t; q <= E; q += kEpThreads) s_off[q] = a.local_offsets[q];
    for (int q = t; q < E; q += kEpThreads) s_gs[q] = a.gstart[q];
    for (int q = t; q <= G; q += kEpThreads) s_base[q] = a.base[q];
    __syncthreads();
    const int n = s_off[E];  // local rows used
    const int r = blockIdx.x * kEpRowsPerBlock + w;
    if (r < n) {
        const int e = ep_row_instance(s_off, E, r), q = e / El;
        const int grow = s_gs[e] + (r - s_off[e]);  // global row
        const int prow = grow - s_base[q];          // row in the owner's buffer
        if (prow < a.recv_rows) {
            const size_t lb = (size_t)r * a.row_bytes, pb = (size_t)prow * a.row_bytes;
            if (PUSH) {
                const uint4 *src = reinterpret_cast<const uint4 *>(local_rows + lb);
                uint4 *dst = reinterpret_cast<uint4 *>(peer_rows[q] + pb);
                for (int v = lane; v < a.row_bytes / 16; v += 32) dst[v] = ld_stream(src + v);
                if (a.scale_bytes > 0) {
                    const uint8_t *ss = local_scales + (size_t)r * a.scale_bytes;
                    uint8_t *ds = peer_scales[q] + (size_t)prow * a.scale_bytes;
                    for (int b = lane; b < a.scale_bytes; b += 32) ds[b] = ss[b];
                }
                if (peer_src != nullptr && lane == 0)  // the copy's id in the group: (g * bs + i) * K + k
                    peer_src[q][prow] = a.rank * a.bs * a.top_k + src_of_row[r];
            } else {
                const uint4 *src = reinterpret_cast<const uint4 *>(peer_rows[q] + pb);
                uint4 *dst = reinterpret_cast<uint4 *>(local_out + lb);
                for (int v = lane; v < a.row_bytes / 16; v += 32) dst[v] = ld_stream(src + v);
            }
        } else if (lane == 0) {
            raise_error(a.err, kDevCapacity);
        }
    }
    if (PUSH) {  // every copy's global row (-1 if not sent)
        const int N = a.bs * a.top_k;
        for (int j = blockIdx.x * kEpThreads + t; j < N; j += gridDim.x * kEpThreads) {
            const int lr = local_idx[j];
            int g = -1;
            if (lr >= 0) {
                const int e = instance_ids[j];
                g = (e >= 0 && e < E) ? s_gs[e] + (lr - s_off[e]) : -1;
            }
            global_idx[j] = g;
        }
    }
    pdl_launch_dependents();
}

}  // namespace moe
