// dispatch.cuh -- quantize the tokens and scatter their K copies into the
// expert-major receive buffer (aclnnMoeDistributeDispatchV2, "计算公式").
//
// The EP AllToAllV is, on one GPU, a permutation of the (token, k) copies
// into rank-major rows.  The page requires a deterministic result
// ("确定性计算"), so a copy's row is its position in (instance, token, k)
// order: the route kernel computes that order once -- a stable counting sort
// over slices of copies -- and the quantize-and-scatter kernels only look
// their rows up.
//
// The scatter kernels are launched as programmatic dependents of the route
// kernel: everything that depends only on the call's inputs (loading the
// token row and the smooth row, the absmax reduction, the quantization
// itself) runs while the route kernel is still sorting, and only the final
// row writes wait for it.  That is safe because the route kernel releases
// them only after its own wait, when everything before the call is complete.
// A scatter kernel that routes its own copies (FUSED, small calls) is the
// call's first kernel and reads nothing before its wait.
//
// dispatch_token_kernel<MODE>   no smooth scales: one block per token; the
//   row is loaded, quantized once (all K copies are identical) and written K
//   times.
// dispatch_token_smooth_kernel<MODE>  smooth scales (modes 2, 3): one block
//   per token; the row and the K instance ids are loaded once; each copy's
//   smooth row arrives in shared memory by a bulk asynchronous copy, so
//   four blocks fit on an SM and a decode batch runs in one wave.
//
// Quantization, per mode ("计算公式" cases 1 to 5):
//   0  copy the bf16 row;
//   1  static: xFp32 = x * scales (one coefficient, per column, or the
//      destination instance's row); q = Cast(xFp32, int8), saturating;
//   2  xFp32 = x * smooth; dyn = 127 / max|xFp32| over the row;
//      q = rint(xFp32 * dyn); scale = 1 / dyn;
//   3  the same per 128-element tile;
//   4  mxfp8: per 32-element block sharedExp = floor(log2 max|x|) - 8 taken
//      from the exponent bits; q = e4m3_satfinite(x * 2^-sharedExp); scale
//      byte = sharedExp + 127.
// All arithmetic is IEEE binary32 rounded to nearest, so no contraction or
// approximation can move a code.
#pragma once
#include "common.cuh"

namespace moe {

struct DispatchArgs {
    int bs, hidden, top_k, num_instances;
    int tiles;           // ceil(H / 128) (mode 3)
    uint32_t k_magic;    // div_magic(top_k)
    const uint16_t *x;    // bf16 bits [bs, H]
    const int32_t *ids;   // instance ids [bs, K]
    const uint8_t *mask;  // [bs, K] or null
    const float *smooth;  // modes 2/3: [E, H] smooth scales or null; mode 1: static scales
    int scales_len;       // floats in smooth: 0, 1 (one coefficient), H (per column) or E * H (per instance)
    void *expand_x;
    void *dyn_scales;
    int32_t *expand_idx;
    int32_t *src_of_row;
    int32_t *counts;
    int32_t *offsets;
    uint32_t *err;
    // Expert parallelism across GPUs (the EP kernels; the others write
    // expand_x on this GPU).  Copy (instance e, local row r) goes to GPU
    // q = e / ep_el, row gstart[e] + (r - offsets[e]) - gbase[q] of q's
    // receive buffer.
    uint8_t *const *peer_x;      // [G] receive buffers
    uint8_t *const *peer_sc;     // [G] their scales (modes 2 to 4)
    int32_t *const *peer_src;    // [G] copy ids, optional
    const int32_t *gstart;       // [E] global row of this GPU's first copy of each instance
    const int32_t *gbase;        // [G + 1] first global row of every GPU
    int32_t *global_idx;         // [bs, K] out: every copy's global row (-1 if not sent)
    int ep_el, ep_recv_rows, ep_src_base;
    int scale_bytes;             // bytes of one row's scales in the receive buffers
};

// Where a copy's row goes: the row buffer, its scales and the row in them.
struct RowDst {
    uint8_t *x;
    uint8_t *sc;
    int row;
};

// Copy j of instance e at local row r.  On one GPU, row r of expand_x; with
// expert parallelism (EP), the owner's receive buffer.  False if the row
// falls outside the receive buffer (reported by ep_record; the copy is
// dropped).
template <bool EP>
__device__ __forceinline__ bool copy_dst(const DispatchArgs &a, int e, int r, RowDst &d) {
    if constexpr (!EP) {
        d.x = reinterpret_cast<uint8_t *>(a.expand_x);
        d.sc = reinterpret_cast<uint8_t *>(a.dyn_scales);
        d.row = r;
        return true;
    }
    const int q = e / a.ep_el;
    const int grow = a.gstart[e] + (r - a.offsets[e]);
    d.row = grow - a.gbase[q];
    if (d.row < 0 || d.row >= a.ep_recv_rows) return false;
    d.x = a.peer_x[q];
    d.sc = a.peer_sc != nullptr ? a.peer_sc[q] : nullptr;
    return true;
}

// Key of copy j: its instance if it is sent, -1 if masked out, -2 if its id
// is out of range (then it is dropped and reported).
__device__ __forceinline__ int copy_key(const DispatchArgs &a, int j) {
    const int id = ld_in(a.ids + j);  // both loads issue before either is used
    const bool sent = a.mask ? ld_in(a.mask + j) != 0 : true;
    if (!sent) return -1;
    return (id >= 0 && id < a.num_instances) ? id : -2;
}

// ----------------------------------------------------------- route kernel ---
//
// The copies are cut into G = ceil(N / 512) slices of 512 consecutive copies,
// one block of 512 threads (16 warps, one copy per thread) each.  Every block
// builds, in shared memory, the histogram of all sent copies per instance and
// the histogram of the copies of earlier slices (plain atomic adds: counts do
// not depend on order).  A scan of the first gives the bucket offsets; the
// second gives this slice's start inside each bucket.  Inside the slice,
// __match_any_sync groups the lanes of a warp with equal instances, so a
// copy's rank within its warp is the number of lower lanes with the same
// instance, and a per-instance prefix over the 16 warps extends that to the
// slice.  row = bucket offset + earlier slices + rank in the slice, the same
// on every run.

constexpr int kRtThreads = 512;
constexpr int kRtWarps = kRtThreads / 32;
constexpr int kRtKeys = 16;  // keys per thread for the histograms: N <= 8192 = 512 * 16

__host__ __device__ inline int route_slices(int copies) { return (copies + kRtThreads - 1) / kRtThreads; }

// Dynamic shared memory: per-(instance, warp) uint16 counters, then three
// int arrays over the instances (all copies, earlier slices, offsets).
inline size_t route_smem_bytes(int num_instances) {
    return (size_t)num_instances * kRtWarps * sizeof(uint16_t) + 3 * (size_t)num_instances * sizeof(int);
}

__global__ void __launch_bounds__(kRtThreads) route_kernel(DispatchArgs a) {
    extern __shared__ __align__(16) unsigned char smem_r[];
    const int E = a.num_instances, N = a.bs * a.top_k, g = blockIdx.x;
    uint16_t *s_cnt = reinterpret_cast<uint16_t *>(smem_r);                                  // [E][16]
    int *s_all = reinterpret_cast<int *>(smem_r + (size_t)E * kRtWarps * sizeof(uint16_t));  // [E]
    int *s_before = s_all + E;                                                              // [E]
    int *s_off = s_before + E;                                                              // [E]
    __shared__ int s_warp[32];
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int mine0 = g * kRtThreads;  // first copy of this slice

    // shared-memory counters cleared while the previous kernel may still run
    uint32_t *cnt32 = reinterpret_cast<uint32_t *>(s_cnt);
    for (int q = t; q < 8 * E; q += kRtThreads) cnt32[q] = 0;  // E * 16 uint16
    for (int q = t; q < 2 * E; q += kRtThreads) s_all[q] = 0;  // s_all and s_before
    __syncthreads();
    pdl_wait();               // the instance ids may come from the previous kernel
    pdl_launch_dependents();  // the scatter kernel may start its input-only work now

    // every copy's key (for the histograms) and this thread's own copy; the
    // loads are unconditional (indices clamped into range) so that all of
    // them are in flight together
    int key[kRtKeys];
    uint8_t sent[kRtKeys];
    const int jm = mine0 + t;
    int k = ld_in(a.ids + min(jm, N - 1));
    bool k_sent = jm < N;
#pragma unroll
    for (int u = 0; u < kRtKeys; ++u) key[u] = ld_in(a.ids + min(u * kRtThreads + t, N - 1));
    if (a.mask) {
        k_sent = k_sent && ld_in(a.mask + min(jm, N - 1)) != 0;
#pragma unroll
        for (int u = 0; u < kRtKeys; ++u) sent[u] = ld_in(a.mask + min(u * kRtThreads + t, N - 1));
    } else {
#pragma unroll
        for (int u = 0; u < kRtKeys; ++u) sent[u] = 1;
    }
#pragma unroll
    for (int u = 0; u < kRtKeys; ++u) {
        const int id = key[u];
        key[u] = (u * kRtThreads + t < N && sent[u] != 0) ? ((id >= 0 && id < E) ? id : -2) : -1;
    }
    k = k_sent ? ((k >= 0 && k < E) ? k : -2) : -1;
    if (k == -2) {
        raise_error(a.err, kDevBadId);
        k = -1;
    }

#pragma unroll
    for (int u = 0; u < kRtKeys; ++u) {
        const int kk = key[u];
        if (kk >= 0) {
            atomicAdd(&s_all[kk], 1);
            if (u * kRtThreads + t < mine0) atomicAdd(&s_before[kk], 1);
        }
    }
    const unsigned peers = __match_any_sync(kFull, k);
    if (k >= 0 && lane == __ffs(peers) - 1) s_cnt[k * kRtWarps + w] = (uint16_t)__popc(peers);
    const int local = __popc(peers & ((1u << lane) - 1u));
    __syncthreads();

    // per-instance exclusive prefix over the 16 warps of this slice
    for (int b = t; b < E; b += kRtThreads) {
        int run = 0;
#pragma unroll
        for (int q = 0; q < kRtWarps; ++q) {
            const int c = s_cnt[b * kRtWarps + q];
            s_cnt[b * kRtWarps + q] = (uint16_t)run;
            run += c;
        }
    }
    // exclusive scan of the instance totals: 2 consecutive instances per thread (E <= 1024)
    int v2[2], sum = 0;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int b = t * 2 + u;
        v2[u] = b < E ? s_all[b] : 0;
        sum += v2[u];
    }
    const int incl = block_inclusive_scan(sum, s_warp);  // its barriers also publish s_cnt
    const int total = s_warp[kRtWarps - 1];
    int run = incl - sum;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int b = t * 2 + u;
        if (b < E) {
            s_off[b] = run;
            if (g == 0) {
                a.counts[b] = v2[u];
                a.offsets[b] = run;
            }
        }
        run += v2[u];
    }
    if (g == 0 && t == 0) a.offsets[E] = total;
    __syncthreads();

    if (jm < N) {
        if (k < 0) {
            a.expand_idx[jm] = -1;
        } else {
            const int row = s_off[k] + s_before[k] + s_cnt[k * kRtWarps + w] + local;
            a.expand_idx[jm] = row;
            a.src_of_row[row] = jm;
        }
    }
}

// --------------------------------------------------- TP domain counts ---
//
// With a TP domain of two ranks and one instance per EP rank, the rows of
// instance e come from the 2 * ws source devices in TP-major order, so
// TP domain 0's rows of e (sources < ws) come first.  One thread per
// instance finds the first row of domain 1 by a binary search over the
// rows' copy ids (source = id / (bs * K)).
__global__ void __launch_bounds__(1024) tp_counts_kernel(const int32_t *src_of_row, const int32_t *offsets,
                                                         int32_t *tp_counts, int num_instances, int copies,
                                                         int copies_per_source, int ws, uint32_t *err) {
    pdl_wait();  // the routing comes from earlier kernels
    for (int e = threadIdx.x; e < num_instances; e += blockDim.x) {
        const int lo0 = ld_in(offsets + e), hi0 = ld_in(offsets + e + 1);
        if (lo0 < 0 || hi0 < lo0 || hi0 > copies) {
            raise_error(err, kDevBadId);
            tp_counts[2 * e] = 0;
            tp_counts[2 * e + 1] = 0;
            continue;
        }
        int lo = lo0, hi = hi0;  // first row in [lo0, hi0) whose source is >= ws
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (ld_in(src_of_row + mid) / copies_per_source < ws) lo = mid + 1; else hi = mid;
        }
        tp_counts[2 * e] = lo - lo0;
        tp_counts[2 * e + 1] = hi0 - lo;
    }
    pdl_launch_dependents();
}

// ----------------------------------------------------------- block route ---
//
// For a small call (at most kFusedRouteMax copies) every token block
// computes the rows of its own K copies itself and no ordering kernel runs,
// which saves a launch and a dependency on the critical path.  A copy's row is its position in (instance,
// token, k) order.  The block builds, in shared memory, the histogram of all
// sent copies per instance and the histogram of the copies of earlier tokens
// (plain atomic adds: counts do not depend on order), prefix-sums the first
// into bucket offsets, and takes
//   row = offset[e] + (copies of earlier tokens on e)
//         + (this token's earlier copies on e),
// the last from __match_any_sync over the token's K lanes.  Every block gets
// the same counts, so the rows are the same on every run.  Block 0 also
// writes counts and offsets.  Every block reads all the call's ids, so this
// pays only for small calls: larger ones use route_kernel.

constexpr int kMaxInstances = 1024;
constexpr int kFusedRouteMax = 1024;  // copies up to which the token blocks route themselves

template <int EMAX>
struct RouteSmemT {
    int cnt[EMAX];     // sent copies per instance
    int before[EMAX];  // sent copies of earlier tokens per instance
    int off[EMAX];     // exclusive prefix of cnt
    int warp[32];
    int key[32];       // this token's copy keys, by k
    int row[32];       // this token's rows, by k (-1: not sent)
};
using RouteSmem = RouteSmemT<kMaxInstances>;

template <int NT, class RS>
__device__ __forceinline__ void block_route_clear(RS &rs, int E) {
    for (int e = threadIdx.x; e < E; e += NT) {
        rs.cnt[e] = 0;
        rs.before[e] = 0;
    }
}

// Call after pdl_wait, with block_route_clear done and a barrier between.
// key0: for the threads of warp 0, copy_key of this token's copy k = lane
// (-1 for lanes >= K).  Leaves rs.key and rs.row filled, after a barrier.
template <int NT, class RS>
__device__ void block_route(const DispatchArgs &a, int i, RS &rs, int key0, bool writer = true) {
    const int t = threadIdx.x, E = a.num_instances, K = a.top_k, N = a.bs * K, mine0 = i * K;
    constexpr int U = 8;
    for (int j0 = 0; j0 < N; j0 += NT * U) {  // loads unconditional (clamped), so all are in flight together
        int id[U];
        uint32_t ms[U];
#pragma unroll
        for (int u = 0; u < U; ++u) id[u] = ld_in(a.ids + min(j0 + u * NT + t, N - 1));
        if (a.mask) {
#pragma unroll
            for (int u = 0; u < U; ++u) ms[u] = ld_in(a.mask + min(j0 + u * NT + t, N - 1));
        } else {
#pragma unroll
            for (int u = 0; u < U; ++u) ms[u] = 1;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int j = j0 + u * NT + t;
            if (j < N && ms[u] != 0 && id[u] >= 0 && id[u] < E) {
                atomicAdd(&rs.cnt[id[u]], 1);
                if (j < mine0) atomicAdd(&rs.before[id[u]], 1);
            }
        }
    }
    __syncthreads();
    // exclusive scan of cnt: thread t owns P consecutive instances
    const int P = (E + NT - 1) / NT;
    int sum = 0;
    for (int u = 0; u < P; ++u) {
        const int e = t * P + u;
        if (e < E) sum += rs.cnt[e];
    }
    const int incl = block_inclusive_scan(sum, rs.warp);
    int run = incl - sum;
    for (int u = 0; u < P; ++u) {
        const int e = t * P + u;
        if (e < E) {
            rs.off[e] = run;
            if (i == 0 && writer) {
                a.counts[e] = rs.cnt[e];
                a.offsets[e] = run;
            }
            run += rs.cnt[e];
        }
    }
    if (i == 0 && writer && t == NT - 1) a.offsets[E] = incl;  // the total
    __syncthreads();
    if (t < 32) {
        const unsigned peers = __match_any_sync(kFull, key0);
        int row = -1;
        if (key0 >= 0) row = rs.off[key0] + rs.before[key0] + __popc(peers & ((1u << t) - 1u));
        if (key0 == -2) raise_error(a.err, kDevBadId);
        rs.key[t] = key0;
        rs.row[t] = row;
        if (t < K && writer) {
            a.expand_idx[mine0 + t] = row;
            if (row >= 0) a.src_of_row[row] = mine0 + t;
        }
    }
    __syncthreads();
}

// ---------------------------------------------------- route, many copies ---
//
// Past 8192 copies (several source ranks), rebuilding the whole histogram in
// every slice no longer pays, so the same order is built in three passes
// over slices of kRlCopies = 4096 copies with a table in the workspace:
//   route_hist_kernel   slice s counts its sent copies per instance: tab[s][e]
//   route_scan_kernel   per instance, the exclusive prefix of tab[.][e] over
//                       the slices (in place), and the total tot[e]
//   route_place_kernel  slice s: bucket offsets from a block scan of tot,
//                       then 8 rounds of 512 copies, each ranked as in
//                       route_kernel (match_any + per-warp prefix) on top of
//                       a running per-instance count of the earlier rounds.
// row = offset[e] + tab[s][e] + earlier rounds + rank in the round: the same
// (instance, token, k) order as route_kernel.

constexpr int kRlRounds = 8;
constexpr int kRlCopies = kRtThreads * kRlRounds;  // 4096 copies per slice

__host__ __device__ inline int route_large_slices(int copies) { return (copies + kRlCopies - 1) / kRlCopies; }

// The workspace table after the error area: tab [S][E], then tot [E].
inline size_t route_large_bytes(int copies, int num_instances) {
    return ((size_t)route_large_slices(copies) * num_instances + num_instances) * sizeof(int);
}

// Keys of this thread's copies in the rounds of slice s (unconditional,
// clamped loads, so all are in flight together); -1 past the end.
__device__ __forceinline__ void slice_keys(const DispatchArgs &a, int s, int (&key)[kRlRounds]) {
    const int N = a.bs * a.top_k, E = a.num_instances, t = threadIdx.x;
    uint32_t sent[kRlRounds];
#pragma unroll
    for (int u = 0; u < kRlRounds; ++u) key[u] = ld_in(a.ids + min(s * kRlCopies + u * kRtThreads + t, N - 1));
    if (a.mask) {
#pragma unroll
        for (int u = 0; u < kRlRounds; ++u) sent[u] = ld_in(a.mask + min(s * kRlCopies + u * kRtThreads + t, N - 1));
    } else {
#pragma unroll
        for (int u = 0; u < kRlRounds; ++u) sent[u] = 1;
    }
#pragma unroll
    for (int u = 0; u < kRlRounds; ++u) {
        const int id = key[u];
        key[u] = (s * kRlCopies + u * kRtThreads + t < N && sent[u] != 0) ? ((id >= 0 && id < E) ? id : -2) : -1;
    }
}

// Dynamic shared memory: E ints.
__global__ void __launch_bounds__(kRtThreads) route_hist_kernel(DispatchArgs a, int *tab) {
    extern __shared__ __align__(16) int s_h[];
    const int E = a.num_instances, s = blockIdx.x, t = threadIdx.x;
    for (int e = t; e < E; e += kRtThreads) s_h[e] = 0;
    __syncthreads();
    pdl_wait();  // the instance ids may come from the previous kernel
    pdl_launch_dependents();
    int key[kRlRounds];
    slice_keys(a, s, key);
#pragma unroll
    for (int u = 0; u < kRlRounds; ++u) {
        if (key[u] >= 0) atomicAdd(&s_h[key[u]], 1);
        if (key[u] == -2) raise_error(a.err, kDevBadId);  // each copy is in exactly one slice
    }
    __syncthreads();
    for (int e = t; e < E; e += kRtThreads) tab[(size_t)s * E + e] = s_h[e];
}

// One thread per instance: the exclusive prefix of its column over the S
// slices (loads batched by the unrolled loop) and its total.
__global__ void __launch_bounds__(1024) route_scan_kernel(DispatchArgs a, int *tab, int *tot, int S) {
    pdl_wait();
    pdl_launch_dependents();
    const int E = a.num_instances, e = blockIdx.x * 1024 + threadIdx.x;
    if (e >= E) return;
    int run = 0;
#pragma unroll 8
    for (int s = 0; s < S; ++s) {
        const int v = tab[(size_t)s * E + e];
        tab[(size_t)s * E + e] = run;
        run += v;
    }
    tot[e] = run;
}

// Dynamic shared memory: per-(instance, warp) uint16 counters, then four
// int arrays over the instances (offset, slice base, running count, round total).
inline size_t route_place_smem_bytes(int num_instances) {
    return (size_t)num_instances * kRtWarps * sizeof(uint16_t) + 4 * (size_t)num_instances * sizeof(int);
}

__global__ void __launch_bounds__(kRtThreads) route_place_kernel(DispatchArgs a, const int *tab, const int *tot) {
    extern __shared__ __align__(16) unsigned char smem_p[];
    const int E = a.num_instances, N = a.bs * a.top_k, s = blockIdx.x;
    uint16_t *s_cnt = reinterpret_cast<uint16_t *>(smem_p);                                  // [E][16]
    int *s_off = reinterpret_cast<int *>(smem_p + (size_t)E * kRtWarps * sizeof(uint16_t));  // [E]
    int *s_base = s_off + E;                                                                // [E]
    int *s_run = s_base + E;                                                                // [E]
    int *s_rtot = s_run + E;                                                                // [E]
    __shared__ int s_warp[32];
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    for (int e = t; e < E; e += kRtThreads) {
        s_run[e] = 0;
        s_rtot[e] = 0;
    }
    pdl_wait();  // the table and the totals come from the previous kernels
    pdl_launch_dependents();

    int key[kRlRounds];
    slice_keys(a, s, key);
    // bucket offsets: exclusive scan of the totals, 2 consecutive instances per thread (E <= 1024)
    int v2[2], sum = 0;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int b = t * 2 + u;
        v2[u] = b < E ? ld_in(tot + b) : 0;
        sum += v2[u];
    }
    const int incl = block_inclusive_scan(sum, s_warp);
    const int total = s_warp[kRtWarps - 1];
    int run = incl - sum;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int b = t * 2 + u;
        if (b < E) {
            s_off[b] = run;
            if (s == 0) {
                a.counts[b] = v2[u];
                a.offsets[b] = run;
            }
        }
        run += v2[u];
    }
    if (s == 0 && t == 0) a.offsets[E] = total;
    for (int e = t; e < E; e += kRtThreads) s_base[e] = ld_in(tab + (size_t)s * E + e);

    uint32_t *cnt32 = reinterpret_cast<uint32_t *>(s_cnt);
    for (int u = 0; u < kRlRounds; ++u) {
        for (int q = t; q < 8 * E; q += kRtThreads) cnt32[q] = 0;  // E * 16 uint16
        __syncthreads();  // counters clear; the previous round's readers are done
        const int k = key[u];
        const unsigned peers = __match_any_sync(kFull, k);
        if (k >= 0 && lane == __ffs(peers) - 1) s_cnt[k * kRtWarps + w] = (uint16_t)__popc(peers);
        const int local = __popc(peers & ((1u << lane) - 1u));
        __syncthreads();
        for (int b = t; b < E; b += kRtThreads) {  // per-instance prefix over the 16 warps
            s_run[b] += s_rtot[b];                 // the previous round's copies of b
            int r = 0;
#pragma unroll
            for (int q = 0; q < kRtWarps; ++q) {
                const int c = s_cnt[b * kRtWarps + q];
                s_cnt[b * kRtWarps + q] = (uint16_t)r;
                r += c;
            }
            s_rtot[b] = r;
        }
        __syncthreads();
        const int j = s * kRlCopies + u * kRtThreads + t;
        if (j < N) {
            if (k < 0) {
                a.expand_idx[j] = -1;
            } else {
                const int row = s_off[k] + s_base[k] + s_run[k] + s_cnt[k * kRtWarps + w] + local;
                a.expand_idx[j] = row;
                a.src_of_row[row] = j;
            }
        }
        __syncthreads();  // every thread has read this pass's counters
    }
}

// ------------------------------------------------------------ quantizers ---

constexpr int kDpVecs = 4;  // 8-element vectors per thread: H / 8 <= 1024 = 256 * 4

// Threads of a token block for rows of V 8-element vectors: the fewest
// threads, from a fixed set of block sizes, that cover the row with kDpVecs
// vectors each.  H = 7168 (V = 896) takes 224 threads, every one with 4
// vectors, so no warp idles at a per-row barrier.  The block size is a
// template parameter of the kernels, which makes every vector's offset a
// compile-time constant.
__host__ __device__ inline int dp_threads(int V) {
    const int need = ((V + kDpVecs - 1) / kDpVecs + 31) / 32 * 32;
    return need <= 64 ? 64 : need <= 128 ? 128 : need <= 192 ? 192 : need <= 224 ? 224 : 256;
}

// int8 codes of 8 values (4 fp32 pairs) for a finite multiplier dyn.
// rint(v * dyn) is the low byte of v * dyn + 1.5 * 2^23: IEEE addition
// rounds half to even and the spacing there is 1, so the sum is
// 1.5 * 2^23 + rint(v * dyn), exact while |v * dyn| < 2^22.  Here |v| <=
// amax and dyn = RN(127 / amax), so |v * dyn| <= 127 (1 + 2^-24): codes stay
// in [-127, 127] and the clamp to that range is never active.
//
// The product must be rounded to fp32 on its own before the add (the page's
// quantOut = CastToInt8(xFp32 * dynamicScales) rounds it); a fused
// multiply-add would skip that rounding and break ties such as a product
// that rounds to exactly 63.5.  Scalar round-to-nearest intrinsics are never
// contracted (packed fp32x2 pairs are, even with contraction switched off),
// and unlike packed pairs they need no register pairing moves.
constexpr float kRintMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ uint2 int8x8(const uint64_t (&v)[4], float dyn) {
    const uint64_t d2 = f2_pack(dyn, dyn);
    uint32_t b[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint64_t p = f2_mul(v[q], d2);  // both products rounded (packed multiply)
        b[2 * q] = __float_as_uint(__fadd_rn(f2_lo(p), kRintMagic));
        b[2 * q + 1] = __float_as_uint(__fadd_rn(f2_hi(p), kRintMagic));
    }
    const uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
    return make_uint2(lo, hi);
}

// Static int8 codes of 8 values (quantMode 1): Cast(v, int8) rounds half to
// even and saturates to [-128, 127], a NaN giving 0.  Clamping before the
// rounding gives the same codes (every value beyond the range rounds to a
// saturated code either way) and keeps the magic-number add exact.
__device__ __forceinline__ uint2 int8x8_static(const uint64_t (&v)[4]) {
    uint32_t b[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float lo = f2_lo(v[q]), hi = f2_hi(v[q]);
        const float cl = lo != lo ? 0.0f : fminf(fmaxf(lo, -128.0f), 127.0f);
        const float ch = hi != hi ? 0.0f : fminf(fmaxf(hi, -128.0f), 127.0f);
        b[2 * q] = __float_as_uint(__fadd_rn(cl, kRintMagic));
        b[2 * q + 1] = __float_as_uint(__fadd_rn(ch, kRintMagic));
    }
    const uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
    return make_uint2(lo, hi);
}

// The codes when dyn = +inf (amax == 0, or 127 / amax overflows fp32): v * inf
// is +-inf, which saturates to +-127, or NaN (v = 0), which casts to 0.
__device__ __forceinline__ uint32_t q8_inf(float v) { return v > 0.0f ? 0x7fu : (v < 0.0f ? 0x81u : 0u); }
__device__ __forceinline__ uint2 int8x8_inf(const uint64_t (&v)[4]) {
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
        w[h] = q8_inf(f2_lo(v[2 * h])) | (q8_inf(f2_hi(v[2 * h])) << 8) | (q8_inf(f2_lo(v[2 * h + 1])) << 16) |
               (q8_inf(f2_hi(v[2 * h + 1])) << 24);
    return make_uint2(w[0], w[1]);
}

// Codes of this thread's vectors for a multiplier dyn shared by the whole
// block.  The rare dyn = +inf case is a separate branch over all vectors.
__device__ __forceinline__ void int8_vecs(const uint64_t (&v)[kDpVecs][4], float dyn, uint2 (&qv)[kDpVecs]) {
    if (__builtin_expect(isinf(dyn), 0)) {
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) qv[q] = int8x8_inf(v[q]);
    } else {
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) qv[q] = int8x8(v[q], dyn);
    }
}

// max |v| of 8 values with three-input maxima (4 steps, 2 dependent).
__device__ __forceinline__ float abs_max8(const uint64_t (&v)[4]) {
    const float m0 = fmax3(fabsf(f2_lo(v[0])), fabsf(f2_hi(v[0])), fabsf(f2_lo(v[1])));
    const float m1 = fmax3(fabsf(f2_hi(v[1])), fabsf(f2_lo(v[2])), fabsf(f2_hi(v[2])));
    return fmax3(m0, m1, fmaxf(fabsf(f2_lo(v[3])), fabsf(f2_hi(v[3]))));
}

// max |v| over this thread's vectors (vectors past the row's end hold 0).
__device__ __forceinline__ float abs_max_vecs(const uint64_t (&v)[kDpVecs][4]) {
    static_assert(kDpVecs == 4, "the tree below covers four vectors");
    return fmaxf(fmax3(abs_max8(v[0]), abs_max8(v[1]), abs_max8(v[2])), abs_max8(v[3]));
}

// 8 bf16 -> 4 fp32 pairs (exact).
__device__ __forceinline__ void vec_to_f2(const uint4 &x, uint64_t (&v)[4]) {
    v[0] = bf16x2_to_f2(x.x);
    v[1] = bf16x2_to_f2(x.y);
    v[2] = bf16x2_to_f2(x.z);
    v[3] = bf16x2_to_f2(x.w);
}

// sharedExp = floor(log2 amax) - 8 (emax of e4m3), clamped to >= -127; -127
// for an all-zero block.  floor(log2) comes from the exponent field (or the
// leading mantissa bit of a subnormal), never from a logarithm routine.
__device__ __forceinline__ int mx_shared_exp(float amax) {
    if (amax == 0.0f) return -127;
    const uint32_t b = __float_as_uint(amax);
    const int ex = (int)(b >> 23);
    const int fl = ex ? ex - 127 : (31 - __clz(b & 0x7fffffu)) - 149;
    const int se = fl - 8;
    return se < -127 ? -127 : se;
}

// e4m3 codes of 8 values, round to nearest even, saturating at +-448.  The
// multiply by the exact power of two 2^-se equals the page's X / 2^se.
__device__ __forceinline__ uint2 e4m3x8(const uint64_t (&v)[4], int se) {
    const float inv = __uint_as_float((uint32_t)(127 - se) << 23);  // 2^-se; normal for se in [-127, 119]
    const uint64_t i2 = f2_pack(inv, inv);
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint64_t s = f2_mul(v[q], i2);
        w[q] = __nv_cvt_float2_to_fp8x2(make_float2(f2_lo(s), f2_hi(s)), __NV_SATFINITE, __NV_E4M3);
    }
    return make_uint2(w[0] | (w[1] << 16), w[2] | (w[3] << 16));
}

// max over the NW per-warp partials in shared memory, as a tree.
template <int NW>
__device__ __forceinline__ float max_partials(const float *s_red) {
    float v[NW];
#pragma unroll
    for (int w = 0; w < NW; ++w) v[w] = s_red[w];
#pragma unroll
    for (int span = 1; span < NW; span *= 2)
#pragma unroll
        for (int w = 0; w + span < NW; w += 2 * span) v[w] = fmaxf(v[w], v[w + span]);
    return v[0];
}

// Block-wide max of m; every thread turns it into dyn = 127 / max.  One
// barrier; s_red must not be reused before the next barrier.
template <int NT>
__device__ __forceinline__ float block_dyn(float m, float *s_red) {
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
    __syncthreads();
    return __fdiv_rn(127.0f, max_partials<NT / 32>(s_red));  // +inf when the max is 0 or 127 / max overflows
}

// Quantize this thread's vectors of one row for the modes without a
// block-wide reduction (xf: fp32 pairs, x * smooth already applied).
template <int MODE, int NT>
__device__ __forceinline__ void quantize_local(const uint64_t (&xf)[kDpVecs][4], int V, uint2 (&qv)[kDpVecs],
                                               float (&seg)[kDpVecs]) {
    const int t = threadIdx.x;
    if constexpr (MODE == 1) {
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) qv[q] = int8x8_static(xf[q]);
    } else if constexpr (MODE == 3) {
        float dq[kDpVecs];
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {  // a 128-element tile = 16 vectors = 16 consecutive lanes
            float m = abs_max8(xf[q]);       // 0 past the row's end
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 8));
            const bool lead = (t & 15) == 0 && t + q * NT < V;
            float dyn = 0.0f;
            if (lead) dyn = __fdiv_rn(127.0f, m);  // one division per tile
            dyn = __shfl_sync(kFull, dyn, (t & 31) & ~15);
            if (lead) seg[q] = __frcp_rn(dyn);
            dq[q] = dyn;
        }
        // per-tile multipliers: the +inf branch is taken by a warp only if
        // one of its tiles has one
        bool any_inf = false;
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) any_inf = any_inf || isinf(dq[q]);
        if (__builtin_expect(__any_sync(kFull, any_inf), 0)) {
#pragma unroll
            for (int q = 0; q < kDpVecs; ++q) qv[q] = isinf(dq[q]) ? int8x8_inf(xf[q]) : int8x8(xf[q], dq[q]);
        } else {
#pragma unroll
            for (int q = 0; q < kDpVecs; ++q) qv[q] = int8x8(xf[q], dq[q]);
        }
    } else if constexpr (MODE == 4) {
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {  // a 32-element block = 4 consecutive lanes
            float m = abs_max8(xf[q]);
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
            const int se = mx_shared_exp(m);
            seg[q] = __int_as_float(se + 127);
            qv[q] = e4m3x8(xf[q], se);
        }
    }
}

// Write this thread's codes (and scales) of one row.
template <int MODE, int NT>
__device__ __forceinline__ void write_row(const DispatchArgs &a, const RowDst &d, int V, const uint2 (&qv)[kDpVecs],
                                          const float (&seg)[kDpVecs], float row_scale) {
    const int t = threadIdx.x, H = a.hidden, row = d.row;
    uint8_t *dst = d.x + (size_t)row * H;
#pragma unroll
    for (int q = 0; q < kDpVecs; ++q) {
        const int p = t + q * NT;
        if (p >= V) continue;
        *reinterpret_cast<uint2 *>(dst + p * 8) = qv[q];
        if constexpr (MODE == 3) {
            if ((t & 15) == 0) reinterpret_cast<float *>(d.sc)[(size_t)row * a.tiles + (p >> 4)] = seg[q];
        }
        if constexpr (MODE == 4) {
            if ((t & 3) == 0) d.sc[(size_t)row * (H >> 5) + (p >> 2)] = (uint8_t)__float_as_int(seg[q]);
        }
    }
    if constexpr (MODE == 2) {
        if (t == 0) reinterpret_cast<float *>(d.sc)[row] = row_scale;
    }
}

// With expert parallelism, thread t < K of a token block records copy t's
// global row and, at its owner, the copy's id in the group.
__device__ __forceinline__ void ep_record(const DispatchArgs &a, int j, int e, int r) {
    int g = -1;
    if (r >= 0) {
        const int q = e / a.ep_el;
        g = a.gstart[e] + (r - a.offsets[e]);
        const int prow = g - a.gbase[q];
        if (prow < 0) raise_error(a.err, kDevBadId);  // the plan does not match this GPU's routing
        else if (prow >= a.ep_recv_rows) raise_error(a.err, kDevCapacity);
        else if (a.peer_src != nullptr) a.peer_src[q][prow] = a.ep_src_base + j;
    }
    a.global_idx[j] = g;
}

// This thread's vectors of a bf16 row (zeros past the row's end).
template <int NT>
__device__ __forceinline__ void load_row(const uint16_t *row, int V, uint4 (&xv)[kDpVecs]) {
#pragma unroll
    for (int q = 0; q < kDpVecs; ++q) {
        const int p = threadIdx.x + q * NT;
        xv[q] = p < V ? ld_stream(row + p * 8) : make_uint4(0, 0, 0, 0);
    }
}

// --------------------------------------------------------- token kernel ---

// FUSED: the block routes its own copies (block_route, small calls) instead
// of reading the rows route_kernel wrote.
// EP: rows go to their owners' receive buffers (expert parallelism across
// GPUs); the rows were routed by an earlier call, so this kernel is its
// call's first and waits before it reads anything.
template <int MODE, int NT, bool FUSED, bool EP = false>
__global__ void __launch_bounds__(NT) dispatch_token_kernel(DispatchArgs a) {
    static_assert(!(FUSED && EP), "an EP scatter follows an earlier route call");
    __shared__ float s_red[NT / 32];
    __shared__ int s_row[16];
    __shared__ RouteSmemT<FUSED ? kMaxInstances : 1> rs;
    // EP: copy k's destination in its owner's receive buffer (row -1: none),
    // resolved once per token rather than by every thread at every copy
    __shared__ uint8_t *s_dx[EP ? 16 : 1], *s_dsc[EP ? 16 : 1];
    __shared__ int s_drow[EP ? 16 : 1];
    const int i = blockIdx.x, t = threadIdx.x;
    const int H = a.hidden, V = H >> 3, K = a.top_k;
    if constexpr (FUSED) {
        // This kernel is the call's first: x itself may come from the kernel
        // before it (a combine whose y feeds the next layer), so nothing is
        // read before the wait.  The x loads issued right after it stay in
        // flight while the block routes its copies.
        block_route_clear<NT>(rs, a.num_instances);
        if (t == 0) prefetch_l2(a.x + (size_t)i * H, (uint32_t)H * 2u);  // the token row, while the predecessor drains
        pdl_wait();
    } else if constexpr (EP) {
        if (t == 0) prefetch_l2(a.x + (size_t)i * H, (uint32_t)H * 2u);
        pdl_wait();
    }

    // FUSED: after the wait.  Otherwise this kernel follows the call's route
    // kernel, which releases it only after its own wait, so every input of
    // the call is final and may be read before this kernel's wait.
    uint4 xv[kDpVecs];
    load_row<NT>(a.x + (size_t)i * H, V, xv);
    uint2 qv[kDpVecs];
    float seg[kDpVecs] = {0.0f, 0.0f, 0.0f, 0.0f};
    float row_scale = 0.0f;
    auto quantize = [&]() {
        if constexpr (MODE != 0) {
            uint64_t xf[kDpVecs][4];
#pragma unroll
            for (int q = 0; q < kDpVecs; ++q) vec_to_f2(xv[q], xf[q]);
            if constexpr (MODE == 1) {  // xFp32 = x * scales: one coefficient, or one per column
                if (a.scales_len == 1) {
                    const float c = ld_in(a.smooth);
                    const uint64_t c2 = f2_pack(c, c);
#pragma unroll
                    for (int q = 0; q < kDpVecs; ++q)
#pragma unroll
                        for (int j = 0; j < 4; ++j) xf[q][j] = f2_mul(xf[q][j], c2);
                } else {
#pragma unroll
                    for (int q = 0; q < kDpVecs; ++q) {
                        const int p = t + q * NT;
                        if (p >= V) continue;
                        const float4 s0 = ld_in(reinterpret_cast<const float4 *>(a.smooth + p * 8));
                        const float4 s1 = ld_in(reinterpret_cast<const float4 *>(a.smooth + p * 8) + 1);
                        xf[q][0] = f2_mul(xf[q][0], f2_pack(s0.x, s0.y));
                        xf[q][1] = f2_mul(xf[q][1], f2_pack(s0.z, s0.w));
                        xf[q][2] = f2_mul(xf[q][2], f2_pack(s1.x, s1.y));
                        xf[q][3] = f2_mul(xf[q][3], f2_pack(s1.z, s1.w));
                    }
                }
            }
            if constexpr (MODE == 2) {
                const float dyn = block_dyn<NT>(abs_max_vecs(xf), s_red);
                row_scale = __frcp_rn(dyn);  // 1 / dynamicScales
                int8_vecs(xf, dyn, qv);
            } else {
                quantize_local<MODE, NT>(xf, V, qv, seg);
            }
        }
    };

    if constexpr (FUSED) {
        __syncthreads();  // the counters are clear
        block_route<NT>(a, i, rs, t < 32 && t < K ? copy_key(a, i * K + t) : -1);
        pdl_launch_dependents();
        quantize();  // x arrived while the block routed
    } else {
        quantize();  // while the route kernel is still sorting
        pdl_wait();  // the rows come from route_kernel
        if (t < K) {
            const int r = a.expand_idx[i * K + t];
            s_row[t] = r;
            if constexpr (EP) {
                const int e = a.ids[i * K + t];
                ep_record(a, i * K + t, e, r);
                RowDst d{nullptr, nullptr, -1};
                const bool ok = r >= 0 && copy_dst<true>(a, e, r, d);  // r >= 0: e is in range
                s_dx[t] = d.x;
                s_dsc[t] = d.sc;
                s_drow[t] = ok ? d.row : -1;
            }
        }
        __syncthreads();
    }
    for (int k = 0; k < K; ++k) {
        const int row = FUSED ? rs.row[k] : s_row[k];
        if (row < 0) continue;
        RowDst d;
        if constexpr (EP) {
            d.x = s_dx[k];
            d.sc = s_dsc[k];
            d.row = s_drow[k];
            if (d.row < 0) continue;
        } else {
            copy_dst<false>(a, 0, row, d);
        }
        if constexpr (MODE == 0) {
            uint16_t *dst = reinterpret_cast<uint16_t *>(d.x) + (size_t)d.row * H;
#pragma unroll
            for (int q = 0; q < kDpVecs; ++q) {
                const int p = t + q * NT;
                if (p < V) st_v4(dst + p * 8, xv[q]);
            }
        } else {
            write_row<MODE, NT>(a, d, V, qv, seg, row_scale);
        }
    }
}

// -------------------------------------------------- token smooth kernel ---
//
// Smooth scales (modes 2, 3), one block per token.  The token's row stays in
// registers; warp 0 lists the token's sent copies.  Each copy's smooth row
// (H fp32) is brought into shared memory by one bulk asynchronous copy
// issued as soon as every thread has read the previous row, so no registers
// hold rows in flight: the block stays small enough (at most 72 registers a
// thread at 224 threads) for four blocks per SM, so a 512-token batch runs
// in a single wave with the other blocks covering each one's waits.
//
// Small batches (too few tokens to fill the SMs) split each token's sent
// copies over P = gridDim.y blocks: block (i, p) quantizes copies p, p + P,
// ... of token i, so more copies run at once; every such block loads the
// token's row itself.
//
// Per copy: wait for the smooth row; xFp32 = x * smooth; mode 2 publishes
// each warp's partial max and takes one barrier (which also frees the
// shared row for the next copy's load), then every thread finishes the max,
// dyn = 127 / max and the codes; mode 3's reductions stay within 16 lanes.

// The shared smooth row, padded to the NT * kDpVecs vectors the threads
// cover, so that every thread reads all its vectors without a bound check;
// the padding is zeroed once and no copy writes it (x is 0 there too).
template <int NT>
__host__ __device__ inline int smooth_smem_floats(int hidden) {
    return hidden > NT * kDpVecs * 8 ? hidden : NT * kDpVecs * 8;
}

template <int MODE, int NT, bool FUSED, bool EP = false, bool GROUPS = false>
__global__ void __launch_bounds__(NT, NT <= 224 ? 4 : 3) dispatch_token_smooth_kernel(DispatchArgs a) {
    static_assert(!(FUSED && EP), "an EP scatter follows an earlier route call");
    constexpr int NW = NT / 32;
    extern __shared__ __align__(128) float s_smooth[];  // the current copy's smooth row, then zeros
    __shared__ float s_red[2][NW];
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ int s_key[16], s_pos[16], s_row[16], s_ns;
    __shared__ RouteSmemT<FUSED ? kMaxInstances : 1> rs;
    // EP: copy k's destination in its owner's receive buffer (row -1: none),
    // resolved once per token rather than by every thread at every copy
    __shared__ uint8_t *s_dx[EP ? 16 : 1], *s_dsc[EP ? 16 : 1];
    __shared__ int s_drow[EP ? 16 : 1];
    const int i = blockIdx.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int P = GROUPS ? (int)gridDim.y : 1, p = GROUPS ? (int)blockIdx.y : 0;  // copy group p of the token's P
    const int H = a.hidden, V = H >> 3, K = a.top_k;
    const uint32_t row_bytes = (uint32_t)H * sizeof(float);  // a multiple of 16 (H % 16 == 0)

    // Shared-memory banks: a 16-byte read per lane at a 32-byte lane stride
    // would put two lanes of each quarter-warp on the same banks.  Lanes
    // with bit 2 set therefore hold their vectors' two 4-element halves
    // swapped (x here, the smooth halves at the reads, the codes back at the
    // writes), so each quarter-warp's reads cover all 32 banks once.
    const bool swap = (lane >> 2) & 1;
    for (int e = H + t; e < smooth_smem_floats<NT>(H); e += NT) s_smooth[e] = 0.0f;
    if constexpr (FUSED) {
        // The call's first kernel: x, the ids and the scales may all come
        // from the kernel before it, so nothing is read before the wait.
        block_route_clear<NT>(rs, a.num_instances);
        if (t == 0) {
            mbar_init(&s_bar, 1);
            prefetch_l2(a.x + (size_t)i * H, (uint32_t)H * 2u);  // the token row, while the predecessor drains
        }
        __syncthreads();
        pdl_wait();
    } else if constexpr (EP) {
        if (t == 0) prefetch_l2(a.x + (size_t)i * H, (uint32_t)H * 2u);
        pdl_wait();  // the call's first kernel (routed by an earlier call)
    }
    // FUSED: after the wait.  Otherwise the call's route kernel runs first
    // and releases this kernel only after its own wait, so the call's inputs
    // are final and may be read before this kernel's wait.
    uint4 xv[kDpVecs];
    load_row<NT>(a.x + (size_t)i * H, V, xv);
#pragma unroll
    for (int q = 0; q < kDpVecs; ++q)
        if (swap) xv[q] = make_uint4(xv[q].z, xv[q].w, xv[q].x, xv[q].y);
    const float *s_first = s_smooth + (swap ? 4 : 0), *s_second = s_smooth + (swap ? 0 : 4);
    int key0 = -1;
    if (w == 0) {  // the sent copies, in k order: instance and position k
        key0 = lane < K ? copy_key(a, i * K + lane) : -1;
        const unsigned sent = __ballot_sync(kFull, key0 >= 0);
        if (key0 >= 0) {
            const int c = __popc(sent & ((1u << lane) - 1u));
            s_key[c] = key0;
            s_pos[c] = lane;
        }
        if (lane == 0) {
            s_ns = __popc(sent);
            if constexpr (!FUSED) mbar_init(&s_bar, 1);
        }
    }
    __syncthreads();
    const int ns = s_ns;
    auto fetch_smooth = [&](int c) {  // thread 0 only
        mbar_arrive_expect_tx(&s_bar, row_bytes);
        bulk_copy_g2s(s_smooth, a.smooth + (size_t)s_key[c] * H, row_bytes, &s_bar);
    };
    if (t == 0 && p < ns) fetch_smooth(p);
    if constexpr (FUSED) block_route<NT>(a, i, rs, key0, p == 0);  // while the first smooth row is in flight

    int jj = 0;  // copies this block has taken (the mbarrier's phase and the partials' buffer)
    for (int c = p; c < ns; c += P, ++jj) {
        const int j = GROUPS ? jj : c;
        const bool landed = mbar_wait_bounded(&s_bar, j & 1);
        uint64_t xf[kDpVecs][4];
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {  // xFp32 = x * smooth (0 past the row's end)
            const int p = t + q * NT;
            uint64_t f[4];
            vec_to_f2(xv[q], f);
            const float4 s0 = *reinterpret_cast<const float4 *>(s_first + p * 8);
            const float4 s1 = *reinterpret_cast<const float4 *>(s_second + p * 8);
            xf[q][0] = f2_mul(f[0], f2_pack(s0.x, s0.y));
            xf[q][1] = f2_mul(f[1], f2_pack(s0.z, s0.w));
            xf[q][2] = f2_mul(f[2], f2_pack(s1.x, s1.y));
            xf[q][3] = f2_mul(f[3], f2_pack(s1.z, s1.w));
        }
        uint2 qv[kDpVecs];
        float seg[kDpVecs] = {0.0f, 0.0f, 0.0f, 0.0f};
        float row_scale = 0.0f;
        if constexpr (MODE == 2) {
            const float m = warp_max(abs_max_vecs(xf));
            if (lane == 0) s_red[j & 1][w] = m;
        }
        // every thread has read the smooth row (and published its partial):
        // the buffer may be refilled.  A row that never landed stops the
        // block (the same verdict in every thread) once a second bounded
        // wait has given the copy in flight its chance to finish.
        if (__syncthreads_or(!landed)) {
            if (t == 0) {
                raise_error(a.err, kDevTimeout);
                mbar_wait_bounded(&s_bar, j & 1);
            }
            return;
        }
        if (t == 0 && c + P < ns && !(kSkipOneCopy && blockIdx.x == 0 && c == 0)) {
            fence_proxy_async_smem();
            fetch_smooth(c + P);
        }
        if (c + P >= ns) pdl_launch_dependents();  // the next kernel may be scheduled as blocks finish
        if constexpr (MODE == 2) {
            const float dyn = __fdiv_rn(127.0f, max_partials<NW>(s_red[j & 1]));  // +inf when the max is 0
            row_scale = __frcp_rn(dyn);                                           // or 127 / max overflows
            int8_vecs(xf, dyn, qv);
        } else {
            quantize_local<MODE, NT>(xf, V, qv, seg);
        }
        if (!FUSED && j == 0) {
            pdl_wait();  // the rows come from the route kernel
            if (t < K) {
                const int r = a.expand_idx[i * K + t];
                s_row[t] = r;
                if constexpr (EP) {
                    const int e = a.ids[i * K + t];
                    if (p == 0) ep_record(a, i * K + t, e, r);  // once per token
                    RowDst d{nullptr, nullptr, -1};
                    const bool ok = r >= 0 && copy_dst<true>(a, e, r, d);  // r >= 0: e is in range
                    s_dx[t] = d.x;
                    s_dsc[t] = d.sc;
                    s_drow[t] = ok ? d.row : -1;
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q)
            if (swap) qv[q] = make_uint2(qv[q].y, qv[q].x);
        RowDst d;
        bool ok;
        if constexpr (EP) {
            const int k = s_pos[c];
            d.x = s_dx[k];
            d.sc = s_dsc[k];
            d.row = s_drow[k];
            ok = d.row >= 0;
        } else {
            ok = copy_dst<false>(a, s_key[c], FUSED ? rs.row[s_pos[c]] : s_row[s_pos[c]], d);
        }
        if (ok) write_row<MODE, NT>(a, d, V, qv, seg, row_scale);
    }
    // A block with no copy still waits for the route kernel, so that this
    // grid ends after it: the next call reads the rows and counts it wrote.
    // With EP the token's first block records its copies' global rows (all
    // -1 then: no copy of the token was sent) for the combine.
    if constexpr (!FUSED) {
        if (ns <= p) {
            pdl_wait();
            if constexpr (EP)
                if (p == 0 && t < K) ep_record(a, i * K + t, a.ids[i * K + t], a.expand_idx[i * K + t]);
        }
    }
}

}  // namespace moe
