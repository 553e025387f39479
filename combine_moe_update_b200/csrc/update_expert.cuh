// update_expert.cuh -- logical expert -> deployed instance, plus pruning.
//
// Follows aclnnMoeUpdateExpert (description: "Load balancing", "Expert
// pruning"; "Restriction on the shape format" for the mapping table).  Each
// block of 1024 threads stages the table in shared memory and does the table
// bookkeeping (steps 1-3, at most 1024 instance positions) itself, then maps
// its own slice of 1024 copies (step 4); the blocks run on different SMs.
//
//   1. Read n_e (column 0) for every logical expert, check 1 <= n_e <= F-1,
//      and prefix-sum it: instance (e, j) gets position first[e] + j.
//   2. Thread p owns position p (<= 1024 positions): it finds its expert by
//      binary search and reads the hosting rank from the table.
//   3. Stable ranking of the positions by rank gives each instance its slot
//      on that rank (earlier positions first), and checks that every rank
//      hosts exactly L = total / ws instances.  inst = rank * L + slot.
//   4. Every (token i, k) copy takes replica i mod n_e of its expert; the
//      keep bit is mask[i] and "not (scale < threshold)".
#pragma once
#include "common.cuh"

namespace moe {

struct UpdateArgs {
    int bs, top_k, num_logical, table_cols, ep_world_size;
    uint32_t k_magic;  // div_magic(top_k)
    float prune_threshold;
    const int32_t *expert_ids;
    const float *expert_scales;  // may be null
    const uint8_t *active_mask;  // may be null
    const int32_t *table;
    int table_mode;  // 0: read from global memory; 1: staged in shared memory by loads; 2: by one bulk copy
    int32_t *balanced_ids;
    uint8_t *balanced_mask;
    uint32_t *err;
};

constexpr int kUeThreads = 1024;
constexpr int kUeItems = 1;  // copies per thread; a block maps kUeThreads * kUeItems copies

// Blocks for `items` copies.  Every block repeats the table bookkeeping (a
// few thousand shared-memory operations) and maps its own slice of copies,
// so the slices run on different SMs at once.
__host__ __device__ inline int update_expert_blocks(int items) {
    return (items + kUeThreads * kUeItems - 1) / (kUeThreads * kUeItems);
}

// Dynamic shared memory: n[1024], first[1024], inst[1024], the division
// magic of every n[e] (1024), one uint16 counter per (rank, warp), then (in
// table modes 1 and 2) the whole [E, F] table, 16-byte aligned.
__host__ __device__ inline size_t update_expert_counters_bytes(int ep_world_size) {
    return ((32 * (size_t)ep_world_size * sizeof(uint16_t)) + 15) / 16 * 16;
}
inline size_t update_expert_smem_bytes(int ep_world_size, int table_mode, int num_logical, int table_cols) {
    return 4 * 1024 * sizeof(int) + update_expert_counters_bytes(ep_world_size) +
           (table_mode ? (size_t)num_logical * table_cols * sizeof(int32_t) : 0);
}
// Tables up to this size are staged in shared memory: both table reads of
// the kernel (column 0, then one entry per instance) then cost no dependent
// global-memory round trip.
constexpr size_t kUeTableSmemMax = 160 * 1024;

// Drop this block's slice of copies (a bad table drops every copy).
__device__ __forceinline__ void update_expert_drop_all(const UpdateArgs &a) {
    const int n = min(a.bs * a.top_k, (int)(blockIdx.x + 1) * kUeThreads * kUeItems);
    for (int it = blockIdx.x * kUeThreads * kUeItems + threadIdx.x; it < n; it += blockDim.x) {
        a.balanced_ids[it] = -1;
        a.balanced_mask[it] = 0;
    }
    if (threadIdx.x == 0) raise_error(a.err, kDevBadTable);
}

__global__ void __launch_bounds__(kUeThreads) update_expert_kernel(UpdateArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    int *s_n = reinterpret_cast<int *>(smem);
    int *s_first = s_n + 1024;
    int *s_inst = s_first + 1024;
    uint32_t *s_mag = reinterpret_cast<uint32_t *>(s_inst + 1024);  // div_magic(n[e])
    const int32_t *s_tab = reinterpret_cast<const int32_t *>(
        smem + 4 * 1024 * sizeof(int) + update_expert_counters_bytes(a.ep_world_size));
    __shared__ __align__(8) uint64_t s_tab_bar;
    uint16_t *s_wc = reinterpret_cast<uint16_t *>(s_mag + 1024);   // [ws][32]
    __shared__ int s_warp[32];
    __shared__ int s_bad, s_total;

    // Ask L2 for the table and this block's slice of ids and scales while
    // the previous kernel drains: a prefetch returns nothing to the program
    // and L2 is the point of coherence, so it is safe on data a predecessor
    // may still write.  Only whole 16-byte words inside each array.
    if (threadIdx.x < 3) {
        const int items = a.bs * a.top_k, base = blockIdx.x * kUeThreads * kUeItems;
        const int mine = min(kUeThreads * kUeItems, items - base);
        const void *ptr = threadIdx.x == 0 ? (const void *)a.table
                        : threadIdx.x == 1 ? (const void *)(a.expert_ids + base)
                                           : (const void *)(a.expert_scales ? a.expert_scales + base : nullptr);
        const uint32_t bytes = threadIdx.x == 0 ? (uint32_t)(a.num_logical * a.table_cols) * 4u : (uint32_t)mine * 4u;
        if (ptr != nullptr && (reinterpret_cast<uintptr_t>(ptr) & 15) == 0 && (bytes & ~15u) != 0)
            prefetch_l2(ptr, bytes & ~15u);
    }
    pdl_wait();               // the ids may come from the previous kernel
    pdl_launch_dependents();  // the next kernel waits for this one before it reads anything

    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int F = a.table_cols, ws = a.ep_world_size, E = a.num_logical;
    const uint32_t tab_bytes = (uint32_t)(E * F) * sizeof(int32_t);

    // The table first (one bulk copy in mode 2), then the copies' inputs,
    // which do not depend on it, so that all the loads are in flight together.
    if (a.table_mode == 2 && t == 0) {
        mbar_init(&s_tab_bar, 1);
        if (!kSkipOneCopy) {
            mbar_arrive_expect_tx(&s_tab_bar, tab_bytes);
            bulk_copy_g2s(const_cast<int32_t *>(s_tab), a.table, tab_bytes, &s_tab_bar);
        }
    }
    if (a.table_mode == 1)
        for (int q = t; q < E * F; q += kUeThreads) const_cast<int32_t *>(s_tab)[q] = ld_in(a.table + q);
    const int items = a.bs * a.top_k;
    const int base = blockIdx.x * kUeThreads * kUeItems;  // this block's first copy
    // Every load is unconditional (indices clamped into range), so all of
    // them are in flight together; items past the end are discarded below.
    int pe[kUeItems];
    float ps[kUeItems];
    bool pa[kUeItems];
#pragma unroll
    for (int u = 0; u < kUeItems; ++u) pe[u] = ld_in(a.expert_ids + min(base + t + u * kUeThreads, items - 1));
#pragma unroll
    for (int u = 0; u < kUeItems; ++u) ps[u] = 0.0f;
    if (a.expert_scales) {
#pragma unroll
        for (int u = 0; u < kUeItems; ++u)
            ps[u] = ld_in(a.expert_scales + min(base + t + u * kUeThreads, items - 1));
    }
#pragma unroll
    for (int u = 0; u < kUeItems; ++u) pa[u] = true;
    if (a.active_mask) {
#pragma unroll
        for (int u = 0; u < kUeItems; ++u)
            pa[u] = ld_in(a.active_mask +
                          div_by_magic((uint32_t)min(base + t + u * kUeThreads, items - 1), a.k_magic)) != 0;
    }
#pragma unroll
    for (int u = 0; u < kUeItems; ++u)
        if (base + t + u * kUeThreads >= items) pe[u] = -1;

    if (t == 0) s_bad = 0;
    for (int q = t; q < 32 * ws; q += kUeThreads) s_wc[q] = 0;
    __syncthreads();  // also publishes the mbarrier's initialisation (and a loaded table)
    const bool tab_ok = a.table_mode != 2 || mbar_wait_bounded(&s_tab_bar, 0);
    if (__syncthreads_or(!tab_ok)) {  // the table copy never landed: report, wait once more, drop all
        if (t == 0) {
            raise_error(a.err, kDevTimeout);
            mbar_wait_bounded(&s_tab_bar, 0);
        }
        update_expert_drop_all(a);
        return;
    }
    const int32_t *tab = a.table_mode ? s_tab : a.table;

    // 1. instance counts and their prefix sum
    int n = 0;
    if (t < E) {
        n = tab[(size_t)t * F];
        if (n < 1 || n > F - 1) {
            s_bad = 1;
            n = 0;
        }
    }
    const int incl = block_inclusive_scan(n, s_warp);
    if (t < E) {
        s_n[t] = n;
        s_first[t] = incl - n;
        s_mag[t] = div_magic((uint32_t)n);
    }
    if (t == kUeThreads - 1) s_total = incl;
    __syncthreads();
    const int total = s_total;
    if (t == 0 && (total < 1 || total > 1024 || total % ws != 0)) s_bad = 1;
    __syncthreads();
    if (s_bad) {
        update_expert_drop_all(a);
        return;
    }
    const int L = total / ws;

    // 2. the rank of instance position t
    int r = -1;
    if (t < total) {
        int lo = 0, hi = E - 1;  // largest e with first[e] <= t (first is strictly increasing)
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (s_first[mid] <= t) lo = mid; else hi = mid - 1;
        }
        r = tab[(size_t)lo * F + 1 + (t - s_first[lo])];
        if (r < 0 || r >= ws) {
            s_bad = 1;
            r = -1;
        }
    }

    // 3. stable rank by r: lanes of one warp first, then warps in order
    const unsigned peers = __match_any_sync(kFull, r);
    const int intra = __popc(peers & ((1u << lane) - 1u));
    if (r >= 0 && lane == __ffs(peers) - 1) s_wc[r * 32 + w] = (uint16_t)__popc(peers);
    __syncthreads();
    if (s_bad) {
        update_expert_drop_all(a);
        return;
    }
    // per-rank exclusive prefix over the 32 warps: one shuffle scan per rank
#pragma unroll 4
    for (int rr = w; rr < ws; rr += 32) {
        const int c = s_wc[rr * 32 + lane];
        const int inc = warp_inclusive_scan(c);
        s_wc[rr * 32 + lane] = (uint16_t)(inc - c);
        if (lane == 31 && inc != L) s_bad = 1;  // every rank hosts the same number of instances
    }
    __syncthreads();
    if (s_bad) {
        update_expert_drop_all(a);
        return;
    }
    if (t < total) s_inst[t] = r * L + s_wc[r * 32 + w] + intra;
    __syncthreads();

    // 4. every (token, k) copy
#pragma unroll
    for (int u = 0; u < kUeItems; ++u) {
        const int it = base + t + u * kUeThreads;
        if (it >= items) continue;
        const int i = (int)div_by_magic((uint32_t)it, a.k_magic);  // it / K
        const int e = pe[u];
        if (e < 0 || e >= E) {
            raise_error(a.err, kDevBadId);
            a.balanced_ids[it] = -1;
            a.balanced_mask[it] = 0;
            continue;
        }
        const int ne = s_n[e];
        const int j = i - ne * (int)div_by_magic((uint32_t)i, s_mag[e]);  // replica i mod n_e
        a.balanced_ids[it] = s_inst[s_first[e] + j];
        bool keep = pa[u];
        if (a.expert_scales && a.prune_threshold > 0.0f && ps[u] < a.prune_threshold) keep = false;
        a.balanced_mask[it] = keep ? 1 : 0;
    }
}

}  // namespace moe
