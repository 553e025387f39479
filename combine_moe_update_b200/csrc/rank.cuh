// rank.cuh -- deterministic expert-major ordering of the dispatched copies.
//
// The EP AllToAllV of aclnnMoeDistributeDispatchV2 ("计算公式") sends each
// token's copies to the ranks owning their experts; on one GPU that is a
// permutation of (token, k) copies into a rank-major receive buffer.  The
// page requires a deterministic result ("确定性计算"), so the row of a copy
// is its position in (instance, token, k) order: a stable counting sort.
//
// One block of 1024 threads, <= 8192 copies, <= 1024 instances:
//   - warp w owns a contiguous run of copies and walks it 32 at a time;
//     __match_any_sync groups equal instance ids, so a copy's rank within
//     its warp is (earlier rounds' count) + (lower lanes with the same id);
//   - a per-instance prefix over the 32 warps turns those into ranks within
//     the instance's bucket;
//   - a block scan over the instance totals gives the bucket offsets.
// No atomics decide an order, so the output is the same on every run.
#pragma once
#include "common.cuh"

namespace moe {

struct RankArgs {
    int items;          // bs * K
    int num_instances;  // E
    const int32_t *ids;
    const uint8_t *mask;  // may be null
    int32_t *expand_idx;
    int32_t *src_of_row;
    int32_t *counts;
    int32_t *offsets;
    uint32_t *err;
};

constexpr int kRkThreads = 1024;
constexpr int kRkMaxRounds = 8;  // 8192 copies / 32 warps / 32 lanes

// Dynamic shared memory: per-(warp, instance) uint16 counters, then the
// bucket offsets.
inline size_t rank_smem_bytes(int num_instances) {
    return 32 * (size_t)num_instances * sizeof(uint16_t) + 1024 * sizeof(int);
}

__global__ void __launch_bounds__(kRkThreads) rank_kernel(RankArgs a) {
    // The dispatch kernel may start now: everything it does before its own
    // pdl_wait() reads only inputs of the dispatch call.
    pdl_launch_dependents();

    extern __shared__ __align__(16) unsigned char smem[];
    const int E = a.num_instances;
    uint16_t *s_wc = reinterpret_cast<uint16_t *>(smem);  // [32][E]
    int *s_off = reinterpret_cast<int *>(smem + 64 * (size_t)E);  // after 32 * E uint16
    __shared__ int s_warp[32];

    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    uint32_t *wc32 = reinterpret_cast<uint32_t *>(s_wc);
    for (int q = t; q < 16 * E; q += kRkThreads) wc32[q] = 0;  // 32 * E uint16
    __syncthreads();

    const int per_warp = (a.items + 31) / 32;
    const int rounds = (per_warp + 31) / 32;
    const int begin = w * per_warp;
    const unsigned lower = (1u << lane) - 1u;

    int key[kRkMaxRounds], local[kRkMaxRounds];
#pragma unroll
    for (int j = 0; j < kRkMaxRounds; ++j) {
        key[j] = -1;
        local[j] = 0;
        if (j >= rounds) continue;  // uniform over the block
        const int off = j * 32 + lane;
        const int it = begin + off;
        int k = -1;
        if (off < per_warp && it < a.items) {
            const bool active = a.mask ? (a.mask[it] != 0) : true;
            if (active) {
                const int id = a.ids[it];
                if (id >= 0 && id < E) k = id;
                else raise_error(a.err, kDevBadId);
            }
        }
        const unsigned peers = __match_any_sync(kFull, k);
        int base = 0;
        if (k >= 0) base = s_wc[w * E + k];
        __syncwarp();
        if (k >= 0 && lane == __ffs(peers) - 1) s_wc[w * E + k] = (uint16_t)(base + __popc(peers));
        __syncwarp();
        key[j] = k;
        local[j] = base + __popc(peers & lower);
    }
    __syncthreads();

    // per-instance exclusive prefix over the warps; instance totals
    int total_b = 0;
    for (int b = t; b < E; b += kRkThreads) {
        int run = 0;
        for (int ww = 0; ww < 32; ++ww) {
            int c = s_wc[ww * E + b];
            s_wc[ww * E + b] = (uint16_t)run;
            run += c;
        }
        total_b = run;  // E <= 1024 = blockDim: thread t owns instance t
    }
    const int incl = block_inclusive_scan(total_b, s_warp);
    if (t < E) {
        s_off[t] = incl - total_b;
        a.counts[t] = total_b;
        a.offsets[t] = incl - total_b;
    }
    if (t == kRkThreads - 1) a.offsets[E] = incl;  // instances >= E contribute 0
    __syncthreads();

#pragma unroll
    for (int j = 0; j < kRkMaxRounds; ++j) {
        if (j >= rounds) continue;
        const int off = j * 32 + lane;
        const int it = begin + off;
        if (off >= per_warp || it >= a.items) continue;
        const int k = key[j];
        if (k < 0) {
            a.expand_idx[it] = -1;
            continue;
        }
        const int row = s_off[k] + s_wc[w * E + k] + local[j];
        a.expand_idx[it] = row;
        a.src_of_row[row] = it;
    }
}

}  // namespace moe
