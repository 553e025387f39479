// combine.cuh -- gather the expert outputs back, weighted top-K sum plus the
// shared-expert term, residual add and RMSNorm, in one pass
// (aclnnMoeDistributeCombineAddRmsNorm, "计算公式"):
//   combineOut = sum_k (s_k * ataOut_k + s_k * sharedExpertX)
//   x = combineOut + residualX
//   y = x / sqrt(mean(x^2) + normEps) * gamma
//
// A persistent, warp-specialized kernel, one block per SM.  Block b owns
// tokens b, b + grid, ...; each token is cut into units of 2048 elements.  A
// unit is that slice of every kept expert row (the AllToAllV back: a gather
// through expand_idx), of the residual row and of the shared-expert row --
// each a contiguous run of bytes, moved into shared memory by one TMA bulk
// copy.  One producer warp keeps a ring of STAGES units in flight (a "full"
// mbarrier per stage counts the bytes in, an "empty" one counts the consumer
// warps out); eight consumer warps each take one 8-element vector per row of
// a unit, accumulate in fp32 (packed fp32x2 FMAs, each lane an ordinary IEEE
// FMA) and keep x of the current token in registers.  Only the per-token
// sum(x^2) needs the consumers together (a named barrier); nothing stops the
// producer.  Every input byte is read from memory once, every output byte
// written once.
//
// Every wait is bounded.  A wait that gives up records MOE_DEV_TIMEOUT and the
// thread carries on (its outputs are then wrong, and flagged), so no thread
// ever leaves a barrier short of one arrival.
#pragma once
#include "common.cuh"

namespace moe {

struct CombineArgs {
    int bs, hidden, top_k, expand_rows;
    float norm_eps;
    const uint16_t *expand_x;  // bf16 bits [expand_rows, H]
    const int32_t *expand_idx;
    const float *scales;
    const uint16_t *shared_x;  // may be null
    const uint16_t *residual;
    const uint16_t *gamma;
    uint16_t *y;
    uint16_t *x_out;  // may be null
    float *rstd_out;  // may be null
    uint32_t *err;
};

constexpr int kCbConsumers = 256;                   // 8 consumer warps
constexpr int kCbThreads = kCbConsumers + 32;       // + 1 producer warp
constexpr int kCbChunk = kCbConsumers * 8;          // elements per unit
constexpr int kCbMaxChunks = 4;                     // H <= 8192
constexpr int kCbMaxTokens = 8;                     // tokens per block (grid >= bs / 8)

// Rows per unit: K expert rows, the residual, and the shared-expert row.
inline int combine_rows(int top_k, bool shared) { return top_k + 1 + (shared ? 1 : 0); }

inline size_t combine_smem_bytes(int stages, int top_k, bool shared) {
    return (size_t)stages * combine_rows(top_k, shared) * kCbChunk * sizeof(uint16_t);
}

template <int KMAX, bool SHARED, int STAGES>
__global__ void __launch_bounds__(kCbThreads, 1) combine_kernel(CombineArgs a) {
    extern __shared__ __align__(128) uint16_t s_stage[];  // [STAGES][R][kCbChunk]
    __shared__ __align__(8) uint64_t s_full[STAGES], s_empty[STAGES];
    __shared__ int s_row[kCbMaxTokens][16];
    __shared__ float s_w[kCbMaxTokens][16];
    __shared__ float s_red[kCbConsumers / 32];

    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int K = a.top_k, H = a.hidden, R = K + 1 + (SHARED ? 1 : 0);
    const int n_chunks = (H + kCbChunk - 1) / kCbChunk;
    const int n_tok = (a.bs - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const int n_units = n_tok * n_chunks;

    if (t == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_empty[s], kCbConsumers / 32);
        }
    }
    pdl_wait();  // expand_idx and the expert rows come from earlier kernels

    // rows and weights of every token this block owns
    for (int q = t; q < n_tok * K; q += kCbThreads) {
        const int lt = q / K, k = q % K;
        const int i = blockIdx.x + lt * gridDim.x;
        int row = a.expand_idx[i * K + k];
        const float w = a.scales[i * K + k];
        if (row < -1 || row >= a.expand_rows) {
            raise_error(a.err, kDevBadId);
            row = -1;
        }
        s_row[lt][k] = row;
        s_w[lt][k] = row >= 0 ? w : 0.0f;  // a pruned copy weighs nothing
    }
    __syncthreads();

    if (warp == kCbConsumers / 32) {
        // ------------------------------------------------------- producer
        if (lane == 0) {
            bool ok = true;
            for (int u = 0; u < n_units; ++u) {
                const int st = u % STAGES;
                if (u >= STAGES) ok &= mbar_wait_bounded(&s_empty[st], (uint32_t)((u / STAGES) & 1) ^ 1u);
                const int lt = u / n_chunks, c = u % n_chunks;
                const int i = blockIdx.x + lt * gridDim.x;
                const int h0 = c * kCbChunk;
                const uint32_t bytes = (uint32_t)((H - h0 < kCbChunk ? H - h0 : kCbChunk) * sizeof(uint16_t));
                uint16_t *base = s_stage + (size_t)st * R * kCbChunk;
                uint32_t total = bytes * (1 + (SHARED ? 1 : 0));
                for (int k = 0; k < K; ++k) total += s_row[lt][k] >= 0 ? bytes : 0;
                mbar_arrive_expect_tx(&s_full[st], total);
                bulk_copy_g2s(base + (size_t)K * kCbChunk, a.residual + (size_t)i * H + h0, bytes, &s_full[st]);
                if (SHARED)
                    bulk_copy_g2s(base + (size_t)(K + 1) * kCbChunk, a.shared_x + (size_t)i * H + h0, bytes,
                                  &s_full[st]);
                for (int k = 0; k < K; ++k) {
                    const int row = s_row[lt][k];
                    if (row >= 0)
                        bulk_copy_g2s(base + (size_t)k * kCbChunk, a.expand_x + (size_t)row * H + h0, bytes,
                                      &s_full[st]);
                }
            }
            if (!ok) raise_error(a.err, kDevTimeout);
        }
        pdl_launch_dependents();
        return;
    }

    // ----------------------------------------------------------- consumers
    uint4 gv[kCbMaxChunks];
#pragma unroll
    for (int c = 0; c < kCbMaxChunks; ++c) {
        const int h = c * kCbChunk + t * 8;
        gv[c] = (c < n_chunks && h < H) ? ld_cached(a.gamma + h) : make_uint4(0, 0, 0, 0);
    }
    bool ok = true;
    int u = 0;
    for (int n = 0; n < n_tok; ++n) {
        const int i = blockIdx.x + n * gridDim.x;
        uint64_t w2[KMAX];
        bool live[KMAX];
        float wsum = 0.0f;  // sum of the kept weights, in k order
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            const float w = k < K ? s_w[n][k] : 0.0f;
            live[k] = k < K && s_row[n][k] >= 0;
            w2[k] = f2_pack(w, w);
            wsum += w;
        }
        const uint64_t ws2 = f2_pack(wsum, wsum);

        uint64_t xs[kCbMaxChunks][4];
        uint64_t ss2 = 0ull;
#pragma unroll
        for (int c = 0; c < kCbMaxChunks; ++c) {
            if (c >= n_chunks) break;  // uniform
            const int st = u % STAGES;
            ok &= mbar_wait_bounded(&s_full[st], (uint32_t)((u / STAGES) & 1));
            ++u;
            const uint16_t *base = s_stage + (size_t)st * R * kCbChunk + t * 8;
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
            if (c * kCbChunk + t * 8 < H) {
#pragma unroll
                for (int k = 0; k < KMAX; ++k) {
                    if (!live[k]) continue;
                    const uint4 v = *reinterpret_cast<const uint4 *>(base + (size_t)k * kCbChunk);
                    acc[0] = f2_fma(w2[k], bf16x2_to_f2(v.x), acc[0]);
                    acc[1] = f2_fma(w2[k], bf16x2_to_f2(v.y), acc[1]);
                    acc[2] = f2_fma(w2[k], bf16x2_to_f2(v.z), acc[2]);
                    acc[3] = f2_fma(w2[k], bf16x2_to_f2(v.w), acc[3]);
                }
                if constexpr (SHARED) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(base + (size_t)(K + 1) * kCbChunk);
                    acc[0] = f2_fma(ws2, bf16x2_to_f2(v.x), acc[0]);
                    acc[1] = f2_fma(ws2, bf16x2_to_f2(v.y), acc[1]);
                    acc[2] = f2_fma(ws2, bf16x2_to_f2(v.z), acc[2]);
                    acc[3] = f2_fma(ws2, bf16x2_to_f2(v.w), acc[3]);
                }
                const uint4 r = *reinterpret_cast<const uint4 *>(base + (size_t)K * kCbChunk);
                acc[0] = f2_add(acc[0], bf16x2_to_f2(r.x));
                acc[1] = f2_add(acc[1], bf16x2_to_f2(r.y));
                acc[2] = f2_add(acc[2], bf16x2_to_f2(r.z));
                acc[3] = f2_add(acc[3], bf16x2_to_f2(r.w));
#pragma unroll
                for (int h = 0; h < 4; ++h) ss2 = f2_fma(acc[h], acc[h], ss2);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[st]);  // this warp is done with the stage
#pragma unroll
            for (int h = 0; h < 4; ++h) xs[c][h] = acc[h];
        }

        // the token is complete: sum(x^2) over the consumers, then y
        float v = warp_sum(f2_lo(ss2) + f2_hi(ss2));
        if (lane == 0) s_red[warp] = v;
        named_barrier(1, kCbConsumers);
        float tot = 0.0f;
#pragma unroll
        for (int w = 0; w < kCbConsumers / 32; ++w) tot += s_red[w];  // fixed order: deterministic
        named_barrier(1, kCbConsumers);
        const float rstd = __frcp_rn(__fsqrt_rn(__fdiv_rn(tot, (float)H) + a.norm_eps));
        if (t == 0 && a.rstd_out) a.rstd_out[i] = rstd;
        const uint64_t r2 = f2_pack(rstd, rstd);
#pragma unroll
        for (int c = 0; c < kCbMaxChunks; ++c) {
            const int h = c * kCbChunk + t * 8;
            if (c >= n_chunks || h >= H) continue;
            const uint32_t gw[4] = {gv[c].x, gv[c].y, gv[c].z, gv[c].w};
            uint32_t yo[4], xo[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint64_t yv = f2_mul(f2_mul(xs[c][q], r2), bf16x2_to_f2(gw[q]));
                yo[q] = pack_bf16x2(f2_lo(yv), f2_hi(yv));
                xo[q] = pack_bf16x2(f2_lo(xs[c][q]), f2_hi(xs[c][q]));
            }
            st_v4(a.y + (size_t)i * H + h, make_uint4(yo[0], yo[1], yo[2], yo[3]));
            if (a.x_out) st_v4(a.x_out + (size_t)i * H + h, make_uint4(xo[0], xo[1], xo[2], xo[3]));
        }
    }
    if (!ok) raise_error(a.err, kDevTimeout);
    pdl_launch_dependents();
}

}  // namespace moe
