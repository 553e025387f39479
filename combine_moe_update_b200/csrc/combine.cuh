// combine.cuh -- gather the expert outputs back, weighted top-K sum plus the
// shared-expert term, residual add and RMSNorm, in one pass
// (aclnnMoeDistributeCombineAddRmsNorm, "计算公式"):
//   combineOut = sum_k (s_k * ataOut_k + s_k * sharedExpertX)
//   x = combineOut + residualX
//   y = x / sqrt(mean(x^2) + normEps) * gamma
//
// A persistent kernel: each block owns tokens blockIdx.x, blockIdx.x + grid,
// ... and streams them as a sequence of (token, H-chunk) units.  A unit is
// the chunk of every kept expert row (the AllToAllV back: a gather through
// expand_idx), of the shared-expert row and of the residual row -- each one
// contiguous run of bytes, so one thread moves it into shared memory with a
// single TMA bulk copy that completes on the unit's mbarrier.  kStages units
// are in flight at once: while the block accumulates one unit (fp32, one
// 8-element vector per thread) and, at a token's last chunk, reduces
// sum(x^2) and writes y, the next units are already on their way.  x of the
// current token stays in registers.  Every input byte is read from memory
// once and every output byte written once.
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

constexpr int kCbThreads = 256;
constexpr int kCbChunk = kCbThreads * 8;  // elements per unit: one 8-element vector per thread
constexpr int kCbMaxChunks = 4;           // H <= 8192
constexpr int kCbStages = 2;
constexpr int kCbMaxTokens = 8;           // tokens per block (grid >= bs / 8)

// Rows per unit: K expert rows, the residual, and the shared-expert row.
inline int combine_rows_per_unit(int top_k, bool shared) { return top_k + 1 + (shared ? 1 : 0); }

inline size_t combine_smem_bytes(int top_k, bool shared) {
    return (size_t)kCbStages * combine_rows_per_unit(top_k, shared) * kCbChunk * sizeof(uint16_t);
}

template <int KMAX, bool SHARED>
__global__ void __launch_bounds__(kCbThreads) combine_kernel(CombineArgs a) {
    extern __shared__ __align__(128) uint16_t s_stage[];  // [kStages][rows][kCbChunk]
    __shared__ __align__(8) uint64_t s_full[kCbStages];
    __shared__ int s_row[kCbMaxTokens][16];
    __shared__ float s_w[kCbMaxTokens][16];
    __shared__ float s_red[kCbThreads / 32];

    const int t = threadIdx.x, K = a.top_k, H = a.hidden;
    const int R = K + 1 + (SHARED ? 1 : 0);  // rows per stage: K experts, residual, shared
    const int n_chunks = (H + kCbChunk - 1) / kCbChunk;
    const int n_tok = (a.bs - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;  // tokens of this block
    const int n_units = n_tok * n_chunks;

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
    if (t == 0) {
        for (int s = 0; s < kCbStages; ++s) mbar_init(&s_full[s], 1);
    }
    __syncthreads();

    // Issue unit u into its stage (one thread).
    auto issue = [&](int u) {
        const int lt = u / n_chunks, c = u % n_chunks;
        const int i = blockIdx.x + lt * gridDim.x;
        const int h0 = c * kCbChunk;
        const int len = (H - h0 < kCbChunk ? H - h0 : kCbChunk);
        const uint32_t bytes = (uint32_t)len * sizeof(uint16_t);
        const int st = u % kCbStages;
        uint16_t *base = s_stage + (size_t)st * R * kCbChunk;
        uint32_t total = bytes;  // residual
        for (int k = 0; k < K; ++k) total += s_row[lt][k] >= 0 ? bytes : 0;
        if (SHARED) total += bytes;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&s_full[st], total);
        bulk_copy_g2s(base + (size_t)K * kCbChunk, a.residual + (size_t)i * H + h0, bytes, &s_full[st]);
        if (SHARED) bulk_copy_g2s(base + (size_t)(K + 1) * kCbChunk, a.shared_x + (size_t)i * H + h0, bytes,
                                  &s_full[st]);
        for (int k = 0; k < K; ++k) {
            const int row = s_row[lt][k];
            if (row >= 0)
                bulk_copy_g2s(base + (size_t)k * kCbChunk, a.expand_x + (size_t)row * H + h0, bytes, &s_full[st]);
        }
    };
    if (t == 0)
        for (int u = 0; u < kCbStages && u < n_units; ++u) issue(u);

    // gamma of this thread's vectors, once
    uint4 gv[kCbMaxChunks];
#pragma unroll
    for (int c = 0; c < kCbMaxChunks; ++c) {
        const int h = c * kCbChunk + t * 8;
        gv[c] = (c < n_chunks && h < H) ? ld_cached(a.gamma + h) : make_uint4(0, 0, 0, 0);
    }

    float xs[kCbMaxChunks][8];
    float ss = 0.0f;
    for (int u = 0; u < n_units; ++u) {
        const int lt = u / n_chunks, c = u % n_chunks;
        const int st = u % kCbStages;
        const uint32_t phase = (uint32_t)(u / kCbStages) & 1u;
        // every thread observes the unit's arrival itself; the verdict is block-uniform
        if (!__syncthreads_and(mbar_wait_bounded(&s_full[st], phase))) {
            // never leave with a bulk copy still in flight: one more bounded wait each
            if (t == 0) {
                raise_error(a.err, kDevTimeout);
                for (int v = u; v < u + kCbStages && v < n_units; ++v)
                    mbar_wait_bounded(&s_full[v % kCbStages], (uint32_t)(v / kCbStages) & 1u);
            }
            return;
        }
        const uint16_t *base = s_stage + (size_t)st * R * kCbChunk;
        const int h = c * kCbChunk + t * 8;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
        if (h < H) {
            float wsum = 0.0f;
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                if (k >= K) break;
                const float w = s_w[lt][k];
                wsum += w;
                if (s_row[lt][k] < 0) continue;
                float f[8];
                unpack8(*reinterpret_cast<const uint4 *>(base + (size_t)k * kCbChunk + t * 8), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, f[e], acc[e]);
            }
            if constexpr (SHARED) {
                float f[8];
                unpack8(*reinterpret_cast<const uint4 *>(base + (size_t)(K + 1) * kCbChunk + t * 8), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(wsum, f[e], acc[e]);
            }
            float r[8];
            unpack8(*reinterpret_cast<const uint4 *>(base + (size_t)K * kCbChunk + t * 8), r);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                acc[e] += r[e];
                ss = fmaf(acc[e], acc[e], ss);
            }
        }
#pragma unroll
        for (int cc = 0; cc < kCbMaxChunks; ++cc)
            if (cc == c) {
#pragma unroll
                for (int e = 0; e < 8; ++e) xs[cc][e] = acc[e];
            }
        __syncthreads();  // every thread is done with this stage
        if (t == 0 && u + kCbStages < n_units) issue(u + kCbStages);

        if (c == n_chunks - 1) {  // the token is complete: normalize and write
            const int i = blockIdx.x + lt * gridDim.x;
            const float tot = block_sum<kCbThreads / 32>(ss, s_red);
            ss = 0.0f;
            const float rstd = __frcp_rn(__fsqrt_rn(__fdiv_rn(tot, (float)H) + a.norm_eps));
            if (t == 0 && a.rstd_out) a.rstd_out[i] = rstd;
#pragma unroll
            for (int cc = 0; cc < kCbMaxChunks; ++cc) {
                const int hh = cc * kCbChunk + t * 8;
                if (cc >= n_chunks || hh >= H) continue;
                float g[8];
                unpack8(gv[cc], g);
                uint4 yo;
                yo.x = pack_bf16x2(xs[cc][0] * rstd * g[0], xs[cc][1] * rstd * g[1]);
                yo.y = pack_bf16x2(xs[cc][2] * rstd * g[2], xs[cc][3] * rstd * g[3]);
                yo.z = pack_bf16x2(xs[cc][4] * rstd * g[4], xs[cc][5] * rstd * g[5]);
                yo.w = pack_bf16x2(xs[cc][6] * rstd * g[6], xs[cc][7] * rstd * g[7]);
                st_v4(a.y + (size_t)i * H + hh, yo);
                if (a.x_out) {
                    uint4 xo;
                    xo.x = pack_bf16x2(xs[cc][0], xs[cc][1]);
                    xo.y = pack_bf16x2(xs[cc][2], xs[cc][3]);
                    xo.z = pack_bf16x2(xs[cc][4], xs[cc][5]);
                    xo.w = pack_bf16x2(xs[cc][6], xs[cc][7]);
                    st_v4(a.x_out + (size_t)i * H + hh, xo);
                }
            }
        }
    }
}

}  // namespace moe
