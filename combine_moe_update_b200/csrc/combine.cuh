// combine.cuh -- gather the expert outputs back, weighted top-K sum plus the
// shared-expert term, residual add and RMSNorm, in one pass
// (aclnnMoeDistributeCombineAddRmsNorm, "计算公式"):
//   combineOut = sum_k (s_k * ataOut_k + s_k * sharedExpertX)
//   x = combineOut + residualX
//   y = x / sqrt(mean(x^2) + normEps) * gamma
//
// A persistent kernel, one block per SM: block b owns tokens b, b + grid, ...
// Thread t owns the 8-element vectors p = t, t + 256, ... of every row.  A
// "unit" is one such vector slot of one token: the slot of every kept expert
// row (the AllToAllV back, a gather through expand_idx), of the residual row
// and of the shared-expert row.  Each thread streams its own units through a
// DEPTH-deep ring of private shared-memory slots with 16-byte cp.async, so
// DEPTH - 1 units per thread are always in flight and no barrier sits on the
// load path; only the per-token sum(x^2) needs the block.  Accumulation is
// fp32 (packed fp32x2 FMAs, each lane an ordinary IEEE FMA) and x of the
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
constexpr int kCbVecs = 4;       // 8-element vectors per thread: H / 8 <= 1024
constexpr int kCbMaxTokens = 8;  // tokens per block (grid >= bs / 8)

// Ring slots: [depth][K experts + residual + shared][kCbThreads] x 16 bytes.
inline size_t combine_smem_bytes(int depth, int top_k, bool shared) {
    return (size_t)depth * (top_k + 1 + (shared ? 1 : 0)) * kCbThreads * sizeof(uint4);
}

template <int KMAX, bool SHARED, int DEPTH>
__global__ void __launch_bounds__(kCbThreads) combine_kernel(CombineArgs a) {
    extern __shared__ __align__(16) uint4 s_buf[];
    __shared__ int s_row[kCbMaxTokens][16];
    __shared__ float s_w[kCbMaxTokens][16];
    __shared__ float s_red[kCbThreads / 32];

    const int t = threadIdx.x, K = a.top_k, H = a.hidden, V = H >> 3;
    const int R = K + 1 + (SHARED ? 1 : 0);
    const int J = (V + kCbThreads - 1) / kCbThreads;  // vector slots per thread (uniform)
    const int n_tok = (a.bs - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

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

    // gamma of this thread's vectors, once
    uint4 gv[kCbVecs];
#pragma unroll
    for (int j = 0; j < kCbVecs; ++j) {
        const int p = t + j * kCbThreads;
        gv[j] = (j < J && p < V) ? ld_cached(a.gamma + p * 8) : make_uint4(0, 0, 0, 0);
    }

    // Issue one unit (token n, slot j) into ring stage st; always commit a
    // group, empty or not, so the group count stays uniform.
    int in_n = 0, in_j = 0, in_st = 0;
    auto issue_next = [&]() {
        const int p = t + in_j * kCbThreads;
        if (in_n < n_tok && p < V) {
            const int i = blockIdx.x + in_n * gridDim.x;
            uint4 *slot = s_buf + (size_t)in_st * R * kCbThreads + t;
#pragma unroll
            for (int k = 0; k < KMAX; ++k) {
                if (k >= K) break;
                const int row = s_row[in_n][k];
                if (row >= 0) cp_async16(slot + k * kCbThreads, a.expand_x + (size_t)row * H + p * 8);
            }
            cp_async16(slot + K * kCbThreads, a.residual + (size_t)i * H + p * 8);
            if (SHARED) cp_async16(slot + (K + 1) * kCbThreads, a.shared_x + (size_t)i * H + p * 8);
        }
        cp_async_commit();
        if (++in_j == J) {
            in_j = 0;
            ++in_n;
        }
        if (++in_st == DEPTH) in_st = 0;
    };
#pragma unroll
    for (int d = 0; d < DEPTH - 1; ++d) issue_next();

    int st = 0;
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

        uint64_t xs[kCbVecs][4];
        uint64_t ss2 = 0ull;
#pragma unroll
        for (int j = 0; j < kCbVecs; ++j) {
            if (j >= J) break;  // uniform
            issue_next();
            cp_async_wait<DEPTH - 1>();  // this thread's copies of the oldest unit have landed
            const int p = t + j * kCbThreads;
            const uint4 *slot = s_buf + (size_t)st * R * kCbThreads + t;
            if (++st == DEPTH) st = 0;
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
            if (p < V) {
#pragma unroll
                for (int k = 0; k < KMAX; ++k) {
                    if (!live[k]) continue;
                    const uint4 v = slot[k * kCbThreads];
                    acc[0] = f2_fma(w2[k], bf16x2_to_f2(v.x), acc[0]);
                    acc[1] = f2_fma(w2[k], bf16x2_to_f2(v.y), acc[1]);
                    acc[2] = f2_fma(w2[k], bf16x2_to_f2(v.z), acc[2]);
                    acc[3] = f2_fma(w2[k], bf16x2_to_f2(v.w), acc[3]);
                }
                if constexpr (SHARED) {
                    const uint4 v = slot[(K + 1) * kCbThreads];
                    acc[0] = f2_fma(ws2, bf16x2_to_f2(v.x), acc[0]);
                    acc[1] = f2_fma(ws2, bf16x2_to_f2(v.y), acc[1]);
                    acc[2] = f2_fma(ws2, bf16x2_to_f2(v.z), acc[2]);
                    acc[3] = f2_fma(ws2, bf16x2_to_f2(v.w), acc[3]);
                }
                const uint4 r = slot[K * kCbThreads];
                acc[0] = f2_add(acc[0], bf16x2_to_f2(r.x));
                acc[1] = f2_add(acc[1], bf16x2_to_f2(r.y));
                acc[2] = f2_add(acc[2], bf16x2_to_f2(r.z));
                acc[3] = f2_add(acc[3], bf16x2_to_f2(r.w));
#pragma unroll
                for (int h = 0; h < 4; ++h) ss2 = f2_fma(acc[h], acc[h], ss2);
            }
#pragma unroll
            for (int h = 0; h < 4; ++h) xs[j][h] = acc[h];
        }

        // the token is complete: normalize and write
        const float tot = block_sum<kCbThreads / 32>(f2_lo(ss2) + f2_hi(ss2), s_red);
        const float rstd = __frcp_rn(__fsqrt_rn(__fdiv_rn(tot, (float)H) + a.norm_eps));
        if (t == 0 && a.rstd_out) a.rstd_out[i] = rstd;
        const uint64_t r2 = f2_pack(rstd, rstd);
#pragma unroll
        for (int j = 0; j < kCbVecs; ++j) {
            const int p = t + j * kCbThreads;
            if (j >= J || p >= V) continue;
            const uint32_t gw[4] = {gv[j].x, gv[j].y, gv[j].z, gv[j].w};
            uint32_t yo[4], xo[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const uint64_t yv = f2_mul(f2_mul(xs[j][h], r2), bf16x2_to_f2(gw[h]));
                yo[h] = pack_bf16x2(f2_lo(yv), f2_hi(yv));
                xo[h] = pack_bf16x2(f2_lo(xs[j][h]), f2_hi(xs[j][h]));
            }
            st_v4(a.y + (size_t)i * H + p * 8, make_uint4(yo[0], yo[1], yo[2], yo[3]));
            if (a.x_out) st_v4(a.x_out + (size_t)i * H + p * 8, make_uint4(xo[0], xo[1], xo[2], xo[3]));
        }
    }
    cp_async_wait<0>();  // only empty groups can remain; leave nothing in flight
}

}  // namespace moe
