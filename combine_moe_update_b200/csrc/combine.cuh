// combine.cuh -- gather the expert outputs back, weighted top-K sum plus the
// shared-expert term, residual add and RMSNorm, in one pass
// (aclnnMoeDistributeCombineAddRmsNorm, "计算公式"):
//   combineOut = sum_k (s_k * ataOut_k + s_k * sharedExpertX)
//   x = combineOut + residualX
//   y = x / sqrt(mean(x^2) + normEps) * gamma
//
// Each token is handled by a cluster of two 128-thread blocks, one per half
// of the row, small enough that every token of a decode batch is resident at
// once (Bs 512 -> 1024 blocks, 7 per SM): the whole transfer -- K expert rows
// gathered through expand_idx (the AllToAllV back), the shared-expert row and
// the residual row -- is in flight in a single wave, and half-token blocks
// spread evenly over the SMs.  Thread t owns 8-element vectors of its half;
// it issues all of its 16-byte loads first, then accumulates in fp32 and
// keeps x in registers.  The two halves' sum(x^2) meet through distributed
// shared memory (added in a fixed order, so both blocks get the same bits);
// then each block writes its half of y (and x).  Every input byte is read
// once and every output byte written once.
#pragma once
#include <cooperative_groups.h>

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

constexpr int kCbThreads = 128;

// VECS: 8-element vectors per thread (ceil(H / 16 / 128) <= 4).
template <int KMAX, bool SHARED, int VECS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kCbThreads, 7) combine_kernel(CombineArgs a) {
    namespace cg = cooperative_groups;
    __shared__ int s_row[16];
    __shared__ float s_w[16];
    __shared__ float s_red[kCbThreads / 32];
    __shared__ float s_part;
    const cg::cluster_group cluster = cg::this_cluster();
    const int half = (int)cluster.block_rank();  // 0: first half of the row, 1: second
    const int i = blockIdx.x >> 1, t = threadIdx.x;
    const int H = a.hidden, V = H >> 3, K = a.top_k;
    const int v0 = half ? (V + 1) / 2 : 0, v1 = half ? V : (V + 1) / 2;  // this block's vectors

    pdl_wait();  // expand_idx and the expert rows come from earlier kernels
    if (t < K) {
        int row = a.expand_idx[i * K + t];
        const float w = a.scales[i * K + t];
        if (row < -1 || row >= a.expand_rows) {
            raise_error(a.err, kDevBadId);
            row = -1;
        }
        s_row[t] = row;
        s_w[t] = row >= 0 ? w : 0.0f;  // a pruned copy weighs nothing
    }
    __syncthreads();
    int row[KMAX];
    float wk[KMAX];
    float wsum = 0.0f;  // sum of the kept weights, in k order
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
        row[k] = k < K ? s_row[k] : -1;
        wk[k] = k < K ? s_w[k] : 0.0f;
        wsum += wk[k];
    }

    const size_t tok = (size_t)i * H;
    float xs[VECS][8];
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < VECS; ++j) {
        const int p = v0 + t + j * kCbThreads;
#pragma unroll
        for (int e = 0; e < 8; ++e) xs[j][e] = 0.0f;
        if (p >= v1) continue;
        uint4 rv[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k)
            if (row[k] >= 0) rv[k] = ld_stream(a.expand_x + (size_t)row[k] * H + p * 8);
        const uint4 res = ld_stream(a.residual + tok + p * 8);
        uint4 sh = make_uint4(0, 0, 0, 0);
        if constexpr (SHARED) sh = ld_stream(a.shared_x + tok + p * 8);
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            if (row[k] < 0) continue;
            float f[8];
            unpack8(rv[k], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(wk[k], f[e], acc[e]);
        }
        if constexpr (SHARED) {
            float f[8];
            unpack8(sh, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(wsum, f[e], acc[e]);
        }
        float r[8];
        unpack8(res, r);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            xs[j][e] = acc[e] + r[e];
            ss = fmaf(xs[j][e], xs[j][e], ss);
        }
    }

    ss = block_sum<kCbThreads / 32>(ss, s_red);
    if (t == 0) s_part = ss;
    cluster.sync();  // both halves' partial sums are in place
    const float other = *cluster.map_shared_rank(&s_part, half ^ 1);
    const float tot = half ? other + ss : ss + other;  // first half + second half, in both blocks
    cluster.sync();  // neither block leaves while the other may still read it
    const float rstd = __frcp_rn(__fsqrt_rn(__fdiv_rn(tot, (float)H) + a.norm_eps));
    if (t == 0 && half == 0 && a.rstd_out) a.rstd_out[i] = rstd;
#pragma unroll
    for (int j = 0; j < VECS; ++j) {
        const int p = v0 + t + j * kCbThreads;
        if (p >= v1) continue;
        float g[8];
        unpack8(ld_cached(a.gamma + p * 8), g);
        uint4 yo;
        yo.x = pack_bf16x2(xs[j][0] * rstd * g[0], xs[j][1] * rstd * g[1]);
        yo.y = pack_bf16x2(xs[j][2] * rstd * g[2], xs[j][3] * rstd * g[3]);
        yo.z = pack_bf16x2(xs[j][4] * rstd * g[4], xs[j][5] * rstd * g[5]);
        yo.w = pack_bf16x2(xs[j][6] * rstd * g[6], xs[j][7] * rstd * g[7]);
        st_v4(a.y + tok + p * 8, yo);
        if (a.x_out) {
            uint4 xo;
            xo.x = pack_bf16x2(xs[j][0], xs[j][1]);
            xo.y = pack_bf16x2(xs[j][2], xs[j][3]);
            xo.z = pack_bf16x2(xs[j][4], xs[j][5]);
            xo.w = pack_bf16x2(xs[j][6], xs[j][7]);
            st_v4(a.x_out + tok + p * 8, xo);
        }
    }
}

// One block of NT threads per token (no cluster): NT is the dispatch token
// block size for the row (224 at H = 7168), so every thread owns exactly
// kCbVecs = 4 vectors when 128 divides H / 8, and four blocks per SM keep a
// 512-token batch resident in one wave.  The reduction of sum(x^2) stays
// inside the block (warp sums added in a fixed order).
constexpr int kCbVecs = 4;

template <int KMAX, bool SHARED, int NT>
__global__ void __launch_bounds__(NT, NT <= 224 ? 4 : 3) combine_token_kernel(CombineArgs a) {
    __shared__ int s_row[16];
    __shared__ float s_w[16];
    __shared__ float s_red[NT / 32];
    const int i = blockIdx.x, t = threadIdx.x;
    const int H = a.hidden, V = H >> 3, K = a.top_k;

    pdl_wait();  // expand_idx and the expert rows come from earlier kernels
    if (t < K) {
        int row = a.expand_idx[i * K + t];
        const float w = a.scales[i * K + t];
        if (row < -1 || row >= a.expand_rows) {
            raise_error(a.err, kDevBadId);
            row = -1;
        }
        s_row[t] = row;
        s_w[t] = row >= 0 ? w : 0.0f;  // a pruned copy weighs nothing
    }
    __syncthreads();
    int row[KMAX];
    float wk[KMAX];
    float wsum = 0.0f;  // sum of the kept weights, in k order
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
        row[k] = k < K ? s_row[k] : -1;
        wk[k] = k < K ? s_w[k] : 0.0f;
        wsum += wk[k];
    }

    const size_t tok = (size_t)i * H;
    float xs[kCbVecs][8];
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < kCbVecs; ++j) {
        const int p = t + j * NT;
#pragma unroll
        for (int e = 0; e < 8; ++e) xs[j][e] = 0.0f;
        if (p >= V) continue;
        uint4 rv[KMAX];
#pragma unroll
        for (int k = 0; k < KMAX; ++k)
            if (row[k] >= 0) rv[k] = ld_stream(a.expand_x + (size_t)row[k] * H + p * 8);
        const uint4 res = ld_stream(a.residual + tok + p * 8);
        uint4 sh = make_uint4(0, 0, 0, 0);
        if constexpr (SHARED) sh = ld_stream(a.shared_x + tok + p * 8);
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll
        for (int k = 0; k < KMAX; ++k) {
            if (row[k] < 0) continue;
            float f[8];
            unpack8(rv[k], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(wk[k], f[e], acc[e]);
        }
        if constexpr (SHARED) {
            float f[8];
            unpack8(sh, f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(wsum, f[e], acc[e]);
        }
        float r[8];
        unpack8(res, r);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            xs[j][e] = acc[e] + r[e];
            ss = fmaf(xs[j][e], xs[j][e], ss);
        }
    }

    const float tot = block_sum<NT / 32>(ss, s_red);
    pdl_launch_dependents();
    const float rstd = __frcp_rn(__fsqrt_rn(__fdiv_rn(tot, (float)H) + a.norm_eps));
    if (t == 0 && a.rstd_out) a.rstd_out[i] = rstd;
#pragma unroll
    for (int j = 0; j < kCbVecs; ++j) {
        const int p = t + j * NT;
        if (p >= V) continue;
        float g[8];
        unpack8(ld_cached(a.gamma + p * 8), g);
        uint4 yo;
        yo.x = pack_bf16x2(xs[j][0] * rstd * g[0], xs[j][1] * rstd * g[1]);
        yo.y = pack_bf16x2(xs[j][2] * rstd * g[2], xs[j][3] * rstd * g[3]);
        yo.z = pack_bf16x2(xs[j][4] * rstd * g[4], xs[j][5] * rstd * g[5]);
        yo.w = pack_bf16x2(xs[j][6] * rstd * g[6], xs[j][7] * rstd * g[7]);
        st_v4(a.y + tok + p * 8, yo);
        if (a.x_out) {
            uint4 xo;
            xo.x = pack_bf16x2(xs[j][0], xs[j][1]);
            xo.y = pack_bf16x2(xs[j][2], xs[j][3]);
            xo.z = pack_bf16x2(xs[j][4], xs[j][5]);
            xo.w = pack_bf16x2(xs[j][6], xs[j][7]);
            st_v4(a.x_out + tok + p * 8, xo);
        }
    }
}

}  // namespace moe
