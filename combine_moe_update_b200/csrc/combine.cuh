// combine.cuh -- gather the expert outputs back, weighted top-K sum plus the
// shared-expert term, residual add and RMSNorm, in one pass
// (aclnnMoeDistributeCombineAddRmsNorm, "计算公式"):
//   combineOut = sum_k (s_k * ataOut_k + s_k * sharedExpertX)
//   x = combineOut + residualX
//   y = x / sqrt(mean(x^2) + normEps) * gamma
//
// One block of 128 threads per token, small enough that every token of a
// decode batch is resident at once (Bs 512 needs 4 blocks per SM): the whole
// transfer -- K expert rows gathered through expand_idx (the AllToAllV back),
// the shared-expert row and the residual row -- is in flight in a single wave
// instead of trickling through a bounded pipeline.  Thread t owns the
// 8-element vectors p = t, t + 128, ... of the row; it issues all of its
// 16-byte loads first, then accumulates in fp32 and keeps x in registers.
// One block reduction gives sum(x^2); then y (and x) are written.  Every
// input byte is read once and every output byte written once.
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

constexpr int kCbThreads = 128;

// VECS: 8-element vectors per thread (ceil(H / 8 / 128) <= 8).
template <int KMAX, bool SHARED, int VECS>
__global__ void __launch_bounds__(kCbThreads, 4) combine_kernel(CombineArgs a) {
    __shared__ int s_row[16];
    __shared__ float s_w[16];
    __shared__ float s_red[kCbThreads / 32];
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
    float xs[VECS][8];
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < VECS; ++j) {
        const int p = t + j * kCbThreads;
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

    ss = block_sum<kCbThreads / 32>(ss, s_red);
    const float rstd = __frcp_rn(__fsqrt_rn(__fdiv_rn(ss, (float)H) + a.norm_eps));
    if (t == 0 && a.rstd_out) a.rstd_out[i] = rstd;
#pragma unroll
    for (int j = 0; j < VECS; ++j) {
        const int p = t + j * kCbThreads;
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
