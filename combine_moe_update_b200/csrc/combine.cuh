// combine.cuh -- gather the expert outputs back, weighted top-K sum plus the
// shared-expert term, residual add and RMSNorm, in one pass
// (aclnnMoeDistributeCombineAddRmsNorm, "计算公式"):
//   combineOut = sum_k (s_k * ataOut_k + s_k * sharedExpertX)
//   x = combineOut + residualX
//   y = x / sqrt(mean(x^2) + normEps) * gamma
//
// One block of 256 threads per token.  For each 8-element vector of the row
// a thread issues the K expert-row loads (the AllToAllV back: a gather
// through expand_idx), the shared-expert and the residual load together,
// accumulates in fp32 and parks x in shared memory (so registers stay low
// and several blocks share an SM, keeping enough bytes in flight).  One
// block reduction gives sum(x^2); a second sweep over shared memory writes y
// (and x).  Every input byte is read once and every output byte written once.
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

inline size_t combine_smem_bytes(int hidden) { return (size_t)hidden * sizeof(float); }

// KB: expert rows whose loads are issued together (<= KMAX).
template <int KMAX, int KB, bool SHARED>
__global__ void __launch_bounds__(kCbThreads) combine_kernel(CombineArgs a) {
    extern __shared__ __align__(16) float s_x[];  // x of this token, fp32 [H]
    __shared__ int s_row[16];
    __shared__ float s_w[16];
    __shared__ float s_red[kCbThreads / 32];
    const int i = blockIdx.x, t = threadIdx.x;
    const int H = a.hidden, V = H >> 3, K = a.top_k;

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
    float ss = 0.0f;
#pragma unroll 1
    for (int p = t; p < V; p += kCbThreads) {
        const uint4 res = ld_stream(a.residual + tok + p * 8);
        uint4 sh = make_uint4(0, 0, 0, 0);
        if constexpr (SHARED) sh = ld_stream(a.shared_x + tok + p * 8);
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll
        for (int k0 = 0; k0 < KMAX; k0 += KB) {
            uint4 rv[KB];
#pragma unroll
            for (int k = 0; k < KB; ++k)
                if (row[k0 + k] >= 0) rv[k] = ld_stream(a.expand_x + (size_t)row[k0 + k] * H + p * 8);
#pragma unroll
            for (int k = 0; k < KB; ++k) {
                if (row[k0 + k] < 0) continue;
                float f[8];
                unpack8(rv[k], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(wk[k0 + k], f[e], acc[e]);
            }
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
            acc[e] += r[e];
            ss = fmaf(acc[e], acc[e], ss);
        }
        float4 *xs = reinterpret_cast<float4 *>(s_x + p * 8);
        xs[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        xs[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }

    ss = block_sum<kCbThreads / 32>(ss, s_red);  // its barriers also publish s_x
    const float rstd = __frcp_rn(__fsqrt_rn(__fdiv_rn(ss, (float)H) + a.norm_eps));
    if (t == 0 && a.rstd_out) a.rstd_out[i] = rstd;

#pragma unroll 1
    for (int p = t; p < V; p += kCbThreads) {
        const float4 *xs = reinterpret_cast<const float4 *>(s_x + p * 8);
        const float4 x0 = xs[0], x1 = xs[1];
        const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
        float g[8];
        unpack8(ld_cached(a.gamma + p * 8), g);
        uint4 yo;
        yo.x = pack_bf16x2(x[0] * rstd * g[0], x[1] * rstd * g[1]);
        yo.y = pack_bf16x2(x[2] * rstd * g[2], x[3] * rstd * g[3]);
        yo.z = pack_bf16x2(x[4] * rstd * g[4], x[5] * rstd * g[5]);
        yo.w = pack_bf16x2(x[6] * rstd * g[6], x[7] * rstd * g[7]);
        st_v4(a.y + tok + p * 8, yo);
        if (a.x_out) {
            uint4 xo;
            xo.x = pack_bf16x2(x[0], x[1]);
            xo.y = pack_bf16x2(x[2], x[3]);
            xo.z = pack_bf16x2(x[4], x[5]);
            xo.w = pack_bf16x2(x[6], x[7]);
            st_v4(a.x_out + tok + p * 8, xo);
        }
    }
}

}  // namespace moe
