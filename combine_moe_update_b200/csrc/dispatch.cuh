// dispatch.cuh -- quantize each token and scatter its K copies into the
// expert-major receive buffer (aclnnMoeDistributeDispatchV2, "计算公式").
//
// One block of 128 threads per token.  Thread t owns the 16-element chunks
// c = t, t + 128, ... of the row (H <= 8192 -> at most 4 chunks): it loads
// them once with 16-byte loads and keeps them in registers.  Then, per mode:
//   0  (case 1)  copy: the bf16 row is written to every destination row;
//   2  (case 3)  per-token int8: block-wide max |xFp32| via warp shuffles,
//                dyn = 127 / amax, q = rint(xFp32 * dyn), scale = 1 / dyn;
//   3  (case 4)  the same per 128-element tile: the 8 threads sharing a tile
//                reduce with three xor-shuffles;
//   4  (case 5)  mxfp8: per 32-element block (two threads, one shuffle)
//                sharedExp = floor(log2 amax) - 8, read exactly from the
//                exponent bits; q = e4m3_satfinite(x * 2^-sharedExp); the
//                scale byte is sharedExp + 127 (E8M0).
// Without smooth scales all K copies are identical, so the codes are made
// once -- while the ranking kernel is still running (programmatic dependent
// launch) -- and only the K row writes wait for it.  With per-instance smooth
// scales (modes 2 and 3) every copy is quantized with its own instance's
// smooth row.
//
// All quantization arithmetic is IEEE binary32 with explicit round-to-
// nearest intrinsics, so no contraction or approximation can move a code.
#pragma once
#include "common.cuh"

namespace moe {

struct DispatchArgs {
    int bs, hidden, top_k, tiles;  // tiles = ceil(H / 128) (mode 3)
    const uint16_t *x;             // bf16 bits [bs, H]
    const int32_t *ids;            // instance ids [bs, K]
    const float *smooth;           // [E, H] or null
    void *expand_x;
    void *dyn_scales;
    const int32_t *expand_idx;  // written by rank_kernel
    uint32_t *err;
};

constexpr int kDpThreads = 128;
constexpr int kDpChunks = 4;  // 16-element chunks per thread (H / 16 <= 512)

// xFp32 of one 16-element chunk: bf16 -> f32 (exact), times the smooth row.
__device__ __forceinline__ void chunk_xf(const uint4 (&xv)[2], const float *sm, float (&f)[16]) {
    float a[8], b[8];
    unpack8(xv[0], a);
    unpack8(xv[1], b);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        f[e] = a[e];
        f[8 + e] = b[e];
    }
    if (sm) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 s = __ldg(reinterpret_cast<const float4 *>(sm) + q);
            f[4 * q + 0] = __fmul_rn(f[4 * q + 0], s.x);
            f[4 * q + 1] = __fmul_rn(f[4 * q + 1], s.y);
            f[4 * q + 2] = __fmul_rn(f[4 * q + 2], s.z);
            f[4 * q + 3] = __fmul_rn(f[4 * q + 3], s.w);
        }
    }
}

__device__ __forceinline__ float chunk_amax(const float (&f)[16]) {
    float m = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) m = fmaxf(m, fabsf(f[e]));
    return m;
}

// int8 codes of a chunk: clamp(rint(xf * dyn), -127, 127); all zero when
// the segment's amax is 0 (dyn would be +inf).
__device__ __forceinline__ uint4 chunk_int8(const float (&f)[16], float dyn, bool zero) {
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int v = __float2int_rn(__fmul_rn(f[4 * q + e], dyn));
            v = v > 127 ? 127 : (v < -127 ? -127 : v);
            word |= (uint32_t)(v & 0xff) << (8 * e);
        }
        w[q] = zero ? 0u : word;
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// sharedExp = floor(log2 amax) - 8 (emax of e4m3), clamped to >= -127;
// -127 for an all-zero block.  floor(log2) comes from the exponent field
// (or the leading mantissa bit of a subnormal), never from a log routine.
__device__ __forceinline__ int mx_shared_exp(float amax) {
    if (amax == 0.0f) return -127;
    const uint32_t b = __float_as_uint(amax);
    const int ex = (int)(b >> 23);
    const int fl = ex ? ex - 127 : (31 - __clz(b & 0x7fffffu)) - 149;
    const int se = fl - 8;
    return se < -127 ? -127 : se;
}

// e4m3 codes of a chunk: round to nearest even, saturate to +-448.  The
// multiply by the exact power of two 2^-se equals the page's X / 2^se.
__device__ __forceinline__ uint4 chunk_e4m3(const float (&f)[16], int se) {
    const float inv = __uint_as_float((uint32_t)(127 - se) << 23);  // 2^-se, normal for se in [-127, 119]
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
            make_float2(__fmul_rn(f[4 * q + 0], inv), __fmul_rn(f[4 * q + 1], inv)), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
            make_float2(__fmul_rn(f[4 * q + 2], inv), __fmul_rn(f[4 * q + 3], inv)), __NV_SATFINITE, __NV_E4M3);
        w[q] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Quantized codes of this thread's chunks plus the scales it must write.
struct QuantOut {
    uint4 q[kDpChunks];
    float seg_scale[kDpChunks];  // mode 3: scale of the chunk's tile
    uint8_t e8[kDpChunks];       // mode 4: E8M0 byte of the chunk's block
    float row_scale;             // mode 2
};

template <int MODE>
__device__ __forceinline__ void quantize_row(const uint4 (&xv)[kDpChunks][2], const float *sm_row,
                                             int nchunk, float *s_red, QuantOut &o) {
    const int t = threadIdx.x;
    float amax[kDpChunks];
#pragma unroll
    for (int j = 0; j < kDpChunks; ++j) {
        const int c = t + j * kDpThreads;
        amax[j] = 0.0f;
        if (c < nchunk) {
            float f[16];
            chunk_xf(xv[j], sm_row ? sm_row + c * 16 : nullptr, f);
            amax[j] = chunk_amax(f);
        }
    }
    if constexpr (MODE == 2) {
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < kDpChunks; ++j) m = fmaxf(m, amax[j]);
        m = block_max<kDpThreads / 32>(m, s_red);
        const float dyn = __fdiv_rn(127.0f, m);  // +inf when m == 0
        o.row_scale = __frcp_rn(dyn);           // 1 / dynamicScales (0 when m == 0)
#pragma unroll
        for (int j = 0; j < kDpChunks; ++j) {
            const int c = t + j * kDpThreads;
            if (c < nchunk) {
                float f[16];
                chunk_xf(xv[j], sm_row ? sm_row + c * 16 : nullptr, f);
                o.q[j] = chunk_int8(f, dyn, m == 0.0f);
            }
        }
    } else if constexpr (MODE == 3) {
#pragma unroll
        for (int j = 0; j < kDpChunks; ++j) {
            float m = amax[j];  // the 8 lanes of one 128-element tile
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
            const float dyn = __fdiv_rn(127.0f, m);
            o.seg_scale[j] = __frcp_rn(dyn);
            const int c = t + j * kDpThreads;
            if (c < nchunk) {
                float f[16];
                chunk_xf(xv[j], sm_row ? sm_row + c * 16 : nullptr, f);
                o.q[j] = chunk_int8(f, dyn, m == 0.0f);
            }
        }
    } else if constexpr (MODE == 4) {
#pragma unroll
        for (int j = 0; j < kDpChunks; ++j) {
            float m = amax[j];  // the 2 lanes of one 32-element block
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            const int se = mx_shared_exp(m);
            o.e8[j] = (uint8_t)(se + 127);
            const int c = t + j * kDpThreads;
            if (c < nchunk) {
                float f[16];
                chunk_xf(xv[j], nullptr, f);
                o.q[j] = chunk_e4m3(f, se);
            }
        }
    }
}

template <int MODE>
__device__ __forceinline__ void write_copy(const DispatchArgs &a, int row, int nchunk, const QuantOut &o) {
    const int t = threadIdx.x, H = a.hidden;
    uint8_t *dst = reinterpret_cast<uint8_t *>(a.expand_x) + (size_t)row * H;
#pragma unroll
    for (int j = 0; j < kDpChunks; ++j) {
        const int c = t + j * kDpThreads;
        if (c < nchunk) {
            st_v4(dst + c * 16, o.q[j]);
            if constexpr (MODE == 3) {
                if ((t & 7) == 0) reinterpret_cast<float *>(a.dyn_scales)[(size_t)row * a.tiles + (c >> 3)] = o.seg_scale[j];
            }
            if constexpr (MODE == 4) {
                if ((t & 1) == 0) reinterpret_cast<uint8_t *>(a.dyn_scales)[(size_t)row * (H >> 5) + (c >> 1)] = o.e8[j];
            }
        }
    }
    if constexpr (MODE == 2) {
        if (t == 0) reinterpret_cast<float *>(a.dyn_scales)[row] = o.row_scale;
    }
}

template <int MODE, bool SMOOTH>
__global__ void __launch_bounds__(kDpThreads) dispatch_kernel(DispatchArgs a) {
    __shared__ float s_red[kDpThreads / 32];
    __shared__ int s_rows[16], s_inst[16];
    const int i = blockIdx.x, t = threadIdx.x;
    const int H = a.hidden, nchunk = H >> 4, K = a.top_k;

    // The token's row: inputs of the call, safe to read before pdl_wait().
    const uint16_t *xrow = a.x + (size_t)i * H;
    uint4 xv[kDpChunks][2];
#pragma unroll
    for (int j = 0; j < kDpChunks; ++j) {
        const int c = t + j * kDpThreads;
        if (c < nchunk) {
            xv[j][0] = ld_stream(xrow + c * 16);
            xv[j][1] = ld_stream(xrow + c * 16 + 8);
        } else {
            xv[j][0] = xv[j][1] = make_uint4(0, 0, 0, 0);
        }
    }

    if constexpr (MODE == 0) {
        pdl_wait();  // expand_idx comes from rank_kernel
        if (t < K) s_rows[t] = a.expand_idx[i * K + t];
        __syncthreads();
        for (int k = 0; k < K; ++k) {
            const int row = s_rows[k];
            if (row < 0) continue;
            uint16_t *dst = reinterpret_cast<uint16_t *>(a.expand_x) + (size_t)row * H;
#pragma unroll
            for (int j = 0; j < kDpChunks; ++j) {
                const int c = t + j * kDpThreads;
                if (c < nchunk) {
                    st_v4(dst + c * 16, xv[j][0]);
                    st_v4(dst + c * 16 + 8, xv[j][1]);
                }
            }
        }
    } else if constexpr (!SMOOTH) {
        QuantOut o;
        quantize_row<MODE>(xv, nullptr, nchunk, s_red, o);
        pdl_wait();
        if (t < K) s_rows[t] = a.expand_idx[i * K + t];
        __syncthreads();
        for (int k = 0; k < K; ++k) {
            const int row = s_rows[k];
            if (row >= 0) write_copy<MODE>(a, row, nchunk, o);
        }
    } else {
        pdl_wait();
        if (t < K) {
            s_rows[t] = a.expand_idx[i * K + t];
            s_inst[t] = a.ids[i * K + t];
        }
        __syncthreads();
        for (int k = 0; k < K; ++k) {
            const int row = s_rows[k];  // same value in every thread: the branch is uniform
            if (row < 0) continue;
            QuantOut o;
            quantize_row<MODE>(xv, a.smooth + (size_t)s_inst[k] * H, nchunk, s_red, o);
            write_copy<MODE>(a, row, nchunk, o);
        }
    }
}

}  // namespace moe
