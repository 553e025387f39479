// dispatch.cuh -- quantize the tokens and scatter their K copies into the
// expert-major receive buffer (aclnnMoeDistributeDispatchV2, "计算公式").
//
// The EP AllToAllV is, on one GPU, a permutation of the (token, k) copies
// into rank-major rows.  The page requires a deterministic result
// ("确定性计算"), so a copy's row is its position in (instance, token, k)
// order: route_kernel computes that order once -- a stable counting sort in
// one block -- and the quantize-and-scatter kernels only look their rows up.
//
// The scatter kernels are launched as programmatic dependents of the route
// kernel: everything that depends only on the call's inputs (loading the
// token row and the smooth row, the absmax reduction, the quantization
// itself) runs while the route kernel is still sorting, and only the final
// row writes wait for it.
//
// dispatch_token_kernel<MODE>   no smooth scales: one block per token; the
//   row is loaded, quantized once (all K copies are identical) and written K
//   times.
// dispatch_copy_kernel<MODE>    smooth scales (modes 2, 3): one block per
//   (token, k) copy, so 4096 independent blocks at Bs 512, K 8; each loads
//   its token row and its instance's smooth row (both mostly from L2).
//
// Quantization, per mode ("计算公式" cases 1, 3, 4, 5):
//   0  copy the bf16 row;
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
    int tiles;  // ceil(H / 128) (mode 3)
    const uint16_t *x;    // bf16 bits [bs, H]
    const int32_t *ids;   // instance ids [bs, K]
    const uint8_t *mask;  // [bs, K] or null
    const float *smooth;  // [E, H] or null
    void *expand_x;
    void *dyn_scales;
    int32_t *expand_idx;
    int32_t *src_of_row;
    int32_t *counts;
    int32_t *offsets;
    uint32_t *err;
};

// Key of copy j: its instance if it is sent, -1 if masked out, -2 if its id
// is out of range (then it is dropped and reported).
__device__ __forceinline__ int copy_key(const DispatchArgs &a, int j) {
    const int id = __ldg(a.ids + j);  // both loads issue before either is used
    const bool sent = a.mask ? __ldg(a.mask + j) != 0 : true;
    if (!sent) return -1;
    return (id >= 0 && id < a.num_instances) ? id : -2;
}

// ---------------------------------------------------------- route kernel ---
//
// One block of 1024 threads, <= 8192 copies, <= 1024 instances.  Warp w owns
// the contiguous copies [w * P, (w + 1) * P) and walks them 32 at a time;
// __match_any_sync groups equal instances, so a copy's rank inside its warp
// is (earlier rounds' count) + (lower lanes with the same instance).  A
// per-instance prefix over the 32 warps, then a scan over the instances,
// turns those into rows.  No atomics decide an order.

constexpr int kRtThreads = 1024;
constexpr int kRtRounds = 8;  // 8192 copies / 32 warps / 32 lanes

inline size_t route_smem_bytes(int num_instances) {
    return 32 * (size_t)num_instances * sizeof(uint16_t) + (size_t)num_instances * sizeof(int);
}

__global__ void __launch_bounds__(kRtThreads, 1) route_kernel(DispatchArgs a) {
    pdl_wait();               // the instance ids may come from the previous kernel
    pdl_launch_dependents();  // the scatter kernel may start its input-only work now

    extern __shared__ __align__(16) unsigned char smem_r[];
    const int E = a.num_instances, N = a.bs * a.top_k;
    uint16_t *s_wc = reinterpret_cast<uint16_t *>(smem_r);               // [32][E]
    int *s_off = reinterpret_cast<int *>(smem_r + 64 * (size_t)E);      // [E]
    __shared__ int s_warp[32];
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int P = (N + 31) / 32;  // copies per warp
    const int rounds = (P + 31) / 32;

    int key[kRtRounds];
#pragma unroll
    for (int j = 0; j < kRtRounds; ++j) {
        const int off = j * 32 + lane, it = w * P + off;
        key[j] = (j < rounds && off < P && it < N) ? copy_key(a, it) : -1;
    }
    uint32_t *wc32 = reinterpret_cast<uint32_t *>(s_wc);
    for (int q = t; q < 16 * E; q += kRtThreads) wc32[q] = 0;
    __syncthreads();

    const unsigned lower = (1u << lane) - 1u;
    int local[kRtRounds];
#pragma unroll
    for (int j = 0; j < kRtRounds; ++j) {
        local[j] = 0;
        if (j >= rounds) continue;  // uniform
        int k = key[j];
        if (k == -2) {
            raise_error(a.err, kDevBadId);
            k = key[j] = -1;
        }
        const unsigned peers = __match_any_sync(kFull, k);
        int base = 0;
        if (k >= 0) base = s_wc[w * E + k];
        __syncwarp();
        if (k >= 0 && lane == __ffs(peers) - 1) s_wc[w * E + k] = (uint16_t)(base + __popc(peers));
        __syncwarp();
        local[j] = base + __popc(peers & lower);
    }
    __syncthreads();

    int total_b = 0;  // E <= 1024: thread t owns instance t
    if (t < E) {
        int run = 0;
#pragma unroll 8
        for (int ww = 0; ww < 32; ++ww) {
            const int c = s_wc[ww * E + t];
            s_wc[ww * E + t] = (uint16_t)run;
            run += c;
        }
        total_b = run;
    }
    const int incl = block_inclusive_scan(total_b, s_warp);
    if (t < E) {
        s_off[t] = incl - total_b;
        a.counts[t] = total_b;
        a.offsets[t] = incl - total_b;
    }
    if (t == kRtThreads - 1) a.offsets[E] = incl;
    __syncthreads();

#pragma unroll
    for (int j = 0; j < kRtRounds; ++j) {
        const int off = j * 32 + lane, it = w * P + off;
        if (j >= rounds || off >= P || it >= N) continue;
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

// ------------------------------------------------------------ quantizers ---

constexpr int kDpThreads = 256;
constexpr int kDpWarps = kDpThreads / 32;
constexpr int kDpVecs = 4;  // 8-element vectors per thread: H / 8 <= 1024 = 256 * 4

// int8 codes of 8 values (4 fp32 pairs) for a finite multiplier dyn.
// rint(v * dyn) is the low byte of v * dyn + 1.5 * 2^23: IEEE addition
// rounds half to even and the spacing there is 1, so the sum is
// 1.5 * 2^23 + rint(v * dyn), exact while |v * dyn| < 2^22.  Here |v| <=
// amax and dyn = RN(127 / amax), so |v * dyn| <= 127 (1 + 2^-24): codes stay
// in [-127, 127] and the clamp to that range is never active.
//
// The product must be rounded to fp32 on its own before the add (the page's
// quantOut = CastToInt8(xFp32 * dynamicScales) rounds it).  A packed multiply
// followed by a packed add may be contracted into one fused multiply-add,
// which skips that rounding and breaks ties such as a product that rounds to
// exactly 63.5; the scalar round-to-nearest multiply is never contracted.
__device__ __forceinline__ uint2 int8x8(const uint64_t (&v)[4], float dyn) {
    const uint64_t magic = f2_pack(12582912.0f, 12582912.0f);
    uint32_t b[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint64_t prod = f2_pack(__fmul_rn(f2_lo(v[q]), dyn), __fmul_rn(f2_hi(v[q]), dyn));
        const uint64_t r = f2_add(prod, magic);
        b[2 * q] = (uint32_t)r;
        b[2 * q + 1] = (uint32_t)(r >> 32);
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

__device__ __forceinline__ uint2 int8x8_any(const uint64_t (&v)[4], float dyn) {
    return isinf(dyn) ? int8x8_inf(v) : int8x8(v, dyn);
}

__device__ __forceinline__ float abs_max8(const uint64_t (&v)[4]) {
    float m = 0.0f;
#pragma unroll
    for (int q = 0; q < 4; ++q) m = fmaxf(m, fmaxf(fabsf(f2_lo(v[q])), fabsf(f2_hi(v[q]))));
    return m;
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

// Block-wide max of m; thread 0 turns it into dyn = 127 / max and
// scale = 1 / dyn, which every thread reads back.  Two barriers.
__device__ __forceinline__ float2 block_dyn(float m, float *s_red, float *s_out) {
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float r = s_red[0];
#pragma unroll
        for (int w = 1; w < kDpWarps; ++w) r = fmaxf(r, s_red[w]);
        const float dyn = __fdiv_rn(127.0f, r);  // +inf when r == 0 or 127 / r overflows
        s_out[0] = dyn;
        s_out[1] = __frcp_rn(dyn);               // 1 / dynamicScales
    }
    __syncthreads();
    return make_float2(s_out[0], s_out[1]);
}

// Quantize this thread's vectors of one row (xf: fp32 pairs, x * smooth
// already applied).  Fills the codes and the scales this thread writes.
template <int MODE>
__device__ __forceinline__ void quantize_vecs(const uint64_t (&xf)[kDpVecs][4], int V, float *s_red, float *s_out,
                                              uint2 (&qv)[kDpVecs], float (&seg)[kDpVecs], float &row_scale) {
    const int t = threadIdx.x;
    if constexpr (MODE == 2) {
        float m = 0.0f;
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) m = fmaxf(m, abs_max8(xf[q]));
        const float2 ds = block_dyn(m, s_red, s_out);
        row_scale = ds.y;
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) qv[q] = int8x8_any(xf[q], ds.x);
    } else if constexpr (MODE == 3) {
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {  // a 128-element tile = 16 vectors = 16 consecutive lanes
            float m = abs_max8(xf[q]);       // 0 past the row's end
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 8));
            const bool lead = (t & 15) == 0 && t + q * kDpThreads < V;
            float dyn = 0.0f;
            if (lead) dyn = __fdiv_rn(127.0f, m);  // one division per tile
            dyn = __shfl_sync(kFull, dyn, (t & 31) & ~15);
            if (lead) seg[q] = __frcp_rn(dyn);
            qv[q] = int8x8_any(xf[q], dyn);
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
template <int MODE>
__device__ __forceinline__ void write_row(const DispatchArgs &a, int row, int V, const uint2 (&qv)[kDpVecs],
                                          const float (&seg)[kDpVecs], float row_scale) {
    const int t = threadIdx.x, H = a.hidden;
    uint8_t *dst = reinterpret_cast<uint8_t *>(a.expand_x) + (size_t)row * H;
#pragma unroll
    for (int q = 0; q < kDpVecs; ++q) {
        const int p = t + q * kDpThreads;
        if (p >= V) continue;
        *reinterpret_cast<uint2 *>(dst + p * 8) = qv[q];
        if constexpr (MODE == 3) {
            if ((t & 15) == 0) reinterpret_cast<float *>(a.dyn_scales)[(size_t)row * a.tiles + (p >> 4)] = seg[q];
        }
        if constexpr (MODE == 4) {
            if ((t & 3) == 0)
                reinterpret_cast<uint8_t *>(a.dyn_scales)[(size_t)row * (H >> 5) + (p >> 2)] =
                    (uint8_t)__float_as_int(seg[q]);
        }
    }
    if constexpr (MODE == 2) {
        if (t == 0) reinterpret_cast<float *>(a.dyn_scales)[row] = row_scale;
    }
}

// --------------------------------------------------------- token kernel ---

template <int MODE>
__global__ void __launch_bounds__(kDpThreads) dispatch_token_kernel(DispatchArgs a) {
    __shared__ float s_red[kDpWarps], s_out[2];
    __shared__ int s_row[16];
    const int i = blockIdx.x, t = threadIdx.x;
    const int H = a.hidden, V = H >> 3, K = a.top_k;

    // inputs of the call only: safe before the route kernel is done
    const uint16_t *xrow = a.x + (size_t)i * H;
    uint4 xv[kDpVecs];
#pragma unroll
    for (int q = 0; q < kDpVecs; ++q) {
        const int p = t + q * kDpThreads;
        xv[q] = p < V ? ld_stream(xrow + p * 8) : make_uint4(0, 0, 0, 0);
    }
    uint2 qv[kDpVecs];
    float seg[kDpVecs] = {0.0f, 0.0f, 0.0f, 0.0f};
    float row_scale = 0.0f;
    if constexpr (MODE != 0) {
        uint64_t xf[kDpVecs][4];
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) vec_to_f2(xv[q], xf[q]);
        quantize_vecs<MODE>(xf, V, s_red, s_out, qv, seg, row_scale);
    }

    pdl_wait();  // the rows come from route_kernel
    if (t < K) s_row[t] = a.expand_idx[i * K + t];
    __syncthreads();
    for (int k = 0; k < K; ++k) {
        const int row = s_row[k];
        if (row < 0) continue;
        if constexpr (MODE == 0) {
            uint16_t *dst = reinterpret_cast<uint16_t *>(a.expand_x) + (size_t)row * H;
#pragma unroll
            for (int q = 0; q < kDpVecs; ++q) {
                const int p = t + q * kDpThreads;
                if (p < V) st_v4(dst + p * 8, xv[q]);
            }
        } else {
            write_row<MODE>(a, row, V, qv, seg, row_scale);
        }
    }
}

// ---------------------------------------------------------- copy kernel ---

template <int MODE>
__global__ void __launch_bounds__(kDpThreads) dispatch_copy_kernel(DispatchArgs a) {
    __shared__ float s_red[kDpWarps], s_out[2];
    const int c = blockIdx.x, t = threadIdx.x;  // c = i * K + k
    const int H = a.hidden, V = H >> 3, K = a.top_k;

    // inputs of the call only: safe before the route kernel is done
    const int e = copy_key(a, c);
    if (e < 0) return;  // not sent (or a bad id, which route_kernel reports)
    const uint16_t *xrow = a.x + (size_t)(c / K) * H;
    const float *srow = a.smooth + (size_t)e * H;
    uint64_t xf[kDpVecs][4];
#pragma unroll
    for (int q = 0; q < kDpVecs; ++q) {
        const int p = t + q * kDpThreads;
        uint4 xv = make_uint4(0, 0, 0, 0);
        float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
        if (p < V) {
            xv = ld_stream(xrow + p * 8);
            s0 = __ldg(reinterpret_cast<const float4 *>(srow + p * 8));
            s1 = __ldg(reinterpret_cast<const float4 *>(srow + p * 8) + 1);
        }
        uint64_t f[4];
        vec_to_f2(xv, f);
        xf[q][0] = f2_mul(f[0], f2_pack(s0.x, s0.y));  // xFp32 = x * smooth
        xf[q][1] = f2_mul(f[1], f2_pack(s0.z, s0.w));
        xf[q][2] = f2_mul(f[2], f2_pack(s1.x, s1.y));
        xf[q][3] = f2_mul(f[3], f2_pack(s1.z, s1.w));
    }
    uint2 qv[kDpVecs];
    float seg[kDpVecs] = {0.0f, 0.0f, 0.0f, 0.0f};
    float row_scale = 0.0f;
    quantize_vecs<MODE>(xf, V, s_red, s_out, qv, seg, row_scale);

    pdl_wait();  // the row comes from route_kernel
    const int row = a.expand_idx[c];
    if (row >= 0) write_row<MODE>(a, row, V, qv, seg, row_scale);
}

}  // namespace moe
