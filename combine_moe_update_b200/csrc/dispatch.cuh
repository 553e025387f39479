// dispatch.cuh -- quantize the tokens and scatter their K copies into the
// expert-major receive buffer (aclnnMoeDistributeDispatchV2, "计算公式").
//
// The EP AllToAllV is, on one GPU, a permutation of the (token, k) copies
// into rank-major rows.  The page requires a deterministic result
// ("确定性计算"), so a copy's row is its position in (instance, token, k)
// order: the route kernel computes that order once -- a stable counting sort
// over slices of copies -- and the quantize-and-scatter kernels only look
// their rows up.
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
// dispatch_token_smooth_kernel<MODE>  smooth scales (modes 2, 3): one block
//   per token; the row and the K instance ids are loaded once and each
//   copy's smooth row is loaded one copy ahead, so memory latency overlaps
//   the per-copy reduction and quantization.
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
    int tiles;           // ceil(H / 128) (mode 3)
    uint32_t k_magic;    // div_magic(top_k)
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

// ----------------------------------------------------------- route kernel ---
//
// The copies are cut into G = ceil(N / 512) slices of 512 consecutive copies,
// one block of 512 threads (16 warps, one copy per thread) each.  Every block
// builds, in shared memory, the histogram of all sent copies per instance and
// the histogram of the copies of earlier slices (plain atomic adds: counts do
// not depend on order).  A scan of the first gives the bucket offsets; the
// second gives this slice's start inside each bucket.  Inside the slice,
// __match_any_sync groups the lanes of a warp with equal instances, so a
// copy's rank within its warp is the number of lower lanes with the same
// instance, and a per-instance prefix over the 16 warps extends that to the
// slice.  row = bucket offset + earlier slices + rank in the slice, the same
// on every run.

constexpr int kRtThreads = 512;
constexpr int kRtWarps = kRtThreads / 32;
constexpr int kRtKeys = 16;  // keys per thread for the histograms: N <= 8192 = 512 * 16

__host__ __device__ inline int route_slices(int copies) { return (copies + kRtThreads - 1) / kRtThreads; }

// Dynamic shared memory: per-(instance, warp) uint16 counters, then three
// int arrays over the instances (all copies, earlier slices, offsets).
inline size_t route_smem_bytes(int num_instances) {
    return (size_t)num_instances * kRtWarps * sizeof(uint16_t) + 3 * (size_t)num_instances * sizeof(int);
}

__global__ void __launch_bounds__(kRtThreads) route_kernel(DispatchArgs a) {
    pdl_wait();               // the instance ids may come from the previous kernel
    pdl_launch_dependents();  // the scatter kernel may start its input-only work now
    extern __shared__ __align__(16) unsigned char smem_r[];
    const int E = a.num_instances, N = a.bs * a.top_k, g = blockIdx.x;
    uint16_t *s_cnt = reinterpret_cast<uint16_t *>(smem_r);                                  // [E][16]
    int *s_all = reinterpret_cast<int *>(smem_r + (size_t)E * kRtWarps * sizeof(uint16_t));  // [E]
    int *s_before = s_all + E;                                                              // [E]
    int *s_off = s_before + E;                                                              // [E]
    __shared__ int s_warp[32];
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int mine0 = g * kRtThreads;  // first copy of this slice

    // every copy's key (for the histograms) and this thread's own copy; the
    // loads are unconditional (indices clamped into range) so that all of
    // them are in flight together
    int key[kRtKeys];
    uint8_t sent[kRtKeys];
    const int jm = mine0 + t;
    int k = __ldg(a.ids + min(jm, N - 1));
    bool k_sent = jm < N;
#pragma unroll
    for (int u = 0; u < kRtKeys; ++u) key[u] = __ldg(a.ids + min(u * kRtThreads + t, N - 1));
    if (a.mask) {
        k_sent = k_sent && __ldg(a.mask + min(jm, N - 1)) != 0;
#pragma unroll
        for (int u = 0; u < kRtKeys; ++u) sent[u] = __ldg(a.mask + min(u * kRtThreads + t, N - 1));
    } else {
#pragma unroll
        for (int u = 0; u < kRtKeys; ++u) sent[u] = 1;
    }
#pragma unroll
    for (int u = 0; u < kRtKeys; ++u) {
        const int id = key[u];
        key[u] = (u * kRtThreads + t < N && sent[u] != 0) ? ((id >= 0 && id < E) ? id : -2) : -1;
    }
    k = k_sent ? ((k >= 0 && k < E) ? k : -2) : -1;
    if (k == -2) {
        raise_error(a.err, kDevBadId);
        k = -1;
    }
    uint32_t *cnt32 = reinterpret_cast<uint32_t *>(s_cnt);
    for (int q = t; q < 8 * E; q += kRtThreads) cnt32[q] = 0;  // E * 16 uint16
    for (int q = t; q < 2 * E; q += kRtThreads) s_all[q] = 0;  // s_all and s_before
    __syncthreads();

#pragma unroll
    for (int u = 0; u < kRtKeys; ++u) {
        const int kk = key[u];
        if (kk >= 0) {
            atomicAdd(&s_all[kk], 1);
            if (u * kRtThreads + t < mine0) atomicAdd(&s_before[kk], 1);
        }
    }
    const unsigned peers = __match_any_sync(kFull, k);
    if (k >= 0 && lane == __ffs(peers) - 1) s_cnt[k * kRtWarps + w] = (uint16_t)__popc(peers);
    const int local = __popc(peers & ((1u << lane) - 1u));
    __syncthreads();

    // per-instance exclusive prefix over the 16 warps of this slice
    for (int b = t; b < E; b += kRtThreads) {
        int run = 0;
#pragma unroll
        for (int q = 0; q < kRtWarps; ++q) {
            const int c = s_cnt[b * kRtWarps + q];
            s_cnt[b * kRtWarps + q] = (uint16_t)run;
            run += c;
        }
    }
    // exclusive scan of the instance totals: 2 consecutive instances per thread (E <= 1024)
    int v2[2], sum = 0;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int b = t * 2 + u;
        v2[u] = b < E ? s_all[b] : 0;
        sum += v2[u];
    }
    const int incl = block_inclusive_scan(sum, s_warp);  // its barriers also publish s_cnt
    const int total = s_warp[kRtWarps - 1];
    int run = incl - sum;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int b = t * 2 + u;
        if (b < E) {
            s_off[b] = run;
            if (g == 0) {
                a.counts[b] = v2[u];
                a.offsets[b] = run;
            }
        }
        run += v2[u];
    }
    if (g == 0 && t == 0) a.offsets[E] = total;
    __syncthreads();

    if (jm < N) {
        if (k < 0) {
            a.expand_idx[jm] = -1;
        } else {
            const int row = s_off[k] + s_before[k] + s_cnt[k * kRtWarps + w] + local;
            a.expand_idx[jm] = row;
            a.src_of_row[row] = jm;
        }
    }
}

// ------------------------------------------------------------ quantizers ---

constexpr int kDpThreads = 256;  // the most threads a token block runs
constexpr int kDpWarps = kDpThreads / 32;
constexpr int kDpVecs = 4;  // 8-element vectors per thread: H / 8 <= 1024 = 256 * 4

// Threads of a token block for rows of V 8-element vectors: the fewest whole
// warps that cover the row with kDpVecs vectors each, so that every warp has
// the same number of vectors when 32 * kDpVecs divides V (H = 7168: 224
// threads of 4 vectors, none idle at the per-row barrier).
__host__ __device__ inline int dp_threads(int V) {
    const int per = (V + kDpVecs - 1) / kDpVecs;
    return ((per + 31) / 32) * 32;
}

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
        b[2 * q] = __float_as_uint(f2_lo(r));
        b[2 * q + 1] = __float_as_uint(f2_hi(r));
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

// Codes of this thread's vectors for a multiplier dyn shared by the whole
// block (or warp).  The rare dyn = +inf case is a separate branch over all
// vectors, so the common case runs only int8x8 and never pays for both.
__device__ __forceinline__ void int8_vecs(const uint64_t (&v)[kDpVecs][4], float dyn, uint2 (&qv)[kDpVecs]) {
    if (__builtin_expect(isinf(dyn), 0)) {
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) qv[q] = int8x8_inf(v[q]);
    } else {
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) qv[q] = int8x8(v[q], dyn);
    }
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
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, s_red[w]);
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
        int8_vecs(xf, ds.x, qv);
    } else if constexpr (MODE == 3) {
        float dq[kDpVecs];
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {  // a 128-element tile = 16 vectors = 16 consecutive lanes
            float m = abs_max8(xf[q]);       // 0 past the row's end
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 8));
            const bool lead = (t & 15) == 0 && t + q * (int)blockDim.x < V;
            float dyn = 0.0f;
            if (lead) dyn = __fdiv_rn(127.0f, m);  // one division per tile
            dyn = __shfl_sync(kFull, dyn, (t & 31) & ~15);
            if (lead) seg[q] = __frcp_rn(dyn);
            dq[q] = dyn;
        }
        // per-tile multipliers: the +inf branch is taken by a warp only if
        // one of its tiles has one
        bool any_inf = false;
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) any_inf = any_inf || isinf(dq[q]);
        if (__builtin_expect(__any_sync(kFull, any_inf), 0)) {
#pragma unroll
            for (int q = 0; q < kDpVecs; ++q) qv[q] = isinf(dq[q]) ? int8x8_inf(xf[q]) : int8x8(xf[q], dq[q]);
        } else {
#pragma unroll
            for (int q = 0; q < kDpVecs; ++q) qv[q] = int8x8(xf[q], dq[q]);
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
    const int t = threadIdx.x, H = a.hidden, nt = blockDim.x;
    uint8_t *dst = reinterpret_cast<uint8_t *>(a.expand_x) + (size_t)row * H;
#pragma unroll
    for (int q = 0; q < kDpVecs; ++q) {
        const int p = t + q * nt;
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
    const int i = blockIdx.x, t = threadIdx.x, nt = blockDim.x;
    const int H = a.hidden, V = H >> 3, K = a.top_k;

    // inputs of the call only: safe before the route kernel is done
    const uint16_t *xrow = a.x + (size_t)i * H;
    uint4 xv[kDpVecs];
#pragma unroll
    for (int q = 0; q < kDpVecs; ++q) {
        const int p = t + q * nt;
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
                const int p = t + q * nt;
                if (p < V) st_v4(dst + p * 8, xv[q]);
            }
        } else {
            write_row<MODE>(a, row, V, qv, seg, row_scale);
        }
    }
}

// -------------------------------------------------- token smooth kernel ---
//
// Smooth scales (modes 2, 3), one block per token: the token's row and its K
// instance ids are loaded once; copy k's smooth row is loaded one copy ahead
// (while copy k - 1 reduces and quantizes), so the per-copy memory latency
// overlaps compute.  The block waits for the route only before its first
// row write.

template <int MODE>
__global__ void __launch_bounds__(kDpThreads, 2) dispatch_token_smooth_kernel(DispatchArgs a) {
    __shared__ float s_red[2][kDpWarps];
    __shared__ int s_key[16], s_row[16];
    const int i = blockIdx.x, t = threadIdx.x, nt = blockDim.x, nw = nt >> 5;
    const int H = a.hidden, V = H >> 3, K = a.top_k;

    // inputs of the call only: safe before the route kernel is done
    const uint16_t *xrow = a.x + (size_t)i * H;
    uint4 xv[kDpVecs];
#pragma unroll
    for (int q = 0; q < kDpVecs; ++q) {
        const int p = t + q * nt;
        xv[q] = p < V ? ld_stream(xrow + p * 8) : make_uint4(0, 0, 0, 0);
    }
    if (t < K) s_key[t] = copy_key(a, i * K + t);
    __syncthreads();

    auto load_smooth = [&](int e, float4 (&sv)[kDpVecs][2]) {
        const float *srow = a.smooth + (size_t)e * H;
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {
            const int p = t + q * nt;
            if (p < V) {
                sv[q][0] = __ldg(reinterpret_cast<const float4 *>(srow + p * 8));
                sv[q][1] = __ldg(reinterpret_cast<const float4 *>(srow + p * 8) + 1);
            } else {
                sv[q][0] = sv[q][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
        }
    };
    auto next_sent = [&](int k) {  // first copy >= k that is sent, or K
        while (k < K && s_key[k] < 0) ++k;
        return k;
    };

    float4 sn[kDpVecs][2];
    int k = next_sent(0);
    if (k < K) load_smooth(s_key[k], sn);
    bool waited = false;
    int par = 0;
    while (k < K) {  // uniform over the block
        uint64_t xf[kDpVecs][4];
        float m = 0.0f;
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {
            uint64_t f[4];
            vec_to_f2(xv[q], f);
            xf[q][0] = f2_mul(f[0], f2_pack(sn[q][0].x, sn[q][0].y));  // xFp32 = x * smooth
            xf[q][1] = f2_mul(f[1], f2_pack(sn[q][0].z, sn[q][0].w));
            xf[q][2] = f2_mul(f[2], f2_pack(sn[q][1].x, sn[q][1].y));
            xf[q][3] = f2_mul(f[3], f2_pack(sn[q][1].z, sn[q][1].w));
        }
        const int kn = next_sent(k + 1);
        if (kn < K) load_smooth(s_key[kn], sn);  // the next copy's smooth row, in flight during this one

        uint2 qv[kDpVecs];
        float seg[kDpVecs] = {0.0f, 0.0f, 0.0f, 0.0f};
        float row_scale = 0.0f;
        if constexpr (MODE == 2) {
#pragma unroll
            for (int q = 0; q < kDpVecs; ++q) m = fmaxf(m, abs_max8(xf[q]));
            // one barrier per copy: partials in alternating buffers, every thread
            // finishes the max and the division itself
            m = warp_max(m);
            if ((t & 31) == 0) s_red[par][t >> 5] = m;
            __syncthreads();
            float r = s_red[par][0];
#pragma unroll
            for (int w = 1; w < nw; ++w) r = fmaxf(r, s_red[par][w]);
            par ^= 1;
            const float dyn = __fdiv_rn(127.0f, r);  // +inf when r == 0 or 127 / r overflows
            if (t == 0) row_scale = __frcp_rn(dyn);
            int8_vecs(xf, dyn, qv);
        } else {
            quantize_vecs<MODE>(xf, V, nullptr, nullptr, qv, seg, row_scale);
        }

        if (!waited) {
            pdl_wait();  // the rows come from the route kernel
            if (t < K) s_row[t] = a.expand_idx[i * K + t];
            __syncthreads();
            waited = true;
        }
        write_row<MODE>(a, s_row[k], V, qv, seg, row_scale);
        k = kn;
    }
}

}  // namespace moe
