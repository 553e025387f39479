// dispatch.cuh -- quantize the tokens and scatter their K copies into the
// expert-major receive buffer (aclnnMoeDistributeDispatchV2, "计算公式").
//
// The EP AllToAllV is, on one GPU, a permutation of the (token, k) copies
// into rank-major rows; the page requires a deterministic result
// ("确定性计算"), so a copy's row is its position in (instance, token, k)
// order.  Each kernel below is the whole operation in one launch: every
// block rebuilds what it needs of that order from the (at most 8192) copy
// keys -- a warp-aggregated shared-memory histogram plus a scan -- while its
// own row loads are in flight.  Counts decide nothing about order, so the
// result is the same on every run.
//
// dispatch_token_kernel<MODE>   one block per token, no smooth scales: the
//   row is loaded once (16-byte loads kept in registers), quantized once
//   (all K copies are identical) and written K times.
// dispatch_instance_kernel<MODE> smooth scales (modes 2, 3): one block per
//   (instance, slice of its rows).  The instance's smooth row is staged in
//   shared memory by one TMA bulk copy; the block then streams its rows'
//   tokens from L2, one row ahead, so every smooth row is read from memory
//   once instead of once per copy.
//
// Quantization, per mode ("计算公式" cases 1, 3, 4, 5):
//   0  copy the bf16 row;
//   2  xFp32 = x * smooth; dyn = 127 / max|xFp32| over the row;
//      q = rint(xFp32 * dyn) clamped to [-127, 127]; scale = 1 / dyn;
//   3  the same per 128-element tile (reduced with xor-shuffles);
//   4  mxfp8: per 32-element block sharedExp = floor(log2 max|x|) - 8 taken
//      from the exponent bits; q = e4m3_satfinite(x * 2^-sharedExp); scale
//      byte = sharedExp + 127.
// All of it in IEEE binary32 with explicit round-to-nearest intrinsics, so no
// contraction or approximation can move a code.
#pragma once
#include "common.cuh"

namespace moe {

struct DispatchArgs {
    int bs, hidden, top_k, num_instances;
    int tiles;   // ceil(H / 128) (mode 3)
    int splits;  // blocks per instance (instance kernel)
    const uint16_t *x;  // bf16 bits [bs, H]
    const int32_t *ids;  // instance ids [bs, K]
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

constexpr int kDpThreads = 256;
constexpr int kDpWarps = kDpThreads / 32;
constexpr int kKeyBatch = 16;  // copy keys loaded per thread before they are used

// Key of copy j: its instance if it is sent, -1 if masked out, -2 if its id
// is out of range (then it is dropped and reported).
__device__ __forceinline__ int copy_key(const DispatchArgs &a, int j) {
    const int id = __ldg(a.ids + j);  // both loads issue before either is used
    const bool sent = a.mask ? __ldg(a.mask + j) != 0 : true;
    if (!sent) return -1;
    return (id >= 0 && id < a.num_instances) ? id : -2;
}

// ------------------------------------------------------------ quantizers ---

// 16 bf16 of a chunk -> floats (exact).
__device__ __forceinline__ void chunk16(const uint4 (&xv)[2], float (&f)[16]) {
    float a[8], b[8];
    unpack8(xv[0], a);
    unpack8(xv[1], b);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        f[e] = a[e];
        f[8 + e] = b[e];
    }
}

template <int N>
__device__ __forceinline__ float abs_max(const float (&f)[N]) {
    float m = 0.0f;
#pragma unroll
    for (int e = 0; e < N; ++e) m = fmaxf(m, fabsf(f[e]));
    return m;
}

// rint(v * dyn) as the low byte of a float: adding 1.5 * 2^23 leaves
// 1.5 * 2^23 + rint(v * dyn) (IEEE addition rounds half to even, and the
// spacing there is 1), whose low byte is the code in two's complement.  Exact
// while |v * dyn| < 2^22; here |v| <= amax and dyn = RN(127 / amax), so
// |v * dyn| <= 127 (1 + 2^-24) and the code never leaves [-127, 127]: the
// clamp to that range is never active.  Full-rate adds replace the slower
// float-to-int conversion.
__device__ __forceinline__ uint32_t q8_bits(float v, float dyn) {
    return __float_as_uint(__fadd_rn(__fmul_rn(v, dyn), 12582912.0f));
}

// The code when dyn = +inf (amax == 0, or 127 / amax overflows fp32): v * inf
// is +-inf, which saturates to +-127, or NaN (v = 0), which casts to 0.
__device__ __forceinline__ uint32_t q8_inf(float v) { return v > 0.0f ? 0x7fu : (v < 0.0f ? 0x81u : 0u); }

// Four int8 codes per 32-bit word (element 0 in the low byte).
template <int NW>
__device__ __forceinline__ void pack_int8(const float *f, float dyn, uint32_t *w) {
    if (isinf(dyn)) {  // uniform over the segment
#pragma unroll
        for (int q = 0; q < NW; ++q)
            w[q] = q8_inf(f[4 * q]) | (q8_inf(f[4 * q + 1]) << 8) | (q8_inf(f[4 * q + 2]) << 16) |
                   (q8_inf(f[4 * q + 3]) << 24);
        return;
    }
#pragma unroll
    for (int q = 0; q < NW; ++q) {
        const uint32_t lo = __byte_perm(q8_bits(f[4 * q], dyn), q8_bits(f[4 * q + 1], dyn), 0x0040);
        const uint32_t hi = __byte_perm(q8_bits(f[4 * q + 2], dyn), q8_bits(f[4 * q + 3], dyn), 0x0040);
        w[q] = __byte_perm(lo, hi, 0x5410);
    }
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

// e4m3 codes of 16 values, round to nearest even, saturating at +-448.  The
// multiply by the exact power of two 2^-se equals the page's X / 2^se.
__device__ __forceinline__ uint4 e4m3x16(const float (&f)[16], int se) {
    const float inv = __uint_as_float((uint32_t)(127 - se) << 23);  // 2^-se; normal for se in [-127, 119]
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

// --------------------------------------------------------- token kernel ---

constexpr int kTkChunks = 2;  // 16-element chunks per thread: H / 16 <= 512 = 256 * 2

inline size_t token_smem_bytes(int num_instances) { return 3 * (size_t)num_instances * sizeof(int); }

template <int MODE>
__global__ void __launch_bounds__(kDpThreads) dispatch_token_kernel(DispatchArgs a) {
    extern __shared__ __align__(16) int smem_i[];
    const int E = a.num_instances;
    int *hist = smem_i;       // sent copies per instance
    int *pref = hist + E;     // ... among the copies of earlier tokens
    int *off = pref + E;      // exclusive prefix of hist
    __shared__ float s_red[kDpWarps];
    __shared__ int s_warp[32];
    __shared__ int s_key[16], s_row[16];

    const int i = blockIdx.x, t = threadIdx.x, lane = t & 31;
    const int H = a.hidden, nchunk = H >> 4, K = a.top_k, N = a.bs * K, mine = i * K;

    // 1. this token's row: issue the loads first, use them last
    const uint16_t *xrow = a.x + (size_t)i * H;
    uint4 xv[kTkChunks][2];
#pragma unroll
    for (int j = 0; j < kTkChunks; ++j) {
        const int c = t + j * kDpThreads;
        if (c < nchunk) {
            xv[j][0] = ld_stream(xrow + c * 16);
            xv[j][1] = ld_stream(xrow + c * 16 + 8);
        } else {
            xv[j][0] = xv[j][1] = make_uint4(0, 0, 0, 0);
        }
    }

    // 2. histogram of all sent copies and of those of earlier tokens
    for (int q = t; q < 2 * E; q += kDpThreads) smem_i[q] = 0;
    if (t < K) s_key[t] = copy_key(a, mine + t);
    __syncthreads();
    for (int j0 = 0; j0 < N; j0 += kDpThreads * kKeyBatch) {  // uniform trip count
        int key[kKeyBatch];
#pragma unroll
        for (int u = 0; u < kKeyBatch; ++u) {
            const int j = j0 + u * kDpThreads + t;
            key[u] = j < N ? copy_key(a, j) : -1;
        }
#pragma unroll
        for (int u = 0; u < kKeyBatch; ++u) {
            const int j = j0 + u * kDpThreads + t;
            int k = key[u];
            if (k == -2) {
                if (i == 0) raise_error(a.err, kDevBadId);
                k = -1;
            }
            const bool early = j < mine;
            const unsigned peers = __match_any_sync(kFull, k < 0 ? -1 : (k << 1) | (early ? 1 : 0));
            if (k >= 0 && lane == __ffs(peers) - 1) {
                atomicAdd(&hist[k], __popc(peers));
                if (early) atomicAdd(&pref[k], __popc(peers));
            }
        }
    }
    __syncthreads();

    // 3. bucket offsets: 4 consecutive instances per thread (E <= 1024)
    int v[4], sum = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int b = t * 4 + u;
        v[u] = b < E ? hist[b] : 0;
        sum += v[u];
    }
    const int incl = block_inclusive_scan(sum, s_warp);
    const int total = s_warp[kDpWarps - 1];
    int run = incl - sum;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int b = t * 4 + u;
        if (b < E) {
            off[b] = run;
            if (i == 0) {
                a.counts[b] = v[u];
                a.offsets[b] = run;
            }
        }
        run += v[u];
    }
    if (i == 0 && t == 0) a.offsets[E] = total;
    __syncthreads();

    // 4. rows of this token's copies
    if (t < K) {
        const int k = s_key[t];
        int row = -1;
        if (k >= 0) {
            int same = 0;
            for (int u = 0; u < t; ++u) same += (s_key[u] == k);
            row = off[k] + pref[k] + same;
            a.src_of_row[row] = mine + t;
        }
        a.expand_idx[mine + t] = row;
        s_row[t] = row;
    }
    __syncthreads();

    // 5. quantize once, write every copy
    uint4 q[kTkChunks];
    float seg[kTkChunks];
    uint8_t e8[kTkChunks];
    float row_scale = 0.0f;
    if constexpr (MODE == 2) {
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < kTkChunks; ++j) {
            float f[16];
            chunk16(xv[j], f);
            m = fmaxf(m, abs_max(f));
        }
        m = block_max<kDpWarps>(m, s_red);
        const float dyn = __fdiv_rn(127.0f, m);  // +inf when m == 0
        row_scale = __frcp_rn(dyn);              // 1 / dynamicScales (0 when m == 0)
#pragma unroll
        for (int j = 0; j < kTkChunks; ++j) {
            float f[16];
            chunk16(xv[j], f);
            uint32_t w[4];
            pack_int8<4>(f, dyn, w);
            q[j] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    } else if constexpr (MODE == 3) {
#pragma unroll
        for (int j = 0; j < kTkChunks; ++j) {
            float f[16];
            chunk16(xv[j], f);
            float m = abs_max(f);  // the 8 lanes sharing a 128-element tile
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
            const float dyn = __fdiv_rn(127.0f, m);
            seg[j] = __frcp_rn(dyn);
            uint32_t w[4];
            pack_int8<4>(f, dyn, w);
            q[j] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    } else if constexpr (MODE == 4) {
#pragma unroll
        for (int j = 0; j < kTkChunks; ++j) {
            float f[16];
            chunk16(xv[j], f);
            float m = abs_max(f);  // the 2 lanes sharing a 32-element block
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            const int se = mx_shared_exp(m);
            e8[j] = (uint8_t)(se + 127);
            q[j] = e4m3x16(f, se);
        }
    }

    for (int k = 0; k < K; ++k) {
        const int row = s_row[k];
        if (row < 0) continue;
        if constexpr (MODE == 0) {
            uint16_t *dst = reinterpret_cast<uint16_t *>(a.expand_x) + (size_t)row * H;
#pragma unroll
            for (int j = 0; j < kTkChunks; ++j) {
                const int c = t + j * kDpThreads;
                if (c < nchunk) {
                    st_v4(dst + c * 16, xv[j][0]);
                    st_v4(dst + c * 16 + 8, xv[j][1]);
                }
            }
        } else {
            uint8_t *dst = reinterpret_cast<uint8_t *>(a.expand_x) + (size_t)row * H;
#pragma unroll
            for (int j = 0; j < kTkChunks; ++j) {
                const int c = t + j * kDpThreads;
                if (c < nchunk) {
                    st_v4(dst + c * 16, q[j]);
                    if constexpr (MODE == 3) {
                        if ((t & 7) == 0)
                            reinterpret_cast<float *>(a.dyn_scales)[(size_t)row * a.tiles + (c >> 3)] = seg[j];
                    }
                    if constexpr (MODE == 4) {
                        if ((t & 1) == 0)
                            reinterpret_cast<uint8_t *>(a.dyn_scales)[(size_t)row * (H >> 5) + (c >> 1)] = e8[j];
                    }
                }
            }
            if constexpr (MODE == 2) {
                if (t == 0) reinterpret_cast<float *>(a.dyn_scales)[row] = row_scale;
            }
        }
    }
}

// ------------------------------------------------------ instance kernel ---

constexpr int kImVecs = 4;  // 8-element vectors per thread: H / 8 <= 1024 = 256 * 4

// Copies per warp in the instance kernel's key scan (a multiple of 32).
__host__ __device__ inline int im_per_warp(int copies) { return ((copies + kDpWarps - 1) / kDpWarps + 31) & ~31; }

// Dynamic shared memory: the smooth row, then one copy list per warp.
inline size_t instance_smem_bytes(int hidden, int copies) {
    return (size_t)hidden * sizeof(float) + (size_t)kDpWarps * im_per_warp(copies) * sizeof(int);
}

template <int MODE>
__global__ void __launch_bounds__(kDpThreads) dispatch_instance_kernel(DispatchArgs a) {
    extern __shared__ __align__(128) unsigned char smem_b[];
    const int H = a.hidden, K = a.top_k, N = a.bs * K, E = a.num_instances, V = H >> 3;
    float *s_sm = reinterpret_cast<float *>(smem_b);
    int *s_list = reinterpret_cast<int *>(smem_b + (size_t)H * sizeof(float));
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ int s_wcnt[kDpWarps], s_wless[kDpWarps];
    __shared__ float s_red[kDpWarps];

    const int e = blockIdx.x / a.splits, sp = blockIdx.x % a.splits;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;

    // 1. the instance's smooth row -> shared memory, one bulk copy
    if (t == 0) {
        mbar_init(&s_bar, 1);
        mbar_arrive_expect_tx(&s_bar, (uint32_t)H * sizeof(float));
        bulk_copy_g2s(s_sm, a.smooth + (size_t)e * H, (uint32_t)H * sizeof(float), &s_bar);
    }

    // 2. the copies sent to instance e, in (token, k) order: warp w scans the
    //    contiguous range [w * per_warp, (w + 1) * per_warp) of copies
    const int per_warp = im_per_warp(N);
    const unsigned lower = (1u << lane) - 1u;
    int cnt = 0, less = 0;
    for (int b0 = 0; b0 < per_warp; b0 += 32 * kKeyBatch) {  // uniform trip count
        int key[kKeyBatch];
#pragma unroll
        for (int u = 0; u < kKeyBatch; ++u) {
            const int off = b0 + u * 32 + lane;
            const int j = w * per_warp + off;
            key[u] = (off < per_warp && j < N) ? copy_key(a, j) : -1;
        }
#pragma unroll
        for (int u = 0; u < kKeyBatch; ++u) {
            const int off = b0 + u * 32 + lane;
            const int j = w * per_warp + off;
            int k = key[u];
            if (k == -2 && blockIdx.x == 0) raise_error(a.err, kDevBadId);
            if (blockIdx.x == 0 && k < 0 && off < per_warp && j < N) a.expand_idx[j] = -1;  // not sent
            less += (k >= 0 && k < e) ? 1 : 0;
            const unsigned hit = __ballot_sync(kFull, k == e);
            if (k == e) s_list[w * per_warp + cnt + __popc(hit & lower)] = j;
            cnt += __popc(hit);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) less += __shfl_xor_sync(kFull, less, o);
    if (lane == 0) {
        s_wcnt[w] = cnt;
        s_wless[w] = less;
    }
    __syncthreads();
    int wpre[kDpWarps + 1];
    wpre[0] = 0;
    int start = 0;
#pragma unroll
    for (int u = 0; u < kDpWarps; ++u) {
        wpre[u + 1] = wpre[u] + s_wcnt[u];
        start += s_wless[u];
    }
    const int count = wpre[kDpWarps];
    if (sp == 0 && t == 0) {
        a.counts[e] = count;
        a.offsets[e] = start;
        if (e == E - 1) a.offsets[E] = start + count;
    }
    const int r0 = (int)((long long)count * sp / a.splits);
    const int r1 = (int)((long long)count * (sp + 1) / a.splits);
    auto copy_of = [&](int r) {  // r-th copy of the bucket: which warp's list holds it
        int u = 0, base = 0;
#pragma unroll
        for (int q = 1; q < kDpWarps; ++q)
            if (wpre[q] <= r) {
                u = q;
                base = wpre[q];
            }
        return s_list[u * per_warp + (r - base)];
    };
    for (int r = r0 + t; r < r1; r += kDpThreads) {
        const int j = copy_of(r);
        a.src_of_row[start + r] = j;
        a.expand_idx[j] = start + r;
    }

    // 3. wait (bounded) for the smooth row; every thread observes it itself
    if (!__syncthreads_and(mbar_wait_bounded(&s_bar, 0))) {
        if (t == 0) {
            raise_error(a.err, kDevTimeout);
            mbar_wait_bounded(&s_bar, 0);  // a last bounded wait for the copy in flight
        }
        return;
    }

    // 4. the smooth row into registers, then quantize the rows, loading the
    //    next row's token while this one reduces
    float sv[kImVecs][8];
#pragma unroll
    for (int q = 0; q < kImVecs; ++q) {
        const int p = t + q * kDpThreads;
#pragma unroll
        for (int e = 0; e < 8; ++e) sv[q][e] = p < V ? s_sm[p * 8 + e] : 0.0f;
    }
    auto load_row = [&](int r, uint4 (&xv)[kImVecs]) {
        const uint16_t *xr = a.x + (size_t)(copy_of(r) / K) * H;
#pragma unroll
        for (int q = 0; q < kImVecs; ++q) {
            const int p = t + q * kDpThreads;
            xv[q] = p < V ? ld_stream(xr + p * 8) : make_uint4(0, 0, 0, 0);
        }
    };
    uint4 xn[kImVecs];
    if (r0 < r1) load_row(r0, xn);
    for (int r = r0; r < r1; ++r) {  // uniform over the block
        float xf[kImVecs][8];
#pragma unroll
        for (int q = 0; q < kImVecs; ++q) {
            unpack8(xn[q], xf[q]);
#pragma unroll
            for (int e = 0; e < 8; ++e) xf[q][e] = __fmul_rn(xf[q][e], sv[q][e]);  // xFp32 = x * smooth
        }
        if (r + 1 < r1) load_row(r + 1, xn);
        const int row = start + r;
        uint8_t *dst = reinterpret_cast<uint8_t *>(a.expand_x) + (size_t)row * H;
        if constexpr (MODE == 2) {
            float m = 0.0f;
#pragma unroll
            for (int q = 0; q < kImVecs; ++q) m = fmaxf(m, abs_max(xf[q]));
            m = block_max<kDpWarps>(m, s_red);
            const float dyn = __fdiv_rn(127.0f, m);
#pragma unroll
            for (int q = 0; q < kImVecs; ++q) {
                const int p = t + q * kDpThreads;
                if (p < V) {
                    uint32_t wd[2];
                    pack_int8<2>(xf[q], dyn, wd);
                    *reinterpret_cast<uint2 *>(dst + p * 8) = make_uint2(wd[0], wd[1]);
                }
            }
            if (t == 0) reinterpret_cast<float *>(a.dyn_scales)[row] = __frcp_rn(dyn);
        } else {  // MODE 3: a 128-element tile is 16 vectors = 16 consecutive lanes
#pragma unroll
            for (int q = 0; q < kImVecs; ++q) {
                const int p = t + q * kDpThreads;
                float m = abs_max(xf[q]);  // 0 for p >= V
                m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
                m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
                m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
                m = fmaxf(m, __shfl_xor_sync(kFull, m, 8));
                if (p < V) {
                    const float dyn = __fdiv_rn(127.0f, m);
                    uint32_t wd[2];
                    pack_int8<2>(xf[q], dyn, wd);
                    *reinterpret_cast<uint2 *>(dst + p * 8) = make_uint2(wd[0], wd[1]);
                    if ((t & 15) == 0)
                        reinterpret_cast<float *>(a.dyn_scales)[(size_t)row * a.tiles + (p >> 4)] = __frcp_rn(dyn);
                }
            }
        }
    }
}

}  // namespace moe
