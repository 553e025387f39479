// dispatch.cuh -- quantize the tokens and scatter their K copies into the
// expert-major receive buffer (aclnnMoeDistributeDispatchV2, "计算公式").
//
// The EP AllToAllV is, on one GPU, a permutation of the (token, k) copies
// into rank-major rows; the page requires a deterministic result
// ("确定性计算"), so a copy's row is its position in (instance, token, k)
// order.  Each kernel below is the whole operation in one launch: every
// block derives what it needs of that order from the (at most 8192) copy
// keys while its own row loads are in flight.  Only counts are accumulated
// concurrently, and counts do not depend on order, so every run gives the
// same bytes.
//
// dispatch_token_kernel<MODE>   one block per token, no smooth scales: the
//   row is loaded once, quantized once (all K copies are identical) and
//   written K times.  A shared-memory histogram of all copies and of the
//   copies of earlier tokens gives the K destination rows.
// dispatch_instance_kernel<MODE> smooth scales (modes 2, 3): one block per
//   (instance, slice of its rows).  The instance's smooth row is staged in
//   shared memory by one TMA bulk copy and then held in registers; the block
//   compacts the copies routed to its instance (ballots over the keys) and
//   streams their tokens' rows from L2, one row ahead, so every smooth row is
//   read from memory once instead of once per copy.
//
// Quantization, per mode ("计算公式" cases 1, 3, 4, 5):
//   0  copy the bf16 row;
//   2  xFp32 = x * smooth; dyn = 127 / max|xFp32| over the row;
//      q = rint(xFp32 * dyn); scale = 1 / dyn;
//   3  the same per 128-element tile;
//   4  mxfp8: per 32-element block sharedExp = floor(log2 max|x|) - 8 taken
//      from the exponent bits; q = e4m3_satfinite(x * 2^-sharedExp); scale
//      byte = sharedExp + 127.
// All arithmetic is IEEE binary32 rounded to nearest (packed fp32x2
// instructions are two such operations each), so no contraction or
// approximation can move a code.
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
constexpr int kDpVecs = 4;     // 8-element vectors per thread: H / 8 <= 1024 = 256 * 4
constexpr int kKeyBatch = 16;  // copy keys a thread loads before using them

// Key of copy j: its instance if it is sent, -1 if masked out, -2 if its id
// is out of range (then it is dropped and reported).
__device__ __forceinline__ int copy_key(const DispatchArgs &a, int j) {
    const int id = __ldg(a.ids + j);  // both loads issue before either is used
    const bool sent = a.mask ? __ldg(a.mask + j) != 0 : true;
    if (!sent) return -1;
    return (id >= 0 && id < a.num_instances) ? id : -2;
}

// ------------------------------------------------------------ quantizers ---

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

// --------------------------------------------------------- token kernel ---

inline size_t token_smem_bytes(int num_instances) { return 3 * (size_t)num_instances * sizeof(int); }

template <int MODE>
__global__ void __launch_bounds__(kDpThreads) dispatch_token_kernel(DispatchArgs a) {
    extern __shared__ __align__(16) int smem_i[];
    const int E = a.num_instances;
    int *hist = smem_i;    // sent copies per instance
    int *pref = hist + E;  // ... among the copies of earlier tokens
    int *off = pref + E;   // exclusive prefix of hist
    __shared__ float s_red[kDpWarps], s_dyn[2];
    __shared__ int s_warp[32];
    __shared__ int s_key[16], s_row[16];

    const int i = blockIdx.x, t = threadIdx.x;
    const int H = a.hidden, V = H >> 3, K = a.top_k, N = a.bs * K, mine = i * K;

    // 1. this token's row: issue the loads first, use them last
    const uint16_t *xrow = a.x + (size_t)i * H;
    uint4 xv[kDpVecs];
#pragma unroll
    for (int q = 0; q < kDpVecs; ++q) {
        const int p = t + q * kDpThreads;
        xv[q] = p < V ? ld_stream(xrow + p * 8) : make_uint4(0, 0, 0, 0);
    }

    // 2. histogram of all sent copies and of those of earlier tokens
    for (int q = t; q < 2 * E; q += kDpThreads) smem_i[q] = 0;
    if (t < K) s_key[t] = copy_key(a, mine + t);
    __syncthreads();
    for (int j0 = 0; j0 < N; j0 += kDpThreads * kKeyBatch) {
        int key[kKeyBatch];
#pragma unroll
        for (int u = 0; u < kKeyBatch; ++u) {
            const int j = j0 + u * kDpThreads + t;
            key[u] = j < N ? copy_key(a, j) : -1;
        }
#pragma unroll
        for (int u = 0; u < kKeyBatch; ++u) {
            const int j = j0 + u * kDpThreads + t;
            const int k = key[u];
            if (k >= 0) {
                atomicAdd(&hist[k], 1);
                if (j < mine) atomicAdd(&pref[k], 1);
            } else if (k == -2 && i == 0) {
                raise_error(a.err, kDevBadId);
            }
        }
    }
    __syncthreads();

    // 3. bucket offsets: 4 consecutive instances per thread (E <= 1024)
    int v4[4], sum = 0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int b = t * 4 + u;
        v4[u] = b < E ? hist[b] : 0;
        sum += v4[u];
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
                a.counts[b] = v4[u];
                a.offsets[b] = run;
            }
        }
        run += v4[u];
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

    // 5. quantize once, then write every copy
    uint2 qv[kDpVecs];
    float seg[kDpVecs];  // mode 3: scale of the slot's tile; mode 4: E8M0 byte of its block (as bits)
    float row_scale = 0.0f;
    if constexpr (MODE == 2) {
        float m = 0.0f;
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {
            uint64_t f[4];
            vec_to_f2(xv[q], f);
            m = fmaxf(m, abs_max8(f));
        }
        const float2 ds = block_dyn(m, s_red, s_dyn);
        row_scale = ds.y;
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {
            uint64_t f[4];
            vec_to_f2(xv[q], f);
            qv[q] = int8x8_any(f, ds.x);
        }
    } else if constexpr (MODE == 3) {
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {  // a 128-element tile = 16 vectors = 16 consecutive lanes
            uint64_t f[4];
            vec_to_f2(xv[q], f);
            float m = abs_max8(f);
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 8));
            const float dyn = __fdiv_rn(127.0f, m);
            seg[q] = __frcp_rn(dyn);
            qv[q] = int8x8_any(f, dyn);
        }
    } else if constexpr (MODE == 4) {
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {  // a 32-element block = 4 consecutive lanes
            uint64_t f[4];
            vec_to_f2(xv[q], f);
            float m = abs_max8(f);
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
            m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
            const int se = mx_shared_exp(m);
            seg[q] = __int_as_float(se + 127);
            qv[q] = e4m3x8(f, se);
        }
    }

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
            uint8_t *dst = reinterpret_cast<uint8_t *>(a.expand_x) + (size_t)row * H;
#pragma unroll
            for (int q = 0; q < kDpVecs; ++q) {
                const int p = t + q * kDpThreads;
                if (p >= V) continue;
                *reinterpret_cast<uint2 *>(dst + p * 8) = qv[q];
                if constexpr (MODE == 3) {
                    if ((t & 15) == 0)
                        reinterpret_cast<float *>(a.dyn_scales)[(size_t)row * a.tiles + (p >> 4)] = seg[q];
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
    }
}

// ------------------------------------------------------ instance kernel ---

constexpr int kImMaxKeys = 32;  // keys per lane in the scan: per warp <= 1024 copies

// Copies per warp in the instance kernel's key scan (a multiple of 32).
__host__ __device__ inline int im_per_warp(int copies) { return ((copies + kDpWarps - 1) / kDpWarps + 31) & ~31; }

// Rows of one instance a block handles at most: ceil(copies / splits).
__host__ __device__ inline int im_row_cap(int copies, int splits) { return (copies + splits - 1) / splits; }

// Dynamic shared memory: the smooth row, then the token of each owned row.
inline size_t instance_smem_bytes(int hidden, int copies, int splits) {
    return (size_t)hidden * sizeof(float) + (size_t)im_row_cap(copies, splits) * sizeof(int);
}

template <int MODE>
__global__ void __launch_bounds__(kDpThreads) dispatch_instance_kernel(DispatchArgs a) {
    extern __shared__ __align__(128) unsigned char smem_b[];
    const int H = a.hidden, K = a.top_k, N = a.bs * K, E = a.num_instances, V = H >> 3;
    float *s_sm = reinterpret_cast<float *>(smem_b);
    int *s_tok = reinterpret_cast<int *>(smem_b + (size_t)H * sizeof(float));  // [cap]
    __shared__ __align__(8) uint64_t s_bar;
    __shared__ int s_wcnt[kDpWarps], s_wless[kDpWarps];
    __shared__ float s_red[kDpWarps], s_dyn[2];

    const int e = blockIdx.x / a.splits, sp = blockIdx.x % a.splits;
    const int t = threadIdx.x, lane = t & 31, w = t >> 5;

    // 1. the instance's smooth row -> shared memory, one bulk copy
    if (t == 0) {
        mbar_init(&s_bar, 1);
        mbar_arrive_expect_tx(&s_bar, (uint32_t)H * sizeof(float));
        bulk_copy_g2s(s_sm, a.smooth + (size_t)e * H, (uint32_t)H * sizeof(float), &s_bar);
    }

    // 2. the copies sent to e, in (token, k) order: warp w scans the contiguous
    //    copies [w * per_warp, (w + 1) * per_warp), 32 per round
    const int per_warp = im_per_warp(N);
    const int rounds = per_warp >> 5;
    const unsigned lower = (1u << lane) - 1u;
    int key[kImMaxKeys];
    int cnt = 0, less = 0;
#pragma unroll
    for (int u = 0; u < kImMaxKeys; ++u) {
        const int j = w * per_warp + u * 32 + lane;
        key[u] = (u < rounds && j < N) ? copy_key(a, j) : -1;
    }
#pragma unroll
    for (int u = 0; u < kImMaxKeys; ++u) {
        if (u >= rounds) break;
        const int k = key[u];
        less += (k >= 0 && k < e) ? 1 : 0;
        cnt += __popc(__ballot_sync(kFull, k == e));
        if (blockIdx.x == 0 && k < 0) {
            const int j = w * per_warp + u * 32 + lane;
            if (j < N) {
                a.expand_idx[j] = -1;  // not sent
                if (k == -2) raise_error(a.err, kDevBadId);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) less += __shfl_xor_sync(kFull, less, o);
    if (lane == 0) {
        s_wcnt[w] = cnt;
        s_wless[w] = less;
    }
    __syncthreads();
    int wbase = 0, count = 0, start = 0;
#pragma unroll
    for (int u = 0; u < kDpWarps; ++u) {
        wbase += (u < w) ? s_wcnt[u] : 0;
        count += s_wcnt[u];
        start += s_wless[u];
    }
    const int r0 = (int)((long long)count * sp / a.splits);
    const int r1 = (int)((long long)count * (sp + 1) / a.splits);
    if (sp == 0 && t == 0) {
        a.counts[e] = count;
        a.offsets[e] = start;
        if (e == E - 1) a.offsets[E] = start + count;
    }
    // second pass over the same keys: place this block's rows
    int pos = wbase;
#pragma unroll
    for (int u = 0; u < kImMaxKeys; ++u) {
        if (u >= rounds) break;
        const int k = key[u];
        const unsigned hit = __ballot_sync(kFull, k == e);
        if (k == e) {
            const int r = pos + __popc(hit & lower);
            if (r >= r0 && r < r1) {
                const int j = w * per_warp + u * 32 + lane;
                s_tok[r - r0] = j / K;
                a.src_of_row[start + r] = j;
                a.expand_idx[j] = start + r;
            }
        }
        pos += __popc(hit);
    }

    // 3. wait (bounded) for the smooth row; every thread observes it itself
    if (!__syncthreads_and(mbar_wait_bounded(&s_bar, 0))) {
        if (t == 0) {
            raise_error(a.err, kDevTimeout);
            mbar_wait_bounded(&s_bar, 0);  // a last bounded wait for the copy in flight
        }
        return;
    }

    // 4. smooth row -> registers (fp32 pairs), then quantize the rows, loading
    //    the next row's token while this one reduces
    uint64_t sv[kDpVecs][4];
#pragma unroll
    for (int q = 0; q < kDpVecs; ++q) {
        const int p = t + q * kDpThreads;
#pragma unroll
        for (int h = 0; h < 4; ++h)
            sv[q][h] = p < V ? *reinterpret_cast<const uint64_t *>(s_sm + p * 8 + 2 * h) : 0ull;
    }
    auto load_row = [&](int r, uint4 (&xv)[kDpVecs]) {
        const uint16_t *xr = a.x + (size_t)s_tok[r - r0] * H;
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {
            const int p = t + q * kDpThreads;
            xv[q] = p < V ? ld_stream(xr + p * 8) : make_uint4(0, 0, 0, 0);
        }
    };
    uint4 xn[kDpVecs];
    if (r0 < r1) load_row(r0, xn);
    for (int r = r0; r < r1; ++r) {  // uniform over the block
        uint64_t xf[kDpVecs][4];
#pragma unroll
        for (int q = 0; q < kDpVecs; ++q) {
            uint64_t f[4];
            vec_to_f2(xn[q], f);
#pragma unroll
            for (int h = 0; h < 4; ++h) xf[q][h] = f2_mul(f[h], sv[q][h]);  // xFp32 = x * smooth
        }
        if (r + 1 < r1) load_row(r + 1, xn);
        const int row = start + r;
        uint8_t *dst = reinterpret_cast<uint8_t *>(a.expand_x) + (size_t)row * H;
        if constexpr (MODE == 2) {
            float m = 0.0f;
#pragma unroll
            for (int q = 0; q < kDpVecs; ++q) m = fmaxf(m, abs_max8(xf[q]));
            const float2 ds = block_dyn(m, s_red, s_dyn);
#pragma unroll
            for (int q = 0; q < kDpVecs; ++q) {
                const int p = t + q * kDpThreads;
                if (p < V) *reinterpret_cast<uint2 *>(dst + p * 8) = int8x8_any(xf[q], ds.x);
            }
            if (t == 0) reinterpret_cast<float *>(a.dyn_scales)[row] = ds.y;
        } else {  // MODE 3: a 128-element tile is 16 vectors = 16 consecutive lanes
#pragma unroll
            for (int q = 0; q < kDpVecs; ++q) {
                const int p = t + q * kDpThreads;
                float m = abs_max8(xf[q]);  // 0 for p >= V
                m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
                m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
                m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
                m = fmaxf(m, __shfl_xor_sync(kFull, m, 8));
                if (p < V) {
                    const float dyn = __fdiv_rn(127.0f, m);
                    *reinterpret_cast<uint2 *>(dst + p * 8) = int8x8_any(xf[q], dyn);
                    if ((t & 15) == 0)
                        reinterpret_cast<float *>(a.dyn_scales)[(size_t)row * a.tiles + (p >> 4)] = __frcp_rn(dyn);
                }
            }
        }
    }
}

}  // namespace moe
