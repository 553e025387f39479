// combine.cuh -- gather the expert outputs back, weighted top-K sum plus the
// shared-expert term, residual add and RMSNorm, in one pass
// (aclnnMoeDistributeCombineAddRmsNorm, "计算公式"):
//   combineOut = sum_k (s_k * ataOut_k + s_k * sharedExpertX)
//   x = combineOut + residualX
//   y = x / sqrt(mean(x^2) + normEps) * gamma
//
// Each token is handled by one block whose size matches the row (224
// threads at H = 7168, every thread owning four 8-element vectors), small
// enough that every token of a decode batch is resident at once (Bs 512 ->
// 512 blocks, 4 per SM): the whole transfer -- K expert rows gathered
// through expand_idx (the AllToAllV back), the shared-expert row and the
// residual row -- is in flight in a single wave.  A thread issues each
// vector's loads together, accumulates in fp32 and keeps x in registers;
// sum(x^2) is reduced in the block in a fixed order; then y (and x) are
// written.  Every input byte is read once and every output byte written once.
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
    // Expert parallelism across GPUs (EP kernels): expand_idx holds global
    // rows; row g lives on GPU q with gbase[q] <= g < gbase[q + 1], at row
    // g - gbase[q] of peer_rows[q] (peer memory, plain loads).
    const uint16_t *const *peer_rows;
    const int32_t *gbase;  // [G + 1]
    int gpus, recv_rows;
    // TP domain of two ranks (TP2 kernels): the second TP rank's partial
    // expert outputs of the same rows; each gathered row is the bf16 of the
    // sum of the two (the ReduceScatterV).
    const uint16_t *expand_x1;
};

// The most GPUs in an EP group (the header's MOE_EP_MAX_GPUS).
constexpr int kCbMaxGpus = 64;

// K 16 with the norm keeps the pre-norm row in shared memory (XS) and runs
// four blocks per SM; otherwise four blocks up to 224 threads, three beyond.
__host__ __device__ constexpr bool cb_xs(int kmax, bool norm) { return norm && kmax == 16; }
__host__ __device__ constexpr int cb_min_blocks(int kmax, int nt, bool norm) {
    return cb_xs(kmax, norm) || nt <= 224 ? 4 : 3;
}
// Dynamic shared memory of a combine block (the XS row).
__host__ __device__ constexpr int cb_smem_bytes(int kmax, int nt, bool norm, int split) {
    return cb_xs(kmax, norm) ? (split == 1 ? 4 : 2) * nt * 32 : 0;
}

// Threads of a block for NV vectors of 8 elements per block and VECS vectors
// per thread, from the same fixed set of block sizes as the dispatch.
__host__ __device__ inline int cb_threads(int NV, int vecs) {
    const int need = ((NV + vecs - 1) / vecs + 31) / 32 * 32;
    return need <= 64 ? 64 : need <= 128 ? 128 : need <= 192 ? 192 : need <= 224 ? 224 : 256;
}

// One token per block (SPLIT = 1, VECS = 4: 224 threads at H = 7168, four
// blocks per SM, a 512-token batch in one wave), or per cluster of SPLIT = 2
// or 4 blocks (VECS = 2) for smaller batches: block h of the cluster holds
// vectors [h * V / SPLIT, (h + 1) * V / SPLIT) of the row and the blocks'
// sums of x^2 meet through distributed shared memory.  Every thread issues
// the loads of one vector together -- all K rows (a pruned copy issues
// none), the shared row and the residual row -- so a vector costs one round
// trip to memory.  NORM false: the plain combine (combineOut to y; no
// residual, no norm).
// EP: the rows come from the GPUs that own them (expert parallelism across
// GPUs, the AllToAllV back fused into the gather).
// TP2: each gathered row is bf16(expand_x[row] + expand_x1[row]) (the TP
// pair's ReduceScatterV fused into the gather; the fp32 sum of two bf16
// values rounds to the same bf16 as their exact sum).
template <int KMAX, bool SHARED, int NT, bool NORM, int SPLIT, bool EP = false, bool TP2 = false>
__global__ void __launch_bounds__(NT, cb_min_blocks(KMAX, NT, NORM)) combine_token_kernel(CombineArgs a) {
    constexpr int VECS = SPLIT == 1 ? 4 : 2;
    // XS: the pre-norm row waits for the sum of squares in shared memory
    // rather than in registers, which (with the top-K rows loaded eight at a
    // time) lets four blocks of 256 threads share an SM at K 16
    constexpr bool XS = cb_xs(KMAX, NORM);
    extern __shared__ float4 s_x[];  // XS: [VECS][NT][2]
    constexpr int NW = NT / 32;
    __shared__ int s_row[16];
    __shared__ float s_w[16];
    __shared__ const uint16_t *s_src[EP ? 16 : 1];
    // EP: the group's row bases and output buffers, staged once per block so
    // the owner search reads shared memory instead of a chain of dependent
    // global loads
    __shared__ int s_gbase[EP ? kCbMaxGpus + 1 : 1];
    __shared__ const uint16_t *s_peer[EP ? kCbMaxGpus : 1];
    __shared__ int s_nk;
    __shared__ float s_red[NW];
    __shared__ float s_part;
    const int t = threadIdx.x;
    const int i = blockIdx.x / SPLIT, h = SPLIT == 1 ? 0 : (int)cluster_ctarank();
    const int H = a.hidden, V = H >> 3, K = a.top_k, Vh = V / SPLIT, p0 = h * Vh;  // V is even (H % 16 == 0)

    if (t == 0) {  // this block's part of the residual and shared rows, into L2 while the predecessor drains
        const size_t off = (size_t)i * H + (size_t)p0 * 8;
        const uint32_t bytes = (uint32_t)Vh * 16;
        if constexpr (NORM) prefetch_l2(a.residual + off, bytes);
        if constexpr (SHARED) prefetch_l2(a.shared_x + off, bytes);
    }
    pdl_wait();  // expand_idx and the expert rows come from earlier kernels
    int row0 = -1;
    float w0 = 0.0f;
    if (t < K) {  // issued before the EP tables' loads, so they are in flight together
        row0 = a.expand_idx[i * K + t];
        w0 = a.scales[i * K + t];
    }
    if constexpr (EP) {
        for (int q = t; q <= a.gpus; q += NT) {
            s_gbase[q] = a.gbase[q];
            if (q < a.gpus) s_peer[q] = a.peer_rows[q];
        }
        __syncthreads();
    }
    if (t < 32) {  // warp 0: the kept copies, compacted in k order (a pruned copy adds nothing)
        int row = row0;
        const float w = w0;
        const uint16_t *src = nullptr;
        if (t < K) {
            if (row < -1 || row >= a.expand_rows) {
                raise_error(a.err, kDevBadId);
                row = -1;
            }
            if constexpr (EP) {  // the owner of global row `row` (the last GPU whose first row is <= row)
                if (row >= 0) {
                    int lo = 0, hi = a.gpus - 1;
                    while (lo < hi) {
                        const int mid = (lo + hi + 1) >> 1;
                        if (s_gbase[mid] <= row) lo = mid; else hi = mid - 1;
                    }
                    const int prow = row - s_gbase[lo];
                    if (prow >= a.recv_rows || row >= s_gbase[a.gpus]) {
                        raise_error(a.err, kDevBadId);
                        row = -1;
                    } else {
                        src = s_peer[lo] + (size_t)prow * H;
                    }
                }
            }
        }
        const unsigned kept = __ballot_sync(kFull, row >= 0);
        if (row >= 0) {
            const int c = __popc(kept & ((1u << t) - 1u));
            s_row[c] = row;
            s_w[c] = w;
            if constexpr (EP) s_src[c] = src;
        }
        if (t == 0) s_nk = __popc(kept);
    }
    __syncthreads();
    const int nk = s_nk;  // kept copies: rows [0, nk) of s_row
    int row[KMAX];
    float wk[KMAX];
    float wsum = 0.0f;  // sum of the kept weights, in k order
#pragma unroll
    for (int k = 0; k < KMAX; ++k) {
        row[k] = k < nk ? s_row[k] : -1;
        wk[k] = k < nk ? s_w[k] : 0.0f;
        wsum += wk[k];
    }

    const size_t tok = (size_t)i * H;
    float xs[VECS][8];
    float ss = 0.0f;
#pragma unroll
    for (int j = 0; j < VECS; ++j) {
        const int pl = t + j * NT, p = p0 + pl;
#pragma unroll
        for (int e = 0; e < 8; ++e) xs[j][e] = 0.0f;
        if (pl >= Vh) continue;
        uint4 res = make_uint4(0, 0, 0, 0), sh = make_uint4(0, 0, 0, 0);
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
        // all top-K rows in flight at once up to K 8; at K 16 eight at a
        // time (registers: four blocks per SM with XS, no spills without);
        // TP2 loads two rows per copy, four copies at a time
        constexpr int CH = TP2 ? (KMAX < 4 ? KMAX : 4) : (KMAX == 16 ? 8 : KMAX);
#pragma unroll
        for (int k0 = 0; k0 < KMAX; k0 += CH) {
            uint4 rv[CH], rw[TP2 ? CH : 1];
#pragma unroll
            for (int k = 0; k < CH; ++k) {  // nk is the same in every thread: a uniform branch
                if (k0 + k >= nk) break;
                rv[k] = ld_stream((EP ? s_src[k0 + k] : a.expand_x + (size_t)row[k0 + k] * H) + p * 8);
                if constexpr (TP2) rw[k] = ld_stream(a.expand_x1 + (size_t)row[k0 + k] * H + p * 8);
            }
            if (k0 == 0) {
                if constexpr (NORM) res = ld_stream(a.residual + tok + p * 8);
                if constexpr (SHARED) sh = ld_stream(a.shared_x + tok + p * 8);
            }
#pragma unroll
            for (int k = 0; k < CH; ++k) {
                if (k0 + k >= nk) break;
                float f[8];
                unpack8(rv[k], f);
                if constexpr (TP2) {
                    float g2[8];
                    unpack8(rw[k], g2);
#pragma unroll
                    for (int e = 0; e < 8; ++e) f[e] = __bfloat162float(__float2bfloat16_rn(f[e] + g2[e]));
                }
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
            xs[j][e] = acc[e] + r[e];
            ss = fmaf(xs[j][e], xs[j][e], ss);
        }
        if constexpr (!NORM) {  // the plain combine: combineOut, rounded to bf16 once
            uint4 o;
            o.x = pack_bf16x2(xs[j][0], xs[j][1]);
            o.y = pack_bf16x2(xs[j][2], xs[j][3]);
            o.z = pack_bf16x2(xs[j][4], xs[j][5]);
            o.w = pack_bf16x2(xs[j][6], xs[j][7]);
            st_v4(a.y + tok + p * 8, o);
        }
        if constexpr (XS) {
            s_x[(j * NT + t) * 2] = make_float4(xs[j][0], xs[j][1], xs[j][2], xs[j][3]);
            s_x[(j * NT + t) * 2 + 1] = make_float4(xs[j][4], xs[j][5], xs[j][6], xs[j][7]);
        }
    }

    if constexpr (!NORM) {  // the rows are written (no residual, no norm)
        pdl_launch_dependents();
        return;
    }
    float tot = block_sum<NW>(ss, s_red);
    if constexpr (SPLIT > 1) {  // the row's parts: the same sum, in the same order, in every block
        if (t == 0) s_part = tot;
        cluster_sync();
        tot = ld_cluster_f32(&s_part, 0);
#pragma unroll
        for (int q = 1; q < SPLIT; ++q) tot += ld_cluster_f32(&s_part, (uint32_t)q);
        cluster_sync();  // the peers have read this block's partial before any block leaves
    }
    pdl_launch_dependents();
    const float rstd = __frcp_rn(__fsqrt_rn(__fdiv_rn(tot, (float)H) + a.norm_eps));
    if (t == 0 && h == 0 && a.rstd_out) a.rstd_out[i] = rstd;
#pragma unroll
    for (int j = 0; j < VECS; ++j) {
        const int pl = t + j * NT, p = p0 + pl;
        if (pl >= Vh) continue;
        if constexpr (XS) {  // written by this thread
            const float4 u = s_x[(j * NT + t) * 2], v = s_x[(j * NT + t) * 2 + 1];
            xs[j][0] = u.x, xs[j][1] = u.y, xs[j][2] = u.z, xs[j][3] = u.w;
            xs[j][4] = v.x, xs[j][5] = v.y, xs[j][6] = v.z, xs[j][7] = v.w;
        }
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
