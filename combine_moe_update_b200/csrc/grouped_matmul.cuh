// grouped_matmul.cuh -- the deployed instances' int8 matmul that sits between
// the dispatch and the combine, on the fifth-generation tensor cores.
//
// The pages place an expert computation between "AllToAllV(quantOut)" (the
// dispatch page's formula) and the gather of "ataOut" (the combine page's
// formula) without defining it.  Built here as the one contraction that
// consumes the dispatch output: instance e multiplies the rows it received,
// [expert_offsets[e], expert_offsets[e+1]) of expand_x (int8 codes, one
// dequantization factor per row), by its own int8 weight [N, H] (one factor
// per output channel):
//   out[r][n] = (sum_h q[r][h] * w[e][n][h]) * dyn_scale[r] * w_scale[e][n]
// rounded to bf16.  The sum is exact: int8 x int8 products accumulate in
// int32 (|sum| <= 8192 * 128 * 128 < 2^31).
//
// Design (sm_100a):
//  * A planning kernel turns the per-instance offsets into work slots of at
//    most 256 rows of one instance (one thread per instance, a block scan).
//  * The matmul kernel computes one 128-channel x (<= 256 rows) tile per CTA
//    with tcgen05.mma kind::i8, "swapped": the weight slab [128 channels, H]
//    is the MMA's A operand (M = 128) and the slot's rows are B (N = rows
//    rounded up to 16).  A decode batch gives an instance ~16 rows, so N
//    follows the rows and no tensor work is spent on padding to 128 rows;
//    every weight byte is read from HBM once per slot.
//  * Operands are staged by TMA (cp.async.bulk.tensor, 128-byte swizzle, each
//    CTA loading its own tiles) through a ring of stages sized at run time
//    from N, tracked by mbarriers; one lane of one warp issues the copies,
//    one lane of another the MMAs, and tcgen05.commit frees each stage for
//    the next copy.  The int32 accumulator lives in TMEM
//    (128 lanes = channels, N columns = rows; 256 columns allocated, two
//    CTAs per SM).
//  * The epilogue reads TMEM with tcgen05.ld (warp w owns lanes 32w..32w+31),
//    applies the row and channel factors in fp32 and stores bf16.
//  * Every wait is bounded; on a timeout the CTA records MOE_DEV_TIMEOUT,
//    drains its copies in flight (again bounded), frees its TMEM and skips
//    its stores.
//
// On mxfp8 rows (the dispatch's quantMode 4: E4M3 codes with one E8M0 factor
// per 32 elements) the weights are mxfp8 as well, and gmm_mx_kernel runs the
// block-scaled MMA (kind::mxf8f6f4.block_scale, fp32 accumulator) with the
// factors placed in TMEM stage by stage:
//   out[r][n] = sum over 32-element blocks j of
//               2^(sx[r][j] - 127) * 2^(sw[e][n][j] - 127) * sum_{h in j} dec(q[r][h]) * dec(w[e][n][h]).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace moe {

constexpr int kGmBM = 128;          // output channels per tile (the MMA's M)
constexpr int kGmBN = 256;          // rows per slot at most, int8 (the MMA's N: 16..256)
constexpr int kGmBNMx = 128;        // rows per slot at most, mxfp8 (TMEM also holds the factors)
constexpr int kGmBK = 128;          // int8 contraction per stage: one 128-byte swizzled row
constexpr int kGmBoxRows = 16;      // rows per TMA box of the row operand
constexpr int kGmABytes = kGmBM * kGmBK;             // 16 KB of weight per stage
constexpr int kGmPipeBytes = 110 * 1024;             // the stage ring (two CTAs per SM)
constexpr int kGmMaxStages = 8;
constexpr int kGmSmemBytes = kGmPipeBytes + 1024;    // + slack to align the ring to 1 KB
constexpr int kGmThreads = 192;  // warps 0-3 epilogue, warp 4 copies, warp 5 MMAs
constexpr uint32_t kGmTmemCols = 256;                // int32 accumulator columns (>= N)
// mxfp8: the fp32 accumulator (128 columns) then, per ring stage s, the
// stage's block factors: 4 columns for the weight rows (A) at 128 + 8 s and
// 4 for the token rows (B) at 128 + 8 s + 4.
constexpr uint32_t kGmTmemColsMx = 256;

struct GmmArgs {
    int rows, hidden, out_dim, num_instances, max_slots;
    int slot_rows;             // rows per slot at most: kGmBN (int8) or kGmBNMx (mxfp8)
    const float *dyn;          // [rows] per-row factor
    const int32_t *offsets;    // [E + 1]
    const float *wscale;       // [E, N] per-channel factor
    const uint8_t *xsf;        // mxfp8: [rows, H/32] E8M0 block factors of the rows
    const uint8_t *wsf;        // mxfp8: [E, N, H/32] E8M0 block factors of the weights
    uint16_t *out;             // [rows, N] bf16
    int4 *slots;               // [max_slots] {instance, first row, rows, 0}
    int *nslots;
    uint32_t *err;
};

__host__ __device__ inline int gmm_max_slots(int rows, int num_instances, int slot_rows) {
    // sum_e ceil(c_e / R) <= sum_e (c_e + R - 1) / R < rows / R + E
    return num_instances + (rows + slot_rows - 1) / slot_rows;
}

// --- planning: one block of 1024 threads, thread e = instance e ---
__global__ void __launch_bounds__(1024) gmm_plan_kernel(GmmArgs a) {
    __shared__ int s_warp[32];
    __shared__ int s_bad;
    const int e = threadIdx.x;
    if (e == 0) s_bad = 0;
    __syncthreads();
    pdl_wait();  // the offsets come from the dispatch
    int lo = 0, cnt = 0;
    if (e < a.num_instances) {
        lo = a.offsets[e];
        const int hi = a.offsets[e + 1];
        if (lo < 0 || hi < lo || hi > a.rows) s_bad = 1;
        cnt = hi - lo;
    }
    __syncthreads();
    const bool bad = s_bad != 0;
    if (bad) cnt = 0;  // offsets that are not a non-decreasing run in [0, rows]: nothing is computed
    const int R = a.slot_rows;
    const int ch = (cnt + R - 1) / R;
    const int incl = block_inclusive_scan(ch, s_warp);
    for (int c = 0, s = incl - ch; c < ch && s < a.max_slots; ++c, ++s)
        a.slots[s] = make_int4(e, lo + c * R, min(R, cnt - c * R), 0);
    if (e == (int)blockDim.x - 1) *a.nslots = min(incl, a.max_slots);
    if (bad && e == 0) raise_error(a.err, kDevBadId);
    pdl_launch_dependents();
}

// --- tcgen05 / TMA wrappers ---

// Shared-memory matrix descriptor, K-major operand with the 128-byte swizzle:
// rows of 128 bytes, 8-row groups 1024 bytes apart (stride byte offset),
// leading byte offset unused for this layout (encoded 1), descriptor
// version 1, base offset 0 (every tile starts on a 1024-byte boundary).
__device__ __forceinline__ uint64_t gm_smem_desc(uint32_t saddr) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::i8: int32 accumulator, signed A and B, both
// K-major, M = 128, N = n (a multiple of 16, <= 256).
__device__ __forceinline__ uint32_t gm_instr_desc(int n) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kGmBM >> 4) << 24);
}

// Block-scaled instruction descriptor, kind::mxf8f6f4: E4M3 A and B, both
// K-major, E8M0 factors (bit 23), M = 128, N = n (a multiple of 8), and the
// byte (0..3) of the factor columns this MMA reads, for A (bits 29-30) and B
// (bits 4-5).  D is always fp32.
__device__ __forceinline__ uint32_t gm_instr_desc_mx(int n, uint32_t sf_id) {
    return (sf_id << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | (1u << 23) |
           ((uint32_t)(kGmBM >> 4) << 24) | (sf_id << 29);
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void umma_i8(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(acc)
        : "memory");
}

// D[128 x N] (+)= A * diag-scaled B with per-32-block E8M0 factors read from
// TMEM at tsfa / tsfb (the byte the descriptor names).
__device__ __forceinline__ void umma_mx(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t tsfa,
                                        uint32_t tsfb, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(acc), "r"(tsfa), "r"(tsfb)
        : "memory");
}

// 32 lanes (this warp's quarter) x 8 consecutive 32-bit columns:
// col..col+3 from va, col+4..col+7 from vb, with one wait for both.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&va)[4], const uint32_t (&vb)[4]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%2, %3, %4, %5};\n\t"
        "tcgen05.st.sync.aligned.32x32b.x4.b32 [%1], {%6, %7, %8, %9};\n\t"
        "tcgen05.wait::st.sync.aligned;" ::"r"(taddr),
        "r"(taddr + 4u), "r"(va[0]), "r"(va[1]), "r"(va[2]), "r"(va[3]), "r"(vb[0]), "r"(vb[1]), "r"(vb[2]),
        "r"(vb[3])
        : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 2-D tiled TMA load into this CTA's shared memory; x is the innermost coordinate in
// elements (here bytes), always a multiple of 128.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread i of the warp gets lane
// (base lane + i), columns col..col+15.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"  // in the same statement, so no use of v can precede it
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

// Bounded wait with a short sleep between polls, for threads that idle
// through the main loop (kWaitLimitNs of device time at most).
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t *bar, uint32_t phase) {
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, phase)) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
        __nanosleep(64);
    }
}

// --- the int8 matmul, warp-specialized: grid (ceil(N / 128), max_slots), 192 threads ---
//
// int8 rows and weights (kind::i8, int32 accumulator), output
// (acc * dyn[row]) * wscale[channel].  Warp 4 (one lane) issues the TMA
// copies, refilling each stage as soon as the MMAs that read it completed;
// warp 5 (one lane) issues the MMAs and owns the TMEM allocation; warps 0-3
// wait for the accumulator and run the epilogue.  Per ring stage s, full[s]
// (the copies landed) and empty[s] (tcgen05.commit: its MMAs completed) hand
// the stage between the two roles, so neither waits for the other except
// through the stage it needs.
__global__ void __launch_bounds__(kGmThreads, 1)
    gmm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x, GmmArgs a) {
    constexpr uint32_t kCols = kGmTmemCols;
    extern __shared__ uint8_t gm_smem_raw[];
    __shared__ __align__(8) uint64_t s_full[kGmMaxStages];
    __shared__ __align__(8) uint64_t s_empty[kGmMaxStages];
    __shared__ __align__(8) uint64_t s_done;
    __shared__ uint32_t s_tmem;
    __shared__ int4 s_slot;
    __shared__ int s_fail;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    // the ring starts on a 1 KB boundary (the 128-byte swizzle repeats every 1 KB)
    uint8_t *ring = gm_smem_raw + ((1024u - (smem_u32(gm_smem_raw) & 1023u)) & 1023u);

    if (t == 0) {
        for (int s = 0; s < kGmMaxStages; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_empty[s], 1);
        }
        mbar_init(&s_done, 1);
        s_fail = 0;
        tma_prefetch_map(&tm_w);
        tma_prefetch_map(&tm_x);
    }
    pdl_wait();  // slots from the planning kernel; rows and factors from earlier kernels
    if (t == 0) {
        const int ns = *a.nslots;
        s_slot = (int)blockIdx.y < ns ? a.slots[blockIdx.y] : make_int4(-1, 0, 0, 0);
    }
    __syncthreads();
    const int4 slot = s_slot;
    if (slot.x < 0) return;  // more slots were launched than the offsets need

    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(kCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    const int n0 = blockIdx.x * kGmBM;
    const int nr = slot.z;
    const int mma_n = (nr + 15) & ~15;
    const int nbox = mma_n / kGmBoxRows;
    const int stage_bytes = kGmABytes + mma_n * kGmBK;  // a multiple of 2 KB
    const int nst = min(kGmMaxStages, kGmPipeBytes / stage_bytes);
    const int nk = (a.hidden + kGmBK - 1) / kGmBK;

    if (warp == 4) {
        if (lane == 0) {  // the TMA producer
            const uint32_t tx = (uint32_t)stage_bytes;  // out-of-range box parts are zero-filled and still counted
            const int wrow = slot.x * a.out_dim + n0;
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % nst;
                if (kb >= nst && !mbar_wait_bounded(&s_empty[s], (uint32_t)(kb / nst - 1) & 1u)) {
                    s_fail = 1;
                    break;
                }
                uint8_t *sa = ring + s * stage_bytes;
                mbar_arrive_expect_tx(&s_full[s], tx);
                tma_load_2d(sa, &tm_w, kb * kGmBK, wrow, &s_full[s]);
                for (int b = 0; b < nbox; ++b)
                    tma_load_2d(sa + kGmABytes + b * kGmBoxRows * kGmBK, &tm_x, kb * kGmBK, slot.y + b * kGmBoxRows,
                                &s_full[s]);
                ++issued;
            }
            // every copy issued has landed before the CTA can end (at once, unless a wait gave up)
            for (int j = max(0, issued - nst); j < issued; ++j)
                if (!mbar_wait_bounded(&s_full[j % nst], (uint32_t)(j / nst) & 1u)) s_fail = 1;
        }
    } else if (warp == 5) {
        if (lane == 0) {  // the MMA issuer
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % nst;
                if (!mbar_wait_bounded(&s_full[s], (uint32_t)(kb / nst) & 1u)) {
                    s_fail = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_u32(ring + s * stage_bytes);
                const uint64_t da = gm_smem_desc(sa), db = gm_smem_desc(sa + kGmABytes);
#pragma unroll
                for (int kk = 0; kk < kGmBK / 32; ++kk)  // K = 32 per MMA: +32 bytes = +2 in 16-byte units
                    umma_i8(tmem, da + 2 * kk, db + 2 * kk, gm_instr_desc(mma_n), (kb | kk) != 0);
                umma_commit(&s_empty[s]);
            }
            umma_commit(&s_done);  // fires once every MMA above has completed
        }
    }
    __syncwarp();
    const bool done = mbar_wait_sleep(&s_done, 0);
    if (!done && lane == 0) raise_error(a.err, kDevTimeout);
    const bool all_done = __syncthreads_and(done);  // also publishes s_fail
    tc_fence_after();
    pdl_launch_dependents();
    if (s_fail != 0 && t == 0) raise_error(a.err, kDevTimeout);
    if (s_fail == 0 && all_done && warp < 4) {
        const int ch = n0 + warp * 32 + lane;  // this thread's TMEM lane = output channel
        const bool ch_ok = ch < a.out_dim;
        const float wsc = ch_ok ? a.wscale[(size_t)slot.x * a.out_dim + ch] : 0.0f;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        for (int c0 = 0; c0 < mma_n; c0 += 16) {
            uint32_t v[16];
            tmem_ld16(lane_base + (uint32_t)c0, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int r = c0 + j;
                if (r < nr && ch_ok) {
                    const int row = slot.y + r;
                    const float val = __fmul_rn(__fmul_rn(__int2float_rn((int)v[j]), a.dyn[row]), wsc);
                    a.out[(size_t)row * a.out_dim + ch] = __bfloat16_as_ushort(__float2bfloat16_rn(val));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols) : "memory");
}

// --- the mxfp8 matmul, warp-specialized: grid (ceil(N / 128), max_slots), 192 threads ---
//
// Warps 0-3 place each stage's block factors in TMEM (warp w writes lanes
// 32w..32w+31, so the four copies the tensor cores read are all written) and
// later run the epilogue; warp 4 (one lane) issues the TMA copies; warp 5
// (one lane) issues the MMAs.  Per ring stage s three mbarriers hand the
// stage around: full[s] (the copies landed), sf_full[s] (the four factor
// warps wrote the stage's factors) and empty[s] (tcgen05.commit: the MMAs
// that read the stage's operands and factors completed), so no role waits
// for another except through the stage it needs.
//
// VEC: the factor rows are 16-byte aligned (H % 512 == 0 and aligned bases),
// so each thread loads four steps of a row in one 16-byte load.  A warp's
// factor load touches 32 rows, i.e. 32 cache lines; four-byte loads (one
// step each) made the factor warps L1-bound and left the MMA issuer waiting.
constexpr int kGmMxThreads = 192;

template <bool VEC>
__global__ void __launch_bounds__(kGmMxThreads, 1)
    gmm_mx_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x, GmmArgs a) {
    extern __shared__ uint8_t gm_smem_raw[];
    __shared__ __align__(8) uint64_t s_full[kGmMaxStages];
    __shared__ __align__(8) uint64_t s_sf[kGmMaxStages];
    __shared__ __align__(8) uint64_t s_empty[kGmMaxStages];
    __shared__ __align__(8) uint64_t s_done;
    __shared__ uint32_t s_tmem;
    __shared__ int4 s_slot;
    __shared__ int s_fail;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    uint8_t *ring = gm_smem_raw + ((1024u - (smem_u32(gm_smem_raw) & 1023u)) & 1023u);

    if (t == 0) {
        for (int s = 0; s < kGmMaxStages; ++s) {
            mbar_init(&s_full[s], 1);
            mbar_init(&s_sf[s], 4);
            mbar_init(&s_empty[s], 1);
        }
        mbar_init(&s_done, 1);
        s_fail = 0;
        tma_prefetch_map(&tm_w);
        tma_prefetch_map(&tm_x);
    }
    pdl_wait();  // slots from the planning kernel; rows and factors from earlier kernels
    if (t == 0) {
        const int ns = *a.nslots;
        s_slot = (int)blockIdx.y < ns ? a.slots[blockIdx.y] : make_int4(-1, 0, 0, 0);
    }
    __syncthreads();
    const int4 slot = s_slot;
    if (slot.x < 0) return;

    if (warp == 5) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(kGmTmemColsMx)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    const int n0 = blockIdx.x * kGmBM;
    const int nr = slot.z;
    const int mma_n = (nr + 31) & ~31;  // the factor layout wants whole 32-row groups
    const int nbox = mma_n / kGmBoxRows;
    const int stage_bytes = kGmABytes + mma_n * kGmBK;  // a multiple of 2 KB
    const int nst = min(kGmMaxStages, kGmPipeBytes / stage_bytes);
    const int nk = (a.hidden + kGmBK - 1) / kGmBK;

    if (warp == 4) {
        if (lane == 0) {  // the TMA producer
            const uint32_t tx = (uint32_t)stage_bytes;
            const int wrow = slot.x * a.out_dim + n0;
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % nst;
                if (kb >= nst && !mbar_wait_bounded(&s_empty[s], (uint32_t)(kb / nst - 1) & 1u)) {
                    s_fail = 1;
                    break;
                }
                uint8_t *sa = ring + s * stage_bytes;
                mbar_arrive_expect_tx(&s_full[s], tx);
                tma_load_2d(sa, &tm_w, kb * kGmBK, wrow, &s_full[s]);
                for (int b = 0; b < nbox; ++b)
                    tma_load_2d(sa + kGmABytes + b * kGmBoxRows * kGmBK, &tm_x, kb * kGmBK, slot.y + b * kGmBoxRows,
                                &s_full[s]);
                ++issued;
            }
            // every copy issued has landed before the CTA can end (at once, unless a wait gave up)
            for (int j = max(0, issued - nst); j < issued; ++j)
                if (!mbar_wait_bounded(&s_full[j % nst], (uint32_t)(j / nst) & 1u)) s_fail = 1;
        }
    } else if (warp == 5) {
        if (lane == 0) {  // the MMA issuer
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % nst;
                const uint32_t ph = (uint32_t)(kb / nst) & 1u;
                if (!mbar_wait_bounded(&s_full[s], ph) || !mbar_wait_bounded(&s_sf[s], ph)) {
                    s_fail = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = smem_u32(ring + s * stage_bytes);
                const uint64_t da = gm_smem_desc(sa), db = gm_smem_desc(sa + kGmABytes);
                const uint32_t col = tmem + 128u + 8u * (uint32_t)s;
#pragma unroll
                for (int kk = 0; kk < kGmBK / 32; ++kk)
                    umma_mx(tmem, da + 2 * kk, db + 2 * kk, gm_instr_desc_mx(mma_n, (uint32_t)kk),
                            col | ((uint32_t)kk << 30), (col + 4u) | ((uint32_t)kk << 30), (kb | kk) != 0);
                umma_commit(&s_empty[s]);
            }
            umma_commit(&s_done);  // fires once every MMA above has completed
        }
    } else {  // warps 0-3: the block factors of every stage
        const int B = a.hidden >> 5;  // factor bytes per row
        // this thread's factor rows: channel n0 + 32c + lane of the weight, row 32c + lane of the slot
        const uint32_t *pa[4], *pb[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int ch = min(n0 + 32 * c + lane, a.out_dim - 1);
            pa[c] = reinterpret_cast<const uint32_t *>(a.wsf + ((size_t)slot.x * a.out_dim + ch) * B);
            const int r = min(32 * c + lane, nr - 1);
            pb[c] = reinterpret_cast<const uint32_t *>(a.xsf + (size_t)(slot.y + r) * B);
        }
        auto load_sf = [&](int k, uint32_t(&fa)[4], uint32_t(&fb)[4]) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                fa[c] = ld_in(pa[c] + k);
                fb[c] = ld_in(pb[c] + k);
            }
        };
        const uint32_t quarter = (uint32_t)(warp * 32) << 16;
        auto sf_step = [&](int kb, const uint32_t(&fa)[4], const uint32_t(&fb)[4]) -> bool {
            const int s = kb % nst;
            // the slot is free once the MMAs of step kb - nst completed
            bool ok = true;
            if (kb >= nst) {
                if (lane == 0) ok = mbar_wait_bounded(&s_empty[s], (uint32_t)(kb / nst - 1) & 1u);
                ok = __shfl_sync(kFull, ok, 0);
                if (!ok) return false;
            }
            tc_fence_after();
            const uint32_t col = tmem + quarter + 128u + 8u * (uint32_t)s;
            tmem_st8(col, fa, fb);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_sf[s]);
            return true;
        };
        if constexpr (VEC) {
            // four steps per 16-byte load, two groups (eight steps) ahead, in
            // two register sets used in turn
            const uint4 *qa[4], *qb[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                qa[c] = reinterpret_cast<const uint4 *>(pa[c]);
                qb[c] = reinterpret_cast<const uint4 *>(pb[c]);
            }
            const int ng = nk >> 2;  // nk % 4 == 0 here
            uint4 ga[2][4], gb[2][4];
            auto load_group = [&](int g, uint4(&va)[4], uint4(&vb)[4]) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    va[c] = ld_in(qa[c] + g);
                    vb[c] = ld_in(qb[c] + g);
                }
            };
            auto word = [](const uint4 &v, int q) { return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w; };
#pragma unroll
            for (int b = 0; b < 2; ++b)
                if (b < ng) load_group(b, ga[b], gb[b]);
            bool stop = false;
            for (int g0 = 0; g0 < ng && !stop; g0 += 2) {
#pragma unroll
                for (int b = 0; b < 2; ++b) {  // constant register-set index after unrolling
                    const int g = g0 + b;
                    if (g >= ng) break;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t fa[4], fb[4];
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            fa[c] = word(ga[b][c], q);
                            fb[c] = word(gb[b][c], q);
                        }
                        if (!sf_step(4 * g + q, fa, fb)) {
                            if (lane == 0) s_fail = 1;
                            stop = true;
                            break;
                        }
                    }
                    if (stop) break;
                    if (g + 2 < ng) load_group(g + 2, ga[b], gb[b]);
                }
            }
        } else {
            // factor words eight steps ahead (a weight row's 32-byte sector
            // holds eight steps, so one load in eight goes to DRAM), in eight
            // register sets used in turn
            constexpr int kPre = 8;
            uint32_t fa[kPre][4], fb[kPre][4];
#pragma unroll
            for (int q = 0; q < kPre; ++q)
                if (q < nk) load_sf(q, fa[q], fb[q]);
            bool stop = false;
            for (int kb0 = 0; kb0 < nk && !stop; kb0 += kPre) {
#pragma unroll
                for (int q = 0; q < kPre; ++q) {  // constant register-set index after unrolling
                    const int kb = kb0 + q;
                    if (kb >= nk) break;
                    if (!sf_step(kb, fa[q], fb[q])) {
                        if (lane == 0) s_fail = 1;
                        stop = true;
                        break;
                    }
                    if (kb + kPre < nk) load_sf(kb + kPre, fa[q], fb[q]);
                }
            }
        }
    }
    __syncwarp();
    const bool done = mbar_wait_sleep(&s_done, 0);
    if (!done && lane == 0) raise_error(a.err, kDevTimeout);
    const bool all_done = __syncthreads_and(done);  // also publishes s_fail
    tc_fence_after();
    pdl_launch_dependents();
    if (s_fail != 0 && t == 0) raise_error(a.err, kDevTimeout);
    if (s_fail == 0 && all_done && warp < 4) {
        const int ch = n0 + warp * 32 + lane;  // this thread's TMEM lane = output channel
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        for (int c0 = 0; c0 < mma_n; c0 += 16) {
            uint32_t v[16];
            tmem_ld16(lane_base + (uint32_t)c0, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int r = c0 + j;
                if (r < nr && ch < a.out_dim)
                    a.out[(size_t)(slot.y + r) * a.out_dim + ch] =
                        __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 5)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kGmTmemColsMx)
                     : "memory");
}

}  // namespace moe
