// common.cuh -- small device helpers shared by the MoE kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

namespace moe {

// Test builds only (-DMOE_FAULT_INJECTION, a separate library the tests load):
// a kernel leaves out one of its bulk copies, so that the bounded wait for it
// runs out with nothing in flight and the timeout path runs.  The shipped
// library never defines it.
#ifdef MOE_FAULT_INJECTION
constexpr bool kSkipOneCopy = true;
#else
constexpr bool kSkipOneCopy = false;
#endif

constexpr uint32_t kDevBadId = 1u;     // id or row index out of range: item dropped
constexpr uint32_t kDevBadTable = 2u;  // mapping table broke its restrictions
constexpr uint32_t kDevTimeout = 4u;   // a bounded wait gave up
constexpr uint32_t kDevCapacity = 8u;  // expert parallelism: a receive buffer too small, rows beyond it dropped
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ void raise_error(uint32_t *err, uint32_t bits) { atomicOr(err, bits); }

// --- one-dimensional TMA bulk copy global -> shared, tracked by an mbarrier ---

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
    // make the initialised barrier visible to the async (TMA) proxy
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// bytes: a multiple of 16; both addresses 16-byte aligned.
__device__ __forceinline__ void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// A waiting thread asks to be suspended until the phase completes, for at
// most this long per poll (ns), instead of spinning on the barrier and
// taking issue slots from the warps that have work.
constexpr uint32_t kWaitHintNs = 1u << 20;  // about a millisecond

// Ask L2 to fetch `bytes` (a multiple of 16, 16-byte aligned) from global
// memory.  Nothing comes back to the program and L2 is the point of
// coherence, so this is safe on data a predecessor kernel may still write:
// its later stores update the lines in L2.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(phase), "r"(kWaitHintNs)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// How long any bounded wait in this library waits before it gives up.
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // one second

// Wait for phase `phase` of an mbarrier, giving up after kWaitLimitNs of
// device time.  Each poll suspends the thread until the phase completes (or
// the hint runs out), so a wait costs a poll or two, not a spin.  Returns
// false on timeout, so a copy that never lands cannot hang the GPU.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t phase) {
    if (mbar_try_wait(bar, phase)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait(bar, phase)) return true;
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
}

// --- thread-block clusters: rank, barrier, and a float from a peer block's
// shared memory (distributed shared memory; plain loads, no multicast) ---
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Every thread of every block of the cluster; orders shared-memory writes
// before it with reads after it, across the cluster.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float ld_cluster_f32(const float *local, uint32_t rank) {
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// Programmatic dependent launch (PTX griddepcontrol, sm_90 and later).  A
// kernel launched with the programmatic-serialization attribute may start
// while its predecessor runs; it must call pdl_wait() before it touches
// anything the predecessor writes.  Without the attribute both are no-ops.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Loads of kernel inputs.  Every kernel is launched as a programmatic
// dependent of the one before it, so its lifetime overlaps its predecessor's
// and any input may still be in flight from that kernel when this one
// starts.  The non-coherent path (ld.global.nc, __ldg) promises data that
// stays constant for the whole kernel and may be scheduled ahead of
// griddepcontrol.wait, so it is never used here: these are ordinary coherent
// loads, which the wait orders after the predecessor's stores.

// 16 bytes, not allocated in L1: for rows that are read once per kernel.
__device__ __forceinline__ uint4 ld_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

// 16 bytes that may stay in L1 (rows reused by a block).
__device__ __forceinline__ uint4 ld_cached(const void *p) { return *reinterpret_cast<const uint4 *>(p); }

// One coherent element load (the plain C++ load, spelled out where a
// read-only cache load would otherwise be the habit).
template <typename T>
__device__ __forceinline__ T ld_in(const T *p) {
    return *p;
}

__device__ __forceinline__ void st_v4(void *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }

// --- packed fp32x2 arithmetic (sm_100): two independent IEEE binary32
// operations, each rounded to nearest even, in one instruction.  A packed
// multiply whose result feeds a packed add is contracted into a fused
// multiply-add by ptxas, even with --fmad=false and explicit .rn rounding
// (measured: codes off by one at rounding ties); where the product's own
// rounding matters, multiply with the scalar __fmul_rn instead, which is
// never contracted. ---

// Pairs are built and split with register-pair moves, which cost no
// instruction once registers are allocated.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}
__device__ __forceinline__ float f2_lo(uint64_t v) {
    float lo;
    asm("{\n\t.reg .f32 hi;\n\tmov.b64 {%0, hi}, %1;\n\t}" : "=f"(lo) : "l"(v));
    return lo;
}
__device__ __forceinline__ float f2_hi(uint64_t v) {
    float hi;
    asm("{\n\t.reg .f32 lo;\n\tmov.b64 {lo, %0}, %1;\n\t}" : "=f"(hi) : "l"(v));
    return hi;
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
// max of three (sm_100a's three-input max; a NaN operand is ignored, as fmaxf ignores it).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// A bf16 pair (one 32-bit word, element 0 in the low half) as an fp32 pair.
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) {
    return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}


// bf16 pair (one 32-bit word, element 0 in the low half) -> two floats, exact.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Eight bf16 in a uint4 -> eight floats.
__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8]) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// Two floats -> bf16 pair, round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half)
    return *reinterpret_cast<uint32_t *>(&h);
}

// Inclusive prefix sum over a block of up to 1024 threads (blockDim.x a
// multiple of 32).  s_warp must hold 32 ints.  Contains two barriers and
// leaves s_warp in use: put a barrier before reusing it.
__device__ __forceinline__ int block_inclusive_scan(int v, int *s_warp) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += y;
    }
    if (lane == 31) s_warp[w] = v;
    __syncthreads();
    if (w == 0) {
        int s = lane < nw ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(kFull, s, o);
            if (lane >= o) s += y;
        }
        s_warp[lane] = s;
    }
    __syncthreads();
    if (w > 0) v += s_warp[w - 1];
    return v;
}

// floor(n / d) for n * (d - 1) < 2^32 and 1 <= d <= 2^16, given
// magic = ceil(2^32 / d) (from div_magic; 0 stands for d = 1, whose magic
// 2^32 does not fit).  Writing magic = (2^32 + r) / d with 0 <= r < d, the
// product n * magic / 2^32 = n / d + n r / (d 2^32); the second term is below
// 1/d while n r < 2^32, so it never carries floor(n / d) past the next
// integer.  (The library divides copy indices < 2^23 by K <= 16 and token
// indices < 2^19 by replica counts <= 768.)
__host__ __device__ inline uint32_t div_magic(uint32_t d) {
    return d <= 1 ? 0u : (uint32_t)((0x100000000ull + d - 1) / d);
}
__device__ __forceinline__ uint32_t div_by_magic(uint32_t n, uint32_t magic) {
    return magic ? __umulhi(n, magic) : n;
}

// Inclusive prefix sum across the 32 lanes of a warp.
__device__ __forceinline__ int warp_inclusive_scan(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(kFull, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

// Max over the 32 lanes of a full warp in one instruction (sm_100a's
// floating-point redux; NaN inputs are ignored, as fmaxf ignores them).
__device__ __forceinline__ float warp_max(float v) {
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
    return v;
}

// Block-wide sum.  s_red holds one float per warp; the warp sums are added
// in a fixed order, so the result is the same on every run.  Two barriers,
// so the buffer can be reused by the next call.
template <int NWARPS>
__device__ __forceinline__ float block_sum(float v, float *s_red) {
    v = warp_sum(v);
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = 0.0f;
#pragma unroll
    for (int w = 0; w < NWARPS; ++w) r += s_red[w];  // fixed order: deterministic
    __syncthreads();
    return r;
}

}  // namespace moe
