// moe_b200.cu -- the C ABI of include/moe_b200.h: host-side validation,
// workspace sizing and kernel launches.  All compute is in the kernels of
// update_expert.cuh, dispatch.cuh, grouped_matmul.cuh and combine.cuh.
#include "moe_b200.h"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "combine.cuh"
#include "common.cuh"
#include "dispatch.cuh"
#include "ep.cuh"
#include "grouped_matmul.cuh"
#include "update_expert.cuh"

namespace {

// The workspace holds the sticky device error word (4 bytes), padded to 256.
constexpr size_t kWorkspaceBytes = 256;

// Tokens of a call: bs per source rank times the source ranks (0 means 1).
inline int total_tokens(int bs, int sources) { return bs * (sources > 1 ? sources : 1); }

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// Copies up to which the single-pass route runs (it rebuilds the whole
// histogram in every slice); beyond, the three-pass route and its table.
constexpr int kRouteSinglePassMax = moe::kRtThreads * moe::kRtKeys;  // 8192

// The dispatch workspace: the error-word area, then (past 8192 copies) the
// route's slice table.
size_t dispatch_workspace_bytes(const moe_dispatch_params &p) {
    const int copies = total_tokens(p.bs, p.sources) * p.top_k;
    if (copies <= kRouteSinglePassMax) return kWorkspaceBytes;
    return kWorkspaceBytes + (moe::route_large_bytes(copies, p.num_instances) + 15) / 16 * 16;
}

bool check_workspace(const void *ws, size_t bytes) {
    return ws != nullptr && aligned(ws, 16) && bytes >= kWorkspaceBytes;
}

// Allow a kernel its dynamic shared memory (beyond 48 KB needs the opt-in)
// and the largest shared-memory carveout on the current device, once per
// (kernel, device).
bool ensure_smem_fn(const void *fn, size_t bytes) {
    struct Done {
        const void *fn;
        int dev;
        size_t bytes;
    };
    static std::mutex mu;
    static Done done[512];
    static int n_done = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(mu);
    for (int j = 0; j < n_done; ++j)
        if (done[j].fn == fn && done[j].dev == dev && done[j].bytes >= bytes) return true;
    if (bytes > 0 && cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return false;
    // prefer the largest shared-memory carveout, so occupancy is not capped by it
    if (cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess) return false;
    if (n_done < 512) done[n_done++] = Done{fn, dev, bytes};
    return true;
}

template <typename Kernel>
bool ensure_smem(Kernel k, size_t bytes) {
    return ensure_smem_fn(reinterpret_cast<const void *>(k), bytes);
}

// Blocks of a kernel resident on one SM at this block size and dynamic
// shared memory (cached per kernel and device; 1 if the query fails).
int resident_blocks_fn(const void *fn, int threads, size_t smem) {
    struct Seen {
        const void *fn;
        int dev, threads;
        size_t smem;
        int n;
    };
    static std::mutex mu;
    static Seen seen[256];
    static int n_seen = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 1;
    std::lock_guard<std::mutex> lock(mu);
    for (int j = 0; j < n_seen; ++j)
        if (seen[j].fn == fn && seen[j].dev == dev && seen[j].threads == threads && seen[j].smem == smem)
            return seen[j].n;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, fn, threads, smem) != cudaSuccess || n < 1) n = 1;
    if (n_seen < 256) seen[n_seen++] = Seen{fn, dev, threads, smem, n};
    return n;
}

// --- parameter checks: the limits of each page's shape-variable section ---

bool valid_update(const moe_update_params &p) {
    if (p.bs < 1 || p.bs > MOE_MAX_BS) return false;
    if (p.num_logical < 1 || p.num_logical > MOE_MAX_EXPERTS) return false;
    if (p.top_k < 1 || p.top_k > MOE_MAX_TOP_K || p.top_k > p.num_logical) return false;
    if (p.ep_world_size < MOE_MIN_EP_WORLD || p.ep_world_size > MOE_MAX_EP_WORLD) return false;
    if (p.table_cols < 2 || p.table_cols > p.ep_world_size + 1) return false;
    if (!(p.prune_threshold == p.prune_threshold)) return false;  // NaN
    if (p.sources < 0 || p.sources > 2 * p.ep_world_size) return false;  // 2 * ws with a TP domain of two
    return true;
}


moe_status valid_dispatch(const moe_dispatch_params &p) {
    if (p.bs < 1 || p.bs > MOE_MAX_BS) return MOE_ERR_INVALID_ARG;
    if (p.hidden < MOE_MIN_HIDDEN || p.hidden > MOE_MAX_HIDDEN || p.hidden % 16 != 0) return MOE_ERR_INVALID_ARG;
    if (p.num_instances < 1 || p.num_instances > MOE_MAX_EXPERTS) return MOE_ERR_INVALID_ARG;
    if (p.top_k < 1 || p.top_k > MOE_MAX_TOP_K || p.top_k > p.num_instances) return MOE_ERR_INVALID_ARG;
    if (p.ep_world_size < MOE_MIN_EP_WORLD || p.ep_world_size > MOE_MAX_EP_WORLD) return MOE_ERR_INVALID_ARG;
    if (p.num_instances % p.ep_world_size != 0) return MOE_ERR_INVALID_ARG;  // equal instances per rank
    if (p.sources < 0 || p.sources > 2 * p.ep_world_size) return MOE_ERR_INVALID_ARG;  // 2 * ws with TP
    if (p.quant_mode < 0 || p.quant_mode > 4) return MOE_ERR_INVALID_ARG;
    const long long eh = (long long)p.num_instances * p.hidden;
    if (p.quant_mode == 1 && p.scales_len != 1 && p.scales_len != p.hidden && p.scales_len != eh)
        return MOE_ERR_INVALID_ARG;  // static scales: (1,), (H,) or (E, H)
    if ((p.quant_mode == 2 || p.quant_mode == 3) && p.scales_len != 0 && p.scales_len != eh)
        return MOE_ERR_INVALID_ARG;  // smooth scales: (E, H)
    if ((p.quant_mode == 0 || p.quant_mode == 4) && p.scales_len != 0) return MOE_ERR_INVALID_ARG;
    if (p.quant_mode == 4 && p.hidden % 32 != 0) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

bool valid_combine(const moe_combine_params &p) {
    if (p.bs < 1 || p.bs > MOE_MAX_BS) return false;
    if (p.hidden < MOE_MIN_HIDDEN || p.hidden > MOE_MAX_HIDDEN || p.hidden % 16 != 0) return false;
    if (p.top_k < 1 || p.top_k > MOE_MAX_TOP_K) return false;
    if (p.expand_rows < 1) return false;
    if (!(p.norm_eps >= 0.0f) || p.norm_eps > 3.0e38f) return false;  // rejects NaN and inf
    if (p.sources < 0 || p.sources > 2 * MOE_MAX_EP_WORLD) return false;
    return true;
}

bool valid_gmm(const moe_gmm_params &p) {
    if (p.rows < 1 || p.num_instances < 1 || p.num_instances > MOE_MAX_EXPERTS) return false;
    if (moe::gmm_max_slots(p.rows, p.num_instances, moe::kGmBNMx) > 65535) return false;  // slots index grid.y
    if (p.hidden < MOE_MIN_HIDDEN || p.hidden > MOE_MAX_HIDDEN || p.hidden % 16 != 0) return false;
    if (p.out_dim < 16 || p.out_dim > MOE_GMM_MAX_OUT_DIM || p.out_dim % 16 != 0) return false;
    return true;
}

// Grouped-matmul workspace: the error-word area, the slot count (padded to
// 16 bytes), then the slots.
size_t gmm_workspace_bytes(const moe_gmm_params &p) {
    return kWorkspaceBytes + 16 + 16 * (size_t)moe::gmm_max_slots(p.rows, p.num_instances, moe::kGmBNMx);
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A row-major int8 matrix [outer, inner] as a 2-D tensor map with boxes of
// box_outer rows x 128 bytes, 128-byte swizzle, zero fill out of range.
bool encode_i8_rows(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint32_t box_outer) {
    const PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner};
    const cuuint32_t box[2] = {(cuuint32_t)moe::kGmBK, box_outer};
    const cuuint32_t elem[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, elem,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Every kernel is launched as a programmatic dependent of whatever precedes it
// on the stream: its blocks may be scheduled while the previous kernel drains.
// The rule that keeps this safe: the FIRST kernel of every call reads no
// global memory before griddepcontrol.wait, since any of the call's inputs
// may be written by the kernel before it (a combine's y is the next layer's
// x), and that kernel may release its dependents before its last store.  A
// later kernel of the same call may read the call's inputs before its own
// wait only when the call's first kernel releases dependents after its wait
// (route -> scatter inside moe_dispatch): everything before the call has then
// completed.  Outputs of earlier kernels of the call are read after the wait.
// The attribute is harmless when the predecessor is not a kernel.
template <typename... KArgs, typename... Args>
cudaError_t launch_in_clusters(void (*kernel)(KArgs...), dim3 grid, int block, size_t smem, cudaStream_t s,
                               int cluster, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cluster > 1) {  // blocks cluster.. along x share distributed shared memory
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = (unsigned)cluster;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, int block, size_t smem, cudaStream_t s, Args... args) {
    return launch_in_clusters(kernel, grid, block, smem, s, 1, args...);
}

// Streaming multiprocessors of the current device (cached per device).
int device_sms() {
    static std::mutex mu;
    static int sms[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    std::lock_guard<std::mutex> lock(mu);
    if (sms[dev] == 0 && cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return sms[dev];
}

// Token kernels are compiled for a few block sizes (dp_threads); pick the
// one for this row length.
template <int MODE, template <int, int> class Sel>
cudaError_t launch_by_threads(const moe::DispatchArgs &a, cudaStream_t s) {
    switch (moe::dp_threads(a.hidden >> 3)) {
        case 64: return Sel<MODE, 64>::go(a, s);
        case 128: return Sel<MODE, 128>::go(a, s);
        case 192: return Sel<MODE, 192>::go(a, s);
        case 224: return Sel<MODE, 224>::go(a, s);
        default: return Sel<MODE, 256>::go(a, s);
    }
}

// Small calls (at most kFusedRouteMax copies) use the instantiations whose
// blocks route their own copies, and no route kernel runs.
inline bool fused_route(const moe::DispatchArgs &a) {
    return a.bs * a.top_k <= moe::kFusedRouteMax && a.peer_x == nullptr;  // EP: routed by an earlier call
}

template <int MODE, int NT>
struct TokenLaunch {
    template <bool FUSED, bool EP>
    static cudaError_t go_(const moe::DispatchArgs &a, cudaStream_t s) {
        auto kernel = moe::dispatch_token_kernel<MODE, NT, FUSED, EP>;
        if (!ensure_smem(kernel, 0)) return cudaErrorInvalidValue;
        return launch(kernel, a.bs, NT, 0, s, a);
    }
    static cudaError_t go(const moe::DispatchArgs &a, cudaStream_t s) {
        if (a.peer_x != nullptr) return go_<false, true>(a, s);
        return fused_route(a) ? go_<true, false>(a, s) : go_<false, false>(a, s);
    }
};

template <int MODE, int NT>
struct TokenSmoothLaunch {
    template <bool FUSED, bool EP>
    static cudaError_t go_(const moe::DispatchArgs &a, cudaStream_t s) {
        auto kernel = moe::dispatch_token_smooth_kernel<MODE, NT, FUSED, EP>;
        const size_t smem = (size_t)moe::smooth_smem_floats<NT>(a.hidden) * sizeof(float);
        if (!ensure_smem(kernel, smem)) return cudaErrorInvalidValue;
        const int P = copy_groups(a, kernel, smem);
        if (P > 1) {
            auto grouped = moe::dispatch_token_smooth_kernel<MODE, NT, FUSED, EP, true>;
            if (!ensure_smem(grouped, smem)) return cudaErrorInvalidValue;
            return launch(grouped, dim3(a.bs, P), NT, smem, s, a);
        }
        return launch(kernel, a.bs, NT, smem, s, a);
    }
    // Copy groups per token: double them (up to 4, and while a group keeps
    // one copy or more) as long as the batch's blocks still fit on the SMs
    // at once; with static scales (mode 1: no per-copy maximum) up to a
    // second wave.  Measured at H 7168, K 8: mode 2 at Bs 256 two groups
    // 13.2 -> 12.0 us per dispatch call, four 13.4 us; mode 2 at Bs 512 two
    // groups 18.1 -> 19.8 us; mode 1 at Bs 512 two groups 20.4 -> 19.4 us.
    template <typename Kernel>
    static int copy_groups(const moe::DispatchArgs &a, Kernel kernel, size_t smem) {
        const long slots = (long)device_sms() * resident_blocks_fn(reinterpret_cast<const void *>(kernel), NT, smem);
        const long fill = MODE == 1 ? 1 : 2;
        int P = 1;
        while (P < 4 && 2 * P <= a.top_k && (long)a.bs * fill * P <= slots) P *= 2;
        return P;
    }
    static cudaError_t go(const moe::DispatchArgs &a, cudaStream_t s) {
        if (a.peer_x != nullptr) return go_<false, true>(a, s);
        return fused_route(a) ? go_<true, false>(a, s) : go_<false, false>(a, s);
    }
};

template <int MODE>
cudaError_t launch_dispatch_token(const moe::DispatchArgs &a, cudaStream_t s) {
    return launch_by_threads<MODE, TokenLaunch>(a, s);
}

template <int MODE>
cudaError_t launch_dispatch_token_smooth(const moe::DispatchArgs &a, cudaStream_t s) {
    return launch_by_threads<MODE, TokenSmoothLaunch>(a, s);
}

// combine: one block per token (SPLIT 1) or a cluster of two half-row blocks
// per token (SPLIT 2); block size from the row length.
template <int KMAX, bool SHARED, int NT, bool NORM, int SPLIT>
cudaError_t launch_combine_nt(const moe::CombineArgs &a, cudaStream_t s) {
    auto kernel = moe::combine_token_kernel<KMAX, SHARED, NT, NORM, SPLIT>;
    constexpr int smem = moe::cb_smem_bytes(KMAX, NT, NORM, SPLIT);
    if (!ensure_smem(kernel, smem)) return cudaErrorInvalidValue;
    return launch_in_clusters(kernel, a.bs * SPLIT, NT, smem, s, SPLIT, a);
}

template <int KMAX, bool SHARED, bool NORM, int SPLIT>
cudaError_t launch_combine_tok(const moe::CombineArgs &a, cudaStream_t s) {
    constexpr int VECS = SPLIT == 1 ? 4 : 2;
    switch (moe::cb_threads((a.hidden >> 3) / SPLIT, VECS)) {
        case 64: return launch_combine_nt<KMAX, SHARED, 64, NORM, SPLIT>(a, s);
        case 128: return launch_combine_nt<KMAX, SHARED, 128, NORM, SPLIT>(a, s);
        case 192: return launch_combine_nt<KMAX, SHARED, 192, NORM, SPLIT>(a, s);
        case 224: return launch_combine_nt<KMAX, SHARED, 224, NORM, SPLIT>(a, s);
        default: return launch_combine_nt<KMAX, SHARED, 256, NORM, SPLIT>(a, s);
    }
}

// Quarter-row blocks per token when the batch has fewer tokens than SMs,
// half-row blocks when it has fewer than two per SM: measured at Bs 128,
// H 2048 (the 32-layer stack: 10.97 against 10.24 us per layer with
// quarters) and at Bs 256, H 7168 (halves 10.9 against 11.6 us unsplit and
// 13.3 us in quarters), while every batch of 512 tokens ran fastest with
// one block per token (the gate shape 16.6 against 18.8 us, H 4096 10.2
// against 12.9 us, H 8192 23.5 against 24.1 us).
template <int KMAX, bool NORM>
cudaError_t launch_combine_split(const moe::CombineArgs &a, cudaStream_t s) {
    const int sms = device_sms();
    const int split = a.bs < sms && (a.hidden >> 3) % 4 == 0 ? 4 : a.bs < 2 * sms ? 2 : 1;
    const bool sh = a.shared_x != nullptr;
    if (split == 4) return sh ? launch_combine_tok<KMAX, true, NORM, 4>(a, s) : launch_combine_tok<KMAX, false, NORM, 4>(a, s);
    if (split == 2) return sh ? launch_combine_tok<KMAX, true, NORM, 2>(a, s) : launch_combine_tok<KMAX, false, NORM, 2>(a, s);
    return sh ? launch_combine_tok<KMAX, true, NORM, 1>(a, s) : launch_combine_tok<KMAX, false, NORM, 1>(a, s);
}

// The combine of a TP pair: each row is the bf16 sum of the two partial outputs (one block per token).
template <int KMAX, bool SHARED, int NT>
cudaError_t launch_combine_tp2_nt(const moe::CombineArgs &a, cudaStream_t s) {
    auto kernel = moe::combine_token_kernel<KMAX, SHARED, NT, true, 1, false, true>;
    constexpr int smem = moe::cb_smem_bytes(KMAX, NT, true, 1);
    if (!ensure_smem(kernel, smem)) return cudaErrorInvalidValue;
    return launch(kernel, a.bs, NT, smem, s, a);
}

template <int KMAX, bool SHARED>
cudaError_t launch_combine_tp2_tok(const moe::CombineArgs &a, cudaStream_t s) {
    switch (moe::cb_threads(a.hidden >> 3, 4)) {
        case 64: return launch_combine_tp2_nt<KMAX, SHARED, 64>(a, s);
        case 128: return launch_combine_tp2_nt<KMAX, SHARED, 128>(a, s);
        case 192: return launch_combine_tp2_nt<KMAX, SHARED, 192>(a, s);
        case 224: return launch_combine_tp2_nt<KMAX, SHARED, 224>(a, s);
        default: return launch_combine_tp2_nt<KMAX, SHARED, 256>(a, s);
    }
}

cudaError_t launch_combine_tp2(const moe::CombineArgs &a, int top_k, cudaStream_t s) {
    const bool sh = a.shared_x != nullptr;
    if (top_k <= 4) return sh ? launch_combine_tp2_tok<4, true>(a, s) : launch_combine_tp2_tok<4, false>(a, s);
    if (top_k <= 8) return sh ? launch_combine_tp2_tok<8, true>(a, s) : launch_combine_tp2_tok<8, false>(a, s);
    return sh ? launch_combine_tp2_tok<16, true>(a, s) : launch_combine_tp2_tok<16, false>(a, s);
}

// The combine that gathers its rows from the GPUs that own them.
template <int KMAX, bool SHARED, int NT, int SPLIT>
cudaError_t launch_combine_ep_nt(const moe::CombineArgs &a, cudaStream_t s) {
    auto kernel = moe::combine_token_kernel<KMAX, SHARED, NT, true, SPLIT, true>;
    constexpr int smem = moe::cb_smem_bytes(KMAX, NT, true, SPLIT);
    if (!ensure_smem(kernel, smem)) return cudaErrorInvalidValue;
    return launch_in_clusters(kernel, a.bs * SPLIT, NT, smem, s, SPLIT, a);
}

template <int KMAX, bool SHARED, int SPLIT>
cudaError_t launch_combine_ep_tok(const moe::CombineArgs &a, cudaStream_t s) {
    constexpr int VECS = SPLIT == 1 ? 4 : 2;
    switch (moe::cb_threads((a.hidden >> 3) / SPLIT, VECS)) {
        case 64: return launch_combine_ep_nt<KMAX, SHARED, 64, SPLIT>(a, s);
        case 128: return launch_combine_ep_nt<KMAX, SHARED, 128, SPLIT>(a, s);
        case 192: return launch_combine_ep_nt<KMAX, SHARED, 192, SPLIT>(a, s);
        case 224: return launch_combine_ep_nt<KMAX, SHARED, 224, SPLIT>(a, s);
        default: return launch_combine_ep_nt<KMAX, SHARED, 256, SPLIT>(a, s);
    }
}

// The EP combine splits rows over clusters by the same rule as the one-GPU
// combine (launch_combine_split): the peers' rows are plain loads, and the
// sums of squares meet in this GPU's distributed shared memory.
template <int KMAX>
cudaError_t launch_combine_ep_k(const moe::CombineArgs &a, cudaStream_t s) {
    const int sms = device_sms();
    const int split = a.bs < sms && (a.hidden >> 3) % 4 == 0 ? 4 : a.bs < 2 * sms ? 2 : 1;
    const bool sh = a.shared_x != nullptr;
    if (split == 4) return sh ? launch_combine_ep_tok<KMAX, true, 4>(a, s) : launch_combine_ep_tok<KMAX, false, 4>(a, s);
    if (split == 2) return sh ? launch_combine_ep_tok<KMAX, true, 2>(a, s) : launch_combine_ep_tok<KMAX, false, 2>(a, s);
    return sh ? launch_combine_ep_tok<KMAX, true, 1>(a, s) : launch_combine_ep_tok<KMAX, false, 1>(a, s);
}

cudaError_t launch_combine_ep(const moe::CombineArgs &a, int top_k, cudaStream_t s) {
    if (top_k <= 4) return launch_combine_ep_k<4>(a, s);
    if (top_k <= 8) return launch_combine_ep_k<8>(a, s);
    return launch_combine_ep_k<16>(a, s);
}

template <bool NORM>
cudaError_t launch_combine_k(const moe::CombineArgs &a, int top_k, cudaStream_t s) {
    if (top_k <= 4) return launch_combine_split<4, NORM>(a, s);
    if (top_k <= 8) return launch_combine_split<8, NORM>(a, s);
    return launch_combine_split<16, NORM>(a, s);
}

// Checks and arguments shared by the normed combine calls.
moe_status combine_norm_args(const moe_combine_params *p, const void *expand_x, const int32_t *expand_idx,
                             const float *expert_scales, const void *shared_x, const void *residual_x,
                             const void *gamma, void *y, void *x_out, float *rstd_out, void *workspace,
                             size_t workspace_bytes, moe::CombineArgs &a) {
    if (p == nullptr || !valid_combine(*p)) return MOE_ERR_INVALID_ARG;
    if (!expand_x || !expand_idx || !expert_scales || !residual_x || !gamma || !y) return MOE_ERR_INVALID_ARG;
    if (!aligned(expand_x, 16) || !aligned(residual_x, 16) || !aligned(gamma, 16) || !aligned(y, 16) ||
        (shared_x && !aligned(shared_x, 16)) || (x_out && !aligned(x_out, 16)) || !aligned(expand_idx, 4) ||
        !aligned(expert_scales, 4) || (rstd_out && !aligned(rstd_out, 4)))
        return MOE_ERR_INVALID_ARG;
    if (!check_workspace(workspace, workspace_bytes)) return MOE_ERR_WORKSPACE;
    a.bs = total_tokens(p->bs, p->sources);
    a.hidden = p->hidden;
    a.top_k = p->top_k;
    a.expand_rows = p->expand_rows;
    a.norm_eps = p->norm_eps;
    a.expand_x = reinterpret_cast<const uint16_t *>(expand_x);
    a.expand_idx = expand_idx;
    a.scales = expert_scales;
    a.shared_x = reinterpret_cast<const uint16_t *>(shared_x);
    a.residual = reinterpret_cast<const uint16_t *>(residual_x);
    a.gamma = reinterpret_cast<const uint16_t *>(gamma);
    a.y = reinterpret_cast<uint16_t *>(y);
    a.x_out = reinterpret_cast<uint16_t *>(x_out);
    a.rstd_out = rstd_out;
    a.err = reinterpret_cast<uint32_t *>(workspace);
    return MOE_OK;
}

}  // namespace

extern "C" {

const char *moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    }
    return "MOE_ERR_UNKNOWN";
}

moe_status moe_workspace_init(void *workspace, size_t bytes, void *cuda_stream) {
    if (!check_workspace(workspace, bytes)) return MOE_ERR_WORKSPACE;
    return cudaMemsetAsync(workspace, 0, bytes, as_stream(cuda_stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_clear_device_error(void *workspace, void *cuda_stream) {
    if (workspace == nullptr || !aligned(workspace, 16)) return MOE_ERR_WORKSPACE;
    return cudaMemsetAsync(workspace, 0, sizeof(uint32_t), as_stream(cuda_stream)) == cudaSuccess ? MOE_OK
                                                                                                   : MOE_ERR_CUDA;
}

moe_status moe_read_device_error(const void *workspace, uint32_t *bits, void *cuda_stream) {
    if (workspace == nullptr || !aligned(workspace, 16)) return MOE_ERR_WORKSPACE;
    if (bits == nullptr) return MOE_ERR_INVALID_ARG;
    uint32_t v = 0;
    cudaStream_t s = as_stream(cuda_stream);
    if (cudaMemcpyAsync(&v, workspace, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    *bits = v;
    return MOE_OK;
}

// ---------------------------------------------------------------- update ---

moe_status moe_update_expert_workspace_size(const moe_update_params *p, size_t *bytes) {
    if (p == nullptr || bytes == nullptr || !valid_update(*p)) return MOE_ERR_INVALID_ARG;
    *bytes = kWorkspaceBytes;
    return MOE_OK;
}

moe_status moe_update_expert(const moe_update_params *p, const int32_t *expert_ids, const float *expert_scales,
                             const uint8_t *active_mask, const int32_t *table, int32_t *balanced_ids,
                             uint8_t *balanced_mask, void *workspace, size_t workspace_bytes, void *cuda_stream) {
    if (p == nullptr || !valid_update(*p)) return MOE_ERR_INVALID_ARG;
    if (!expert_ids || !table || !balanced_ids || !balanced_mask) return MOE_ERR_INVALID_ARG;
    if (!aligned(expert_ids, 4) || !aligned(table, 4) || !aligned(balanced_ids, 4) ||
        (expert_scales && !aligned(expert_scales, 4)))
        return MOE_ERR_INVALID_ARG;
    if (!check_workspace(workspace, workspace_bytes)) return MOE_ERR_WORKSPACE;

    moe::UpdateArgs a;
    a.bs = total_tokens(p->bs, p->sources);  // every source rank's tokens; token t picks replica t mod n_e
    a.top_k = p->top_k;
    a.num_logical = p->num_logical;
    a.table_cols = p->table_cols;
    a.ep_world_size = p->ep_world_size;
    a.k_magic = moe::div_magic((uint32_t)p->top_k);
    a.prune_threshold = p->prune_threshold;
    a.expert_ids = expert_ids;
    a.expert_scales = expert_scales;
    a.active_mask = active_mask;
    a.table = table;
    // stage the table in shared memory when it fits: by one bulk copy when its
    // address and size allow one (16-byte multiples), else by plain loads
    const size_t tab_bytes = (size_t)p->num_logical * p->table_cols * sizeof(int32_t);
    a.table_mode = tab_bytes > moe::kUeTableSmemMax ? 0 : (aligned(table, 16) && tab_bytes % 16 == 0) ? 2 : 1;
    a.balanced_ids = balanced_ids;
    a.balanced_mask = balanced_mask;
    a.err = reinterpret_cast<uint32_t *>(workspace);
    const size_t smem =
        moe::update_expert_smem_bytes(p->ep_world_size, a.table_mode, p->num_logical, p->table_cols);
    if (!ensure_smem(moe::update_expert_kernel, smem)) return MOE_ERR_CUDA;
    return launch(moe::update_expert_kernel, moe::update_expert_blocks(a.bs * p->top_k), moe::kUeThreads, smem,
                  as_stream(cuda_stream), a) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

// -------------------------------------------------------------- dispatch ---

moe_status moe_dispatch_workspace_size(const moe_dispatch_params *p, size_t *bytes) {
    if (p == nullptr || bytes == nullptr) return MOE_ERR_INVALID_ARG;
    moe_status st = valid_dispatch(*p);
    if (st != MOE_OK) return st;
    *bytes = dispatch_workspace_bytes(*p);
    return MOE_OK;
}

}  // extern "C"

namespace {

// The arguments every dispatch kernel shares (pointer checks done by the caller).
moe::DispatchArgs dispatch_args(const moe_dispatch_params &p, const void *x, const int32_t *instance_ids,
                                const uint8_t *mask, const float *smooth_scales, void *expand_x, void *dyn_scales,
                                int32_t *expand_idx, int32_t *src_of_row, int32_t *expert_counts,
                                int32_t *expert_offsets, void *workspace) {
    moe::DispatchArgs a = {};
    a.bs = total_tokens(p.bs, p.sources);  // the kernels see every source rank's tokens
    a.hidden = p.hidden;
    a.top_k = p.top_k;
    a.num_instances = p.num_instances;
    a.tiles = (p.hidden + 127) / 128;
    a.k_magic = moe::div_magic((uint32_t)p.top_k);
    a.x = reinterpret_cast<const uint16_t *>(x);
    a.ids = instance_ids;
    a.mask = mask;
    a.smooth = smooth_scales;
    a.scales_len = p.scales_len;
    a.expand_x = expand_x;
    a.dyn_scales = dyn_scales;
    a.expand_idx = expand_idx;
    a.src_of_row = src_of_row;
    a.counts = expert_counts;
    a.offsets = expert_offsets;
    a.err = reinterpret_cast<uint32_t *>(workspace);
    return a;
}

// The route kernels: one pass up to kRouteSinglePassMax copies, three passes
// (with the slice table in the workspace) beyond.
cudaError_t launch_route(const moe::DispatchArgs &a, int num_instances, void *workspace, cudaStream_t s) {
    const int copies = a.bs * a.top_k;
    if (copies <= kRouteSinglePassMax) {
        const int slices = moe::route_slices(copies);
        const size_t rsmem = moe::route_smem_bytes(num_instances);
        if (!ensure_smem(moe::route_kernel, rsmem)) return cudaErrorInvalidValue;
        return launch(moe::route_kernel, slices, moe::kRtThreads, rsmem, s, a);
    }
    const int S = moe::route_large_slices(copies), E = num_instances;
    int *tab = reinterpret_cast<int *>(reinterpret_cast<unsigned char *>(workspace) + kWorkspaceBytes);
    int *tot = tab + (size_t)S * E;
    const size_t hsmem = (size_t)E * sizeof(int), psmem = moe::route_place_smem_bytes(E);
    if (!ensure_smem(moe::route_hist_kernel, hsmem) || !ensure_smem(moe::route_place_kernel, psmem))
        return cudaErrorInvalidValue;
    cudaError_t e = launch(moe::route_hist_kernel, S, moe::kRtThreads, hsmem, s, a, tab);
    if (e == cudaSuccess) e = launch(moe::route_scan_kernel, (E + 1023) / 1024, 1024, 0, s, a, tab, tot, S);
    if (e == cudaSuccess)
        e = launch(moe::route_place_kernel, S, moe::kRtThreads, psmem, s, a, (const int *)tab, (const int *)tot);
    return e;
}

// The quantize-and-scatter kernel for the mode and the scales' shape.
cudaError_t launch_scatter(const moe::DispatchArgs &a, const moe_dispatch_params &p, cudaStream_t s) {
    // scales that depend on the destination instance (a row per instance) need
    // the per-copy kernel; one coefficient or one per column is per token
    const bool per_instance = a.smooth != nullptr && p.scales_len > p.hidden;
    if (per_instance) {
        switch (p.quant_mode) {
            case 1: return launch_dispatch_token_smooth<1>(a, s);
            case 2: return launch_dispatch_token_smooth<2>(a, s);
            case 3: return launch_dispatch_token_smooth<3>(a, s);
        }
        return cudaErrorInvalidValue;
    }
    switch (p.quant_mode) {
        case 0: return launch_dispatch_token<0>(a, s);
        case 1: return launch_dispatch_token<1>(a, s);
        case 2: return launch_dispatch_token<2>(a, s);
        case 3: return launch_dispatch_token<3>(a, s);
        case 4: return launch_dispatch_token<4>(a, s);
    }
    return cudaErrorInvalidValue;
}

// Pointer rules shared by moe_dispatch and moe_ep_dispatch (the outputs they write differ).
bool dispatch_inputs_ok(const moe_dispatch_params &p, const void *x, const int32_t *instance_ids,
                        const float *smooth_scales) {
    if (!x || !instance_ids) return false;
    if ((smooth_scales != nullptr) != (p.scales_len > 0)) return false;
    return aligned(x, 16) && aligned(instance_ids, 4) &&
           (!smooth_scales || aligned(smooth_scales, p.scales_len == 1 ? 4 : 16));
}

}  // namespace

extern "C" {

moe_status moe_dispatch(const moe_dispatch_params *p, const void *x, const int32_t *instance_ids,
                        const uint8_t *mask, const float *smooth_scales, void *expand_x, void *dyn_scales,
                        int32_t *expand_idx, int32_t *src_of_row, int32_t *expert_counts, int32_t *expert_offsets,
                        void *workspace, size_t workspace_bytes, void *cuda_stream) {
    if (p == nullptr) return MOE_ERR_INVALID_ARG;
    moe_status st = valid_dispatch(*p);
    if (st != MOE_OK) return st;
    const int mode = p->quant_mode;
    if (!dispatch_inputs_ok(*p, x, instance_ids, smooth_scales)) return MOE_ERR_INVALID_ARG;
    if (!expand_x || !expand_idx || !src_of_row || !expert_counts || !expert_offsets) return MOE_ERR_INVALID_ARG;
    if ((mode == 0 || mode == 1) != (dyn_scales == nullptr)) return MOE_ERR_INVALID_ARG;  // no scales sent
    if (!aligned(expand_x, 16) || !aligned(expand_idx, 4) || !aligned(src_of_row, 4) ||
        !aligned(expert_counts, 4) || !aligned(expert_offsets, 4) ||
        ((mode == 2 || mode == 3) && !aligned(dyn_scales, 4)))
        return MOE_ERR_INVALID_ARG;
    if (!check_workspace(workspace, workspace_bytes) || workspace_bytes < dispatch_workspace_bytes(*p))
        return MOE_ERR_WORKSPACE;
    const moe::DispatchArgs a = dispatch_args(*p, x, instance_ids, mask, smooth_scales, expand_x, dyn_scales,
                                              expand_idx, src_of_row, expert_counts, expert_offsets, workspace);
    cudaStream_t s = as_stream(cuda_stream);
    // up to kFusedRouteMax copies the scatter blocks route their own copies (no route kernel)
    if (a.bs * a.top_k > moe::kFusedRouteMax && launch_route(a, p->num_instances, workspace, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return launch_scatter(a, *p, s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_dispatch_route(const moe_dispatch_params *p, const int32_t *instance_ids, const uint8_t *mask,
                              int32_t *expand_idx, int32_t *src_of_row, int32_t *expert_counts,
                              int32_t *expert_offsets, void *workspace, size_t workspace_bytes, void *cuda_stream) {
    if (p == nullptr) return MOE_ERR_INVALID_ARG;
    moe_status st = valid_dispatch(*p);
    if (st != MOE_OK) return st;
    if (!instance_ids || !expand_idx || !src_of_row || !expert_counts || !expert_offsets) return MOE_ERR_INVALID_ARG;
    if (!aligned(instance_ids, 4) || !aligned(expand_idx, 4) || !aligned(src_of_row, 4) ||
        !aligned(expert_counts, 4) || !aligned(expert_offsets, 4))
        return MOE_ERR_INVALID_ARG;
    if (!check_workspace(workspace, workspace_bytes) || workspace_bytes < dispatch_workspace_bytes(*p))
        return MOE_ERR_WORKSPACE;
    const moe::DispatchArgs a = dispatch_args(*p, nullptr, instance_ids, mask, nullptr, nullptr, nullptr, expand_idx,
                                              src_of_row, expert_counts, expert_offsets, workspace);
    return launch_route(a, p->num_instances, workspace, as_stream(cuda_stream)) == cudaSuccess ? MOE_OK
                                                                                                : MOE_ERR_CUDA;
}

// --------------------------------------------------------------- combine ---

moe_status moe_combine_add_rmsnorm_workspace_size(const moe_combine_params *p, size_t *bytes) {
    if (p == nullptr || bytes == nullptr || !valid_combine(*p)) return MOE_ERR_INVALID_ARG;
    *bytes = kWorkspaceBytes;
    return MOE_OK;
}

moe_status moe_combine_add_rmsnorm(const moe_combine_params *p, const void *expand_x, const int32_t *expand_idx,
                                   const float *expert_scales, const void *shared_x, const void *residual_x,
                                   const void *gamma, void *y, void *x_out, float *rstd_out, void *workspace,
                                   size_t workspace_bytes, void *cuda_stream) {
    moe::CombineArgs a = {};
    const moe_status st = combine_norm_args(p, expand_x, expand_idx, expert_scales, shared_x, residual_x, gamma, y,
                                            x_out, rstd_out, workspace, workspace_bytes, a);
    if (st != MOE_OK) return st;
    return launch_combine_k<true>(a, p->top_k, as_stream(cuda_stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_combine_add_rmsnorm_tp2(const moe_combine_params *p, const void *expand_x0, const void *expand_x1,
                                       const int32_t *expand_idx, const float *expert_scales, const void *shared_x,
                                       const void *residual_x, const void *gamma, void *y, void *x_out,
                                       float *rstd_out, void *workspace, size_t workspace_bytes, void *cuda_stream) {
    moe::CombineArgs a = {};
    const moe_status st = combine_norm_args(p, expand_x0, expand_idx, expert_scales, shared_x, residual_x, gamma, y,
                                            x_out, rstd_out, workspace, workspace_bytes, a);
    if (st != MOE_OK) return st;
    if (!expand_x1 || !aligned(expand_x1, 16)) return MOE_ERR_INVALID_ARG;
    a.expand_x1 = reinterpret_cast<const uint16_t *>(expand_x1);
    return launch_combine_tp2(a, p->top_k, as_stream(cuda_stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_dispatch_tp_counts(const moe_dispatch_params *p, const int32_t *src_of_row,
                                  const int32_t *expert_offsets, int32_t *tp_counts, void *workspace,
                                  size_t workspace_bytes, void *cuda_stream) {
    if (p == nullptr) return MOE_ERR_INVALID_ARG;
    moe_status st = valid_dispatch(*p);
    if (st != MOE_OK) return st;
    // a TP domain of two ranks: one instance per EP rank, every one of the 2 * ws devices a source
    if (p->num_instances != p->ep_world_size || p->sources != 2 * p->ep_world_size) return MOE_ERR_INVALID_ARG;
    if (!src_of_row || !expert_offsets || !tp_counts || !aligned(src_of_row, 4) || !aligned(expert_offsets, 4) ||
        !aligned(tp_counts, 4))
        return MOE_ERR_INVALID_ARG;
    if (!check_workspace(workspace, workspace_bytes)) return MOE_ERR_WORKSPACE;
    const int per_source = p->bs * p->top_k;
    const int copies = per_source * p->sources;
    const int threads = p->num_instances < 1024 ? ((p->num_instances + 31) / 32) * 32 : 1024;
    return launch(moe::tp_counts_kernel, 1, threads, 0, as_stream(cuda_stream), src_of_row, expert_offsets,
                  tp_counts, p->num_instances, copies, per_source, p->ep_world_size,
                  reinterpret_cast<uint32_t *>(workspace)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

// The plain combine (CombineV2 series): combineOut only.
moe_status moe_combine(const moe_combine_params *p, const void *expand_x, const int32_t *expand_idx,
                       const float *expert_scales, const void *shared_x, void *out, void *workspace,
                       size_t workspace_bytes, void *cuda_stream) {
    if (p == nullptr || !valid_combine(*p)) return MOE_ERR_INVALID_ARG;
    if (!expand_x || !expand_idx || !expert_scales || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned(expand_x, 16) || !aligned(out, 16) || (shared_x && !aligned(shared_x, 16)) ||
        !aligned(expand_idx, 4) || !aligned(expert_scales, 4))
        return MOE_ERR_INVALID_ARG;
    if (!check_workspace(workspace, workspace_bytes)) return MOE_ERR_WORKSPACE;
    moe::CombineArgs a = {};
    a.bs = total_tokens(p->bs, p->sources);
    a.hidden = p->hidden;
    a.top_k = p->top_k;
    a.expand_rows = p->expand_rows;
    a.expand_x = reinterpret_cast<const uint16_t *>(expand_x);
    a.expand_idx = expand_idx;
    a.scales = expert_scales;
    a.shared_x = reinterpret_cast<const uint16_t *>(shared_x);
    a.y = reinterpret_cast<uint16_t *>(out);
    a.err = reinterpret_cast<uint32_t *>(workspace);
    return launch_combine_k<false>(a, p->top_k, as_stream(cuda_stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ------------------------------------------------------- grouped matmul ---

moe_status moe_grouped_matmul_workspace_size(const moe_gmm_params *p, size_t *bytes) {
    if (p == nullptr || bytes == nullptr || !valid_gmm(*p)) return MOE_ERR_INVALID_ARG;
    *bytes = gmm_workspace_bytes(*p);
    return MOE_OK;
}

}  // extern "C"

namespace {

// The planning kernel, then the matmul kernel (int8 or mxfp8) over
// ceil(N / 128) x max_slots CTAs.
template <bool MX>
moe_status launch_gmm(const moe_gmm_params *p, const void *expand_x, const void *weight, moe::GmmArgs a,
                      void *workspace, cudaStream_t s) {
    CUtensorMap tm_w, tm_x;
    if (!encode_i8_rows(&tm_w, weight, (uint64_t)p->hidden, (uint64_t)p->num_instances * p->out_dim, moe::kGmBM) ||
        !encode_i8_rows(&tm_x, expand_x, (uint64_t)p->hidden, (uint64_t)p->rows, moe::kGmBoxRows))
        return MOE_ERR_CUDA;
    unsigned char *ws = reinterpret_cast<unsigned char *>(workspace);
    a.rows = p->rows;
    a.hidden = p->hidden;
    a.out_dim = p->out_dim;
    a.num_instances = p->num_instances;
    a.slot_rows = MX ? moe::kGmBNMx : moe::kGmBN;
    a.max_slots = moe::gmm_max_slots(p->rows, p->num_instances, a.slot_rows);
    a.nslots = reinterpret_cast<int *>(ws + kWorkspaceBytes);
    a.slots = reinterpret_cast<int4 *>(ws + kWorkspaceBytes + 16);
    a.err = reinterpret_cast<uint32_t *>(workspace);
    // mxfp8: 16-byte factor loads when every factor row starts on a 16-byte boundary
    const bool vec = MX && p->hidden % 512 == 0 && aligned(a.xsf, 16) && aligned(a.wsf, 16);
    auto *kernel = !MX ? moe::gmm_kernel : vec ? moe::gmm_mx_kernel<true> : moe::gmm_mx_kernel<false>;
    if (!ensure_smem(kernel, moe::kGmSmemBytes)) return MOE_ERR_CUDA;
    if (launch(moe::gmm_plan_kernel, dim3(1), 1024, 0, s, a) != cudaSuccess) return MOE_ERR_CUDA;
    const dim3 grid((p->out_dim + moe::kGmBM - 1) / moe::kGmBM, a.max_slots);
    const int threads = MX ? moe::kGmMxThreads : moe::kGmThreads;
    return launch(kernel, grid, threads, moe::kGmSmemBytes, s, tm_w, tm_x, a) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

extern "C" {

moe_status moe_grouped_matmul(const moe_gmm_params *p, const void *expand_x, const float *dyn_scales,
                              const int32_t *expert_offsets, const void *weight, const float *weight_scales,
                              void *out, void *workspace, size_t workspace_bytes, void *cuda_stream) {
    if (p == nullptr || !valid_gmm(*p)) return MOE_ERR_INVALID_ARG;
    if (!expand_x || !dyn_scales || !expert_offsets || !weight || !weight_scales || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned(expand_x, 16) || !aligned(weight, 16) || !aligned(out, 16) || !aligned(dyn_scales, 4) ||
        !aligned(expert_offsets, 4) || !aligned(weight_scales, 4))
        return MOE_ERR_INVALID_ARG;
    if (!check_workspace(workspace, workspace_bytes) || workspace_bytes < gmm_workspace_bytes(*p))
        return MOE_ERR_WORKSPACE;
    moe::GmmArgs a = {};
    a.dyn = dyn_scales;
    a.offsets = expert_offsets;
    a.wscale = weight_scales;
    a.out = reinterpret_cast<uint16_t *>(out);
    return launch_gmm<false>(p, expand_x, weight, a, workspace, as_stream(cuda_stream));
}

moe_status moe_grouped_matmul_mx(const moe_gmm_params *p, const void *expand_x, const uint8_t *x_sf,
                                 const int32_t *expert_offsets, const void *weight, const uint8_t *weight_sf,
                                 void *out, void *workspace, size_t workspace_bytes, void *cuda_stream) {
    if (p == nullptr || !valid_gmm(*p) || p->hidden % 128 != 0) return MOE_ERR_INVALID_ARG;
    if (!expand_x || !x_sf || !expert_offsets || !weight || !weight_sf || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned(expand_x, 16) || !aligned(weight, 16) || !aligned(out, 16) || !aligned(x_sf, 4) ||
        !aligned(expert_offsets, 4) || !aligned(weight_sf, 4))
        return MOE_ERR_INVALID_ARG;
    if (!check_workspace(workspace, workspace_bytes) || workspace_bytes < gmm_workspace_bytes(*p))
        return MOE_ERR_WORKSPACE;
    moe::GmmArgs a = {};
    a.offsets = expert_offsets;
    a.xsf = x_sf;
    a.wsf = weight_sf;
    a.out = reinterpret_cast<uint16_t *>(out);
    return launch_gmm<true>(p, expand_x, weight, a, workspace, as_stream(cuda_stream));
}

// ------------------------------------------------------- dispatch, no alloc ---

}  // extern "C"

namespace {

// The workspace of moe_dispatch_noalloc: a fixed array in every GPU's memory,
// so that callers who cannot allocate need not pass one.  Host code must not
// use this name as an address; the device address is looked up per device.
__device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

// The array's device address on device `dev`, looked up by the first call
// on that device (with `dev` current) and kept for the life of the process.
// Host threads may make that first call at once: the lookup runs under a
// lock and the address is published with release / acquire ordering.  A
// failed lookup stores nothing, so a later call tries again.  The cache does
// not survive cudaDeviceReset (which destroys the array with the context).
void *noalloc_scratch_address(int dev) {
    constexpr int kMaxDevices = 64;
    static std::atomic<void *> addr[kMaxDevices];
    static std::mutex mu;
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    void *p = addr[dev].load(std::memory_order_acquire);
    if (p != nullptr) return p;
    std::lock_guard<std::mutex> lock(mu);
    p = addr[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        addr[dev].store(p, std::memory_order_release);
    }
    return p;
}

}  // namespace

extern "C" moe_status moe_dispatch_noalloc(const moe_dispatch_params *p, const void *x,
                                           const int32_t *instance_ids, const uint8_t *mask,
                                           const float *smooth_scales, void *expand_x, void *dyn_scales,
                                           int32_t *expand_idx, int32_t *src_of_row, int32_t *expert_counts,
                                           int32_t *expert_offsets, uint32_t *device_error_out,
                                           void *cuda_stream) {
    size_t need = 0;
    const moe_status st = moe_dispatch_workspace_size(p, &need);
    if (st != MOE_OK) return st;
    if (need > MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
    if (device_error_out && !aligned(device_error_out, 4)) return MOE_ERR_INVALID_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    void *ws = noalloc_scratch_address(dev);
    if (ws == nullptr) return MOE_ERR_CUDA;
    cudaStream_t s = as_stream(cuda_stream);
    // the array keeps the previous call's error word: start this call from zero
    // (the rest of the scratch is written before it is read within the call)
    if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
    const moe_status r = moe_dispatch(p, x, instance_ids, mask, smooth_scales, expand_x, dyn_scales, expand_idx,
                                      src_of_row, expert_counts, expert_offsets, ws, need, cuda_stream);
    if (r != MOE_OK) return r;
    if (device_error_out &&
        cudaMemcpyAsync(device_error_out, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

// -------------------------------------------- expert parallelism across GPUs ---

namespace {

bool valid_ep(const moe_ep_params &p) {
    if (p.bs < 1 || p.bs > MOE_MAX_BS || p.top_k < 1 || p.top_k > MOE_MAX_TOP_K) return false;
    static_assert(moe::kCbMaxGpus == MOE_EP_MAX_GPUS, "the combine stages every GPU's row base");
    if (p.gpus < 1 || p.gpus > MOE_EP_MAX_GPUS || p.rank < 0 || p.rank >= p.gpus) return false;
    if (p.num_instances < 1 || p.num_instances > MOE_MAX_EXPERTS || p.num_instances % p.gpus != 0) return false;
    if (p.row_bytes < 16 || p.row_bytes % 16 != 0 || p.row_bytes > 2 * MOE_MAX_HIDDEN) return false;
    if (p.scale_bytes < 0 || p.scale_bytes > 4 * MOE_MAX_HIDDEN / 32) return false;
    if (p.recv_rows < 0) return false;
    return true;
}

// The EP workspace: the error-word area, then gstart [E] and base [G + 1].
size_t ep_workspace_bytes(const moe_ep_params &p) {
    return kWorkspaceBytes + (((size_t)p.num_instances + p.gpus + 1) * sizeof(int32_t) + 15) / 16 * 16;
}

moe::EpArgs ep_args(const moe_ep_params &p, void *workspace) {
    moe::EpArgs a = {};
    a.bs = p.bs;
    a.top_k = p.top_k;
    a.num_instances = p.num_instances;
    a.gpus = p.gpus;
    a.rank = p.rank;
    a.row_bytes = p.row_bytes;
    a.scale_bytes = p.scale_bytes;
    a.recv_rows = p.recv_rows;
    unsigned char *ws = reinterpret_cast<unsigned char *>(workspace);
    a.err = reinterpret_cast<uint32_t *>(ws);
    a.gstart = reinterpret_cast<int32_t *>(ws + kWorkspaceBytes);
    a.base = a.gstart + p.num_instances;
    return a;
}

size_t ep_copy_smem(const moe_ep_params &p) { return ((size_t)2 * p.num_instances + p.gpus + 2) * sizeof(int); }

int ep_copy_blocks(const moe_ep_params &p) {
    return (p.bs * p.top_k + moe::kEpRowsPerBlock - 1) / moe::kEpRowsPerBlock;
}

PFN_cuMemGetAddressRange_v3020 address_range_fn() {
    static PFN_cuMemGetAddressRange_v3020 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *q = nullptr;
        cudaDriverEntryPointQueryResult r;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &q, 12000, cudaEnableDefault, &r) ==
                cudaSuccess &&
            r == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(q);
    });
    return fn;
}

}  // namespace

extern "C" {

moe_status moe_ep_workspace_size(const moe_ep_params *p, size_t *bytes) {
    if (p == nullptr || bytes == nullptr || !valid_ep(*p)) return MOE_ERR_INVALID_ARG;
    *bytes = ep_workspace_bytes(*p);
    return MOE_OK;
}

moe_status moe_ep_plan(const moe_ep_params *p, const int32_t *counts_all, int32_t *recv_counts,
                       int32_t *recv_offsets, void *workspace, size_t workspace_bytes, void *cuda_stream) {
    if (p == nullptr || !valid_ep(*p)) return MOE_ERR_INVALID_ARG;
    if (!counts_all || !recv_counts || !recv_offsets || !aligned(counts_all, 4) || !aligned(recv_counts, 4) ||
        !aligned(recv_offsets, 4))
        return MOE_ERR_INVALID_ARG;
    if (!check_workspace(workspace, workspace_bytes) || workspace_bytes < ep_workspace_bytes(*p))
        return MOE_ERR_WORKSPACE;
    moe::EpArgs a = ep_args(*p, workspace);
    a.counts_all = counts_all;
    return launch(moe::ep_plan_kernel, 1, 1024, 0, as_stream(cuda_stream), a, recv_counts, recv_offsets) ==
                   cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_ep_push(const moe_ep_params *p, const void *local_rows, const void *local_scales,
                       const int32_t *local_offsets, const int32_t *src_of_row, const int32_t *expand_idx,
                       const int32_t *instance_ids, void *const *peer_rows, void *const *peer_scales,
                       int32_t *const *peer_src, int32_t *global_idx, void *workspace, size_t workspace_bytes,
                       void *cuda_stream) {
    if (p == nullptr || !valid_ep(*p)) return MOE_ERR_INVALID_ARG;
    if (!local_rows || !local_offsets || !src_of_row || !expand_idx || !instance_ids || !peer_rows || !global_idx)
        return MOE_ERR_INVALID_ARG;
    if ((p->scale_bytes > 0) != (local_scales != nullptr && peer_scales != nullptr)) return MOE_ERR_INVALID_ARG;
    if (!aligned(local_rows, 16) || !aligned(peer_rows, 8) || (peer_scales && !aligned(peer_scales, 8)) ||
        (peer_src && !aligned(peer_src, 8)) || !aligned(local_offsets, 4) || !aligned(src_of_row, 4) ||
        !aligned(expand_idx, 4) || !aligned(instance_ids, 4) || !aligned(global_idx, 4))
        return MOE_ERR_INVALID_ARG;
    if (!check_workspace(workspace, workspace_bytes) || workspace_bytes < ep_workspace_bytes(*p))
        return MOE_ERR_WORKSPACE;
    moe::EpArgs a = ep_args(*p, workspace);
    a.local_offsets = local_offsets;
    const size_t smem = ep_copy_smem(*p);
    auto kernel = moe::ep_copy_kernel<true>;
    if (!ensure_smem(kernel, smem)) return MOE_ERR_CUDA;
    return launch(kernel, ep_copy_blocks(*p), moe::kEpThreads, smem, as_stream(cuda_stream), a,
                  reinterpret_cast<const uint8_t *>(local_rows), (uint8_t *)nullptr,
                  reinterpret_cast<const uint8_t *>(local_scales), reinterpret_cast<uint8_t *const *>(peer_rows),
                  reinterpret_cast<uint8_t *const *>(peer_scales), peer_src, src_of_row, expand_idx, global_idx,
                  instance_ids) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_ep_pull(const moe_ep_params *p, void *const *peer_rows, const int32_t *local_offsets, void *local_rows,
                       void *workspace, size_t workspace_bytes, void *cuda_stream) {
    if (p == nullptr || !valid_ep(*p)) return MOE_ERR_INVALID_ARG;
    if (!peer_rows || !local_offsets || !local_rows) return MOE_ERR_INVALID_ARG;
    if (!aligned(local_rows, 16) || !aligned(peer_rows, 8) || !aligned(local_offsets, 4)) return MOE_ERR_INVALID_ARG;
    if (!check_workspace(workspace, workspace_bytes) || workspace_bytes < ep_workspace_bytes(*p))
        return MOE_ERR_WORKSPACE;
    moe::EpArgs a = ep_args(*p, workspace);
    a.local_offsets = local_offsets;
    const size_t smem = ep_copy_smem(*p);
    auto kernel = moe::ep_copy_kernel<false>;
    if (!ensure_smem(kernel, smem)) return MOE_ERR_CUDA;
    return launch(kernel, ep_copy_blocks(*p), moe::kEpThreads, smem, as_stream(cuda_stream), a,
                  (const uint8_t *)nullptr, reinterpret_cast<uint8_t *>(local_rows), (const uint8_t *)nullptr,
                  reinterpret_cast<uint8_t *const *>(peer_rows), (uint8_t *const *)nullptr, (int32_t *const *)nullptr,
                  (const int32_t *)nullptr, (const int32_t *)nullptr, (int32_t *)nullptr,
                  (const int32_t *)nullptr) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_ep_dispatch(const moe_dispatch_params *p, const moe_ep_params *ep, const void *x,
                           const int32_t *instance_ids, const uint8_t *mask, const float *smooth_scales,
                           const int32_t *expand_idx, const int32_t *expert_offsets, void *const *peer_rows,
                           void *const *peer_scales, int32_t *const *peer_src, int32_t *global_idx,
                           void *ep_workspace, size_t ep_ws_bytes, void *cuda_stream) {
    if (p == nullptr || ep == nullptr || !valid_ep(*ep)) return MOE_ERR_INVALID_ARG;
    moe_status st = valid_dispatch(*p);
    if (st != MOE_OK) return st;
    const int mode = p->quant_mode;
    // one source per GPU; the EP parameters describe the same call
    if (p->sources > 1 || ep->bs != p->bs || ep->top_k != p->top_k || ep->num_instances != p->num_instances)
        return MOE_ERR_INVALID_ARG;
    if (ep->row_bytes != (mode == 0 ? 2 : 1) * p->hidden) return MOE_ERR_INVALID_ARG;
    const int sb = mode == 2 ? 4 : mode == 3 ? 4 * ((p->hidden + 127) / 128) : mode == 4 ? p->hidden / 32 : 0;
    if (ep->scale_bytes != sb) return MOE_ERR_INVALID_ARG;
    if (!dispatch_inputs_ok(*p, x, instance_ids, smooth_scales)) return MOE_ERR_INVALID_ARG;
    if (!expand_idx || !expert_offsets || !peer_rows || !global_idx || ((sb > 0) != (peer_scales != nullptr)))
        return MOE_ERR_INVALID_ARG;
    if (!aligned(expand_idx, 4) || !aligned(expert_offsets, 4) || !aligned(global_idx, 4) || !aligned(peer_rows, 8) ||
        (peer_scales && !aligned(peer_scales, 8)) || (peer_src && !aligned(peer_src, 8)))
        return MOE_ERR_INVALID_ARG;
    if (!check_workspace(ep_workspace, ep_ws_bytes) || ep_ws_bytes < ep_workspace_bytes(*ep))
        return MOE_ERR_WORKSPACE;
    moe::DispatchArgs a = dispatch_args(*p, x, instance_ids, mask, smooth_scales, nullptr, nullptr,
                                        const_cast<int32_t *>(expand_idx), nullptr, nullptr,
                                        const_cast<int32_t *>(expert_offsets), ep_workspace);
    const moe::EpArgs plan = ep_args(*ep, ep_workspace);
    a.peer_x = reinterpret_cast<uint8_t *const *>(peer_rows);
    a.peer_sc = reinterpret_cast<uint8_t *const *>(peer_scales);
    a.peer_src = peer_src;
    a.gstart = plan.gstart;
    a.gbase = plan.base;
    a.global_idx = global_idx;
    a.ep_el = ep->num_instances / ep->gpus;
    a.ep_recv_rows = ep->recv_rows;
    a.ep_src_base = ep->rank * ep->bs * ep->top_k;
    a.scale_bytes = sb;
    return launch_scatter(a, *p, as_stream(cuda_stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_ep_combine_add_rmsnorm(const moe_combine_params *p, const moe_ep_params *ep, void *const *peer_rows,
                                      const int32_t *global_idx, const float *expert_scales, const void *shared_x,
                                      const void *residual_x, const void *gamma, void *y, void *x_out,
                                      float *rstd_out, void *ep_workspace, size_t ep_ws_bytes,
                                      void *cuda_stream) {
    if (p == nullptr || ep == nullptr || !valid_combine(*p) || !valid_ep(*ep)) return MOE_ERR_INVALID_ARG;
    if (p->sources > 1 || ep->bs != p->bs || ep->top_k != p->top_k || ep->row_bytes != 2 * p->hidden)
        return MOE_ERR_INVALID_ARG;
    if (!peer_rows || !global_idx || !expert_scales || !residual_x || !gamma || !y) return MOE_ERR_INVALID_ARG;
    if (!aligned(peer_rows, 8) || !aligned(residual_x, 16) || !aligned(gamma, 16) || !aligned(y, 16) ||
        (shared_x && !aligned(shared_x, 16)) || (x_out && !aligned(x_out, 16)) || !aligned(global_idx, 4) ||
        !aligned(expert_scales, 4) || (rstd_out && !aligned(rstd_out, 4)))
        return MOE_ERR_INVALID_ARG;
    if (!check_workspace(ep_workspace, ep_ws_bytes) || ep_ws_bytes < ep_workspace_bytes(*ep))
        return MOE_ERR_WORKSPACE;
    const moe::EpArgs plan = ep_args(*ep, ep_workspace);
    moe::CombineArgs a = {};
    a.bs = p->bs;
    a.hidden = p->hidden;
    a.top_k = p->top_k;
    a.expand_rows = 0x7fffffff;  // global rows: bounded by the plan's last base instead
    a.norm_eps = p->norm_eps;
    a.expand_idx = global_idx;
    a.scales = expert_scales;
    a.shared_x = reinterpret_cast<const uint16_t *>(shared_x);
    a.residual = reinterpret_cast<const uint16_t *>(residual_x);
    a.gamma = reinterpret_cast<const uint16_t *>(gamma);
    a.y = reinterpret_cast<uint16_t *>(y);
    a.x_out = reinterpret_cast<uint16_t *>(x_out);
    a.rstd_out = rstd_out;
    a.err = plan.err;
    a.peer_rows = reinterpret_cast<const uint16_t *const *>(peer_rows);
    a.gbase = plan.base;
    a.gpus = ep->gpus;
    a.recv_rows = ep->recv_rows;
    return launch_combine_ep(a, p->top_k, as_stream(cuda_stream)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_ipc_export(const void *dev_ptr, void *handle, uint64_t *offset) {
    if (dev_ptr == nullptr || handle == nullptr || offset == nullptr) return MOE_ERR_INVALID_ARG;
    const PFN_cuMemGetAddressRange_v3020 range = address_range_fn();
    if (range == nullptr) return MOE_ERR_CUDA;
    CUdeviceptr base = 0;
    size_t size = 0;
    if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS) return MOE_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess) return MOE_ERR_CUDA;
    static_assert(sizeof(h) == MOE_IPC_HANDLE_BYTES, "IPC handle size");
    std::memcpy(handle, &h, sizeof h);
    *offset = reinterpret_cast<uint64_t>(dev_ptr) - static_cast<uint64_t>(base);
    return MOE_OK;
}

moe_status moe_ipc_import(const void *handle, uint64_t offset, void **base, void **dev_ptr) {
    if (handle == nullptr || base == nullptr || dev_ptr == nullptr) return MOE_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof h);
    void *b = nullptr;
    if (cudaIpcOpenMemHandle(&b, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return MOE_ERR_CUDA;
    *base = b;
    *dev_ptr = static_cast<unsigned char *>(b) + offset;
    return MOE_OK;
}

moe_status moe_ipc_close(void *base) {
    if (base == nullptr) return MOE_ERR_INVALID_ARG;
    return cudaIpcCloseMemHandle(base) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
