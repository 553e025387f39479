/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) MoE update-expert / dispatch /
 * combine+Add+RMSNorm library (libmoe_b200.so).
 *
 * The three operations follow three operator pages:
 *   aclnnMoeUpdateExpert                  -> moe_update_expert
 *   aclnnMoeDistributeDispatchV2          -> moe_dispatch
 *   aclnnMoeDistributeCombineAddRmsNorm   -> moe_combine_add_rmsnorm
 * (with moe_combine, the plain CombineV2-series combine that the dispatch
 * page pairs it with) and, like them, come in two phases: *_workspace_size() checks the
 * parameters and sizes the workspace, then the call itself runs on a CUDA
 * stream ("函数原型" / "Parameters" / "Returns" sections of each page).
 *
 * Expert parallelism on one GPU.  The pages' epWorldSize ranks are simulated
 * as partitions of one rank-major receive buffer in this GPU's memory: the
 * EP AllToAllV of dispatch is a permutation of rows into that buffer, and
 * the AllToAllV of combine is a gather back out of it.  No collective and no
 * inter-GPU traffic is involved.  One source rank of `bs` tokens feeds the
 * exchange.
 *
 * Conventions for every entry point:
 *   - Pointers named as device pointers are CUDA device (or managed) memory
 *     owned by the caller; the library never allocates, frees or keeps them.
 *     Arrays are dense and row-major.  bf16 arrays and the int8 / e4m3 rows of
 *     expand_x must start on a 16-byte boundary; int32 / f32 arrays on 4 bytes.
 *   - `cuda_stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls only enqueue work: they neither allocate nor synchronize
 *     (except moe_read_device_error), so they may be captured in CUDA graphs.
 *   - Errors the host can see (bad sizes, NULL / misaligned pointers, a
 *     workspace that is too small) return a non-zero moe_status and enqueue
 *     nothing.  Errors only the device can see (an id out of range, a bad
 *     mapping table) never trap: the offending item is dropped and a sticky
 *     bit is OR-ed into the error word at the start of the workspace, which
 *     moe_read_device_error returns.
 *   - Every output is a pure function of the inputs: runs are bitwise
 *     reproducible ("确定性计算" / "Deterministic computation" on each page).
 *   - The workspace must be zeroed once (moe_workspace_init) before its first
 *     use; the error word then accumulates until moe_clear_device_error.
 *     Calls that share a workspace share its error word.  A workspace of
 *     MOE_MAX_WORKSPACE_BYTES serves every call with one source rank (and
 *     any call of at most 8192 copies); dispatch with several source ranks
 *     may need more, as moe_dispatch_workspace_size reports.
 *   - Several source ranks (the "sources" field): the pages' AllToAllV has
 *     every EP rank send Bs tokens.  With sources = S, the calls take
 *     T = S * bs tokens, rank-major (token t = r * bs + i of source rank r);
 *     rows are ordered by (instance, r, i, k), the same as (instance, t, k).
 *     0 means 1.  S goes up to 2 * ep_world_size: with a TP domain of two
 *     ranks (tpWorldSize 2 on the pages) every one of the 2 * ep_world_size
 *     devices is a source, numbered TP-major (device t * ep_world_size + g
 *     is EP rank g of TP domain t); see moe_dispatch_tp_counts and
 *     moe_combine_add_rmsnorm_tp2.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported from libmoe_b200.so; everything else in the library is hidden. */
#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,  /* a size outside the pages' limits, a NULL or misaligned pointer */
    MOE_ERR_UNSUPPORTED = 2,  /* a legal value this library does not implement */
    MOE_ERR_WORKSPACE = 3,    /* workspace NULL or smaller than *_workspace_size reported */
    MOE_ERR_CUDA = 4          /* the CUDA runtime refused a launch or a copy */
} moe_status;

/* Bits of the device error word (first 4 bytes of the workspace). */
#define MOE_DEV_BAD_ID    1u  /* an expert / instance id or an expand_idx row out of range */
#define MOE_DEV_BAD_TABLE 2u  /* mapping table broke its restrictions; every copy was dropped */
#define MOE_DEV_TIMEOUT   4u  /* a bounded wait for an asynchronous copy gave up; outputs incomplete */
#define MOE_DEV_CAPACITY  8u  /* expert parallelism: a receive buffer too small; rows beyond it dropped */

/* The largest workspace any *_workspace_size call reports for one source
 * rank (bytes): the 256-byte area that holds the error word. */
#define MOE_MAX_WORKSPACE_BYTES 256

/* Limits taken from the pages (shape-variable constraints of each page). */
#define MOE_MAX_BS        512   /* Bs in (0, 512] */
#define MOE_MIN_HIDDEN    1024  /* H in [1024, 8192] */
#define MOE_MAX_HIDDEN    8192
#define MOE_MAX_TOP_K     16    /* K in (0, 16], K <= expert count */
#define MOE_MAX_EXPERTS   1024  /* logical experts and deployed instances each <= 1024 */
#define MOE_MIN_EP_WORLD  2     /* epWorldSize in [2, 768] */
#define MOE_MAX_EP_WORLD  768

/* ------------------------------------------------------------------------ */
/* Workspace and the device error word                                       */
/* ------------------------------------------------------------------------ */

/* Zero `bytes` of a workspace on `cuda_stream` (cudaMemsetAsync). */
MOE_API moe_status moe_workspace_init(void *workspace, size_t bytes, void *cuda_stream);

/* Synchronize `cuda_stream`, then copy the error word of `workspace` into
 * *bits (a host pointer).  The only call in this library that blocks. */
MOE_API moe_status moe_read_device_error(const void *workspace, uint32_t *bits, void *cuda_stream);

/* Zero the error word of `workspace` on `cuda_stream`. */
MOE_API moe_status moe_clear_device_error(void *workspace, void *cuda_stream);

/* Human-readable name of a status code (static storage). */
MOE_API const char *moe_status_string(moe_status status);

/* ------------------------------------------------------------------------ */
/* moe_update_expert -- aclnnMoeUpdateExpert (load balancing + pruning)      */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t bs;             /* tokens, (0, 512] */
    int32_t top_k;          /* K, (0, 16] and <= num_logical */
    int32_t num_logical;    /* logical experts = rows of the table, (0, 1024] */
    int32_t table_cols;     /* F, [2, ep_world_size + 1] */
    int32_t ep_world_size;  /* simulated ranks, [2, 768] */
    float prune_threshold;  /* copies whose expert_scales entry is strictly below this are
                               pruned; <= 0 (or expert_scales == NULL) disables */
    int32_t sources;        /* source ranks S, [0, 2 * ep_world_size] (0 = 1): arrays hold S * bs tokens */
} moe_update_params;

MOE_API moe_status moe_update_expert_workspace_size(const moe_update_params *p, size_t *bytes);

/*
 * Maps each token's K logical expert ids to deployed instance ids and
 * computes the keep mask (aclnnMoeUpdateExpert, description: "Load
 * balancing", "Expert pruning"; "Restriction on the shape format").
 *
 *   expert_ids    [bs, K] int32  device, logical ids in [0, num_logical)
 *   expert_scales [bs, K] f32    device, optional (NULL = no threshold pruning)
 *   active_mask   [bs]    uint8  device, optional; 0 prunes every copy of a token
 *                                (the (BS,) mask broadcast to (BS,K))
 *   table         [num_logical, F] int32 device: column 0 = n_e instances of
 *                                expert e (>= 1, <= F-1), columns 1..n_e = the
 *                                rank hosting each instance.  All instances
 *                                together <= 1024, every rank hosting the same
 *                                number L of them.
 *   balanced_ids  [bs, K] int32  device, out: instance id = rank * L + slot,
 *                                slots numbered per rank in (expert, replica)
 *                                order; token i uses replica i mod n_e.  So the
 *                                rank is balanced_ids / L.
 *   balanced_mask [bs, K] uint8  device, out: 1 = keep, 0 = pruned
 *
 * Device errors: a bad table sets MOE_DEV_BAD_TABLE and writes -1 / 0 for
 * every copy; an id outside [0, num_logical) sets MOE_DEV_BAD_ID and writes
 * -1 / 0 for that copy.  (The page's own load-balancing formula did not
 * survive extraction; the replica rule above is this library's reading.)
 */
MOE_API moe_status moe_update_expert(const moe_update_params *p, const int32_t *expert_ids,
                             const float *expert_scales, const uint8_t *active_mask,
                             const int32_t *table, int32_t *balanced_ids,
                             uint8_t *balanced_mask, void *workspace, size_t workspace_bytes,
                             void *cuda_stream);

/* ------------------------------------------------------------------------ */
/* moe_dispatch -- aclnnMoeDistributeDispatchV2 (quantize + EP AllToAllV)    */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t bs;             /* tokens, (0, 512] */
    int32_t hidden;         /* H, [1024, 8192]; this library needs H % 16 == 0 (H % 32 == 0 in mode 4) */
    int32_t top_k;          /* K, (0, 16] and <= num_instances */
    int32_t ep_world_size;  /* simulated ranks, [2, 768]; must divide num_instances */
    int32_t num_instances;  /* deployed expert instances E, (0, 1024] */
    int32_t quant_mode;     /* 0 none, 1 static int8, 2 per-token int8, 3 per-128-tile int8, 4 mxfp8 */
    int32_t scales_len;     /* floats in smooth_scales: 0 when it is NULL; modes 2/3 num_instances * H;
                               mode 1: 1, H or num_instances * H (the static scales' shape) */
    int32_t sources;        /* source ranks S, [0, 2 * ep_world_size] (0 = 1): x and the routing hold
                               S * bs tokens, expand_x S * bs * K rows */
} moe_dispatch_params;

MOE_API moe_status moe_dispatch_workspace_size(const moe_dispatch_params *p, size_t *bytes);

/*
 * Orders the active (token, k) copies by destination instance and writes each
 * one, quantized per quant_mode, into the expert-major receive buffer
 * (aclnnMoeDistributeDispatchV2, "计算公式" cases 1 to 5).  Rows are
 * sorted by (instance, token, k); instance ids are rank-major, so simulated
 * rank r receives rows [expert_offsets[r*L], expert_offsets[(r+1)*L]).
 *
 *   x             [bs, H] bf16   device
 *   instance_ids  [bs, K] int32  device, in [0, num_instances) (moe_update_expert's output)
 *   mask          [bs, K] uint8  device, optional; 0 = copy not sent
 *   smooth_scales f32 device, p->scales_len floats:
 *                   modes 2 and 3, optional: [num_instances, H] smooth scales,
 *                     xFp32 = x * smooth_scales[instance];
 *                   mode 1, required: the static scales, shape (1,), (H,) or
 *                     [num_instances, H] (row of the copy's instance),
 *                     xFp32 = x * scale, code = Cast(xFp32, int8);
 *                   modes 0 and 4: NULL.
 *   expand_x      [bs*K, H]      device, out: bf16 (mode 0), int8 (1, 2, 3) or e4m3 (4).
 *                                Rows >= expert_offsets[E] are left untouched.
 *   dyn_scales    device, out, NULL in modes 0 and 1:
 *                   mode 2: [bs*K] f32 = 1 / (127 / max|xFp32|)        (0 for an all-zero row)
 *                   mode 3: [bs*K, ceil(H/128)] f32, the same per 128-element tile
 *                   mode 4: [bs*K, H/32] uint8 E8M0 byte = sharedExp + 127, the
 *                           dequantization factor 2^sharedExp of each 32-block,
 *                           sharedExp = floor(log2 max|x|) - 8 clamped to >= -127
 *   expand_idx    [bs, K] int32  device, out: row of copy (i, k), -1 if not sent
 *   src_of_row    [bs*K]  int32  device, out: i*K + k of each row < expert_offsets[E]
 *   expert_counts [E]     int32  device, out: rows received by each instance
 *   expert_offsets[E+1]   int32  device, out: exclusive prefix sum, [E] = rows used
 *
 * int8 codes round half to even and clamp to [-127, 127] (modes 2 and 3) or
 * saturate to [-128, 127] with NaN giving 0 (mode 1, static); e4m3 codes
 * round half to even and saturate at +-448.  All quantization arithmetic is IEEE
 * binary32, so codes and scales are bit-exact against any IEEE evaluation of
 * the same formulas.  Device errors: an instance id out of range sets
 * MOE_DEV_BAD_ID and the copy is not sent.
 */
MOE_API moe_status moe_dispatch(const moe_dispatch_params *p, const void *x, const int32_t *instance_ids,
                        const uint8_t *mask, const float *smooth_scales, void *expand_x,
                        void *dyn_scales, int32_t *expand_idx, int32_t *src_of_row,
                        int32_t *expert_counts, int32_t *expert_offsets, void *workspace,
                        size_t workspace_bytes, void *cuda_stream);

/*
 * The routing half of moe_dispatch alone: expand_idx, src_of_row,
 * expert_counts and expert_offsets exactly as moe_dispatch writes them, with
 * no row moved (the rows follow from moe_ep_dispatch once the group's counts
 * are known).  Arguments, limits and errors as moe_dispatch.
 */
/*
 * The per-(rank, TP domain) row counts of a dispatch with a TP domain of two
 * ranks (aclnnMoeDistributeDispatchV2, "计算公式": expandXOut =
 * AllGatherV(allToAllXOut); its expertTokenNums has epWorldSize * tpWorldSize
 * * localExpertNum entries).  With one instance per EP rank
 * (num_instances == ep_world_size, the pages allow TP only then) and
 * sources = 2 * ep_world_size numbered TP-major, moe_dispatch's rows of
 * instance e are rank e's gathered buffer: TP domain 0's rows first, then
 * domain 1's.  This call splits each instance's rows at that boundary.
 *   p              the moe_dispatch parameters of the call (sources = 2 * ws,
 *                  num_instances = ws, else MOE_ERR_INVALID_ARG)
 *   src_of_row, expert_offsets: moe_dispatch's outputs
 *   tp_counts      [E, 2] int32 device, out: rows of (instance e, TP domain t)
 * Device errors: offsets outside [0, rows] set MOE_DEV_BAD_ID (that
 * instance's counts are 0).
 */
MOE_API moe_status moe_dispatch_tp_counts(const moe_dispatch_params *p, const int32_t *src_of_row,
                                          const int32_t *expert_offsets, int32_t *tp_counts, void *workspace,
                                          size_t workspace_bytes, void *cuda_stream);

MOE_API moe_status moe_dispatch_route(const moe_dispatch_params *p, const int32_t *instance_ids,
                                      const uint8_t *mask, int32_t *expand_idx, int32_t *src_of_row,
                                      int32_t *expert_counts, int32_t *expert_offsets, void *workspace,
                                      size_t workspace_bytes, void *cuda_stream);

/* ------------------------------------------------------------------------ */
/* moe_combine_add_rmsnorm -- aclnnMoeDistributeCombineAddRmsNorm            */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t bs;           /* tokens, (0, 512] */
    int32_t hidden;       /* H, [1024, 8192], H % 16 == 0 */
    int32_t top_k;        /* K, (0, 16] */
    int32_t expand_rows;  /* rows of expand_x (>= every non-negative expand_idx + 1), > 0 */
    float norm_eps;       /* normEps, finite and >= 0 */
    int32_t sources;      /* source ranks S, [0, 1536] (0 = 1): the token arrays hold S * bs tokens */
} moe_combine_params;

MOE_API moe_status moe_combine_add_rmsnorm_workspace_size(const moe_combine_params *p, size_t *bytes);

/*
 * For each token i (aclnnMoeDistributeCombineAddRmsNorm, "计算公式"):
 *   combineOut = sum over kept k of (s_ik * expand_x[expand_idx[i,k]] + s_ik * shared_x[i])
 *   x          = combineOut + residual_x[i]
 *   y          = x / sqrt(mean_h(x^2) + norm_eps) * gamma
 * accumulated in fp32.  A copy with expand_idx == -1 (pruned) contributes
 * nothing, its weight included.
 *
 *   expand_x      [expand_rows, H] bf16 device (the expert outputs, rows as dispatch laid them out)
 *   expand_idx    [bs, K] int32  device (dispatch's output)
 *   expert_scales [bs, K] f32    device
 *   shared_x      [bs, H] bf16   device, optional (shared-expert output)
 *   residual_x    [bs, H] bf16   device
 *   gamma         [H]     bf16   device
 *   y             [bs, H] bf16   device, out
 *   x_out         [bs, H] bf16   device, optional out: x before the norm
 *   rstd_out      [bs]    f32    device, optional out: 1 / sqrt(mean(x^2) + eps)
 *
 * Device errors: an expand_idx entry >= expand_rows (or < -1) sets
 * MOE_DEV_BAD_ID and that copy is skipped.
 */
MOE_API moe_status moe_combine_add_rmsnorm(const moe_combine_params *p, const void *expand_x,
                                   const int32_t *expand_idx, const float *expert_scales,
                                   const void *shared_x, const void *residual_x, const void *gamma,
                                   void *y, void *x_out, float *rstd_out, void *workspace,
                                   size_t workspace_bytes, void *cuda_stream);

/*
 * The same with a TP domain of two ranks (aclnnMoeDistributeCombineAddRmsNorm,
 * "计算公式": rsOut = ReduceScatterV(expandX), then ataOut = AllToAllV(rsOut)):
 * each TP rank holds a partial expert output of all its pair's rows; row r
 * of rsOut is the bf16 (round to nearest even) of expand_x0[r] + expand_x1[r]
 * (the sum of two bf16 values in fp32 rounds to the same bf16 as their
 * exact sum), and each token reads its own rows of it.  On one device the
 * token arrays hold every source device's tokens (sources = 2 * ws,
 * TP-major), so the scatter half and the AllToAllV back are the gather
 * through expand_idx.
 *   expand_x0, expand_x1 [expand_rows, H] bf16 device, 16-byte aligned: the
 *                        two TP ranks' partial outputs; either may be the
 *                        other GPU's buffer as mapped on this one
 *                        (moe_ipc_import), read with plain loads over
 *                        NVLink, so a TP pair on two GPUs combines each
 *                        GPU's own tokens with this call
 * Other arguments and errors as moe_combine_add_rmsnorm.
 */
MOE_API moe_status moe_combine_add_rmsnorm_tp2(const moe_combine_params *p, const void *expand_x0,
                                               const void *expand_x1, const int32_t *expand_idx,
                                               const float *expert_scales, const void *shared_x,
                                               const void *residual_x, const void *gamma, void *y, void *x_out,
                                               float *rstd_out, void *workspace, size_t workspace_bytes,
                                               void *cuda_stream);

/*
 * The plain combine of the CombineV2 series, which the dispatch page names as
 * its pairing (aclnnMoeDistributeDispatchV2, constraints; the formula is the
 * first line of the one above, with no residual and no norm):
 *   out[i] = sum over kept k of (s_ik * expand_x[expand_idx[i,k]] + s_ik * shared_x[i])
 * accumulated in fp32 and rounded to bf16 once.  Parameters as for
 * moe_combine_add_rmsnorm (norm_eps is not used); out is [bs, H] bf16.
 */
MOE_API moe_status moe_combine(const moe_combine_params *p, const void *expand_x, const int32_t *expand_idx,
                               const float *expert_scales, const void *shared_x, void *out, void *workspace,
                               size_t workspace_bytes, void *cuda_stream);

/* ------------------------------------------------------------------------ */
/* moe_grouped_matmul -- the instances' int8 matmul between dispatch and     */
/* combine                                                                    */
/* ------------------------------------------------------------------------ */

/* Output channels per instance at most. */
#define MOE_GMM_MAX_OUT_DIM 65536

typedef struct {
    int32_t rows;           /* rows of expand_x and out, > 0 (the dispatch's receive rows) */
    int32_t hidden;         /* H, the contraction length, [1024, 8192], H % 16 == 0 */
    int32_t out_dim;        /* N, output channels per instance, [16, 65536], N % 16 == 0 */
    int32_t num_instances;  /* deployed instances E, (0, 1024] */
} moe_gmm_params;

MOE_API moe_status moe_grouped_matmul_workspace_size(const moe_gmm_params *p, size_t *bytes);

/*
 * The expert step between the dispatch ("AllToAllV(quantOut)", dispatch page,
 * "计算公式") and the gather the combine starts from ("ataOut", combine page,
 * "计算公式").  The pages do not define it; this library takes it as the one
 * contraction that consumes the dispatch output: instance e multiplies its
 * rows, [expert_offsets[e], expert_offsets[e+1]) of expand_x, by its own
 * weight:
 *   out[r][n] = (sum_h expand_x[r][h] * weight[e][n][h]) * dyn_scales[r] * weight_scales[e][n]
 * The sum is exact (int32); the two products are binary32; out is bf16
 * (round to nearest even).  With N = H the result is the expand_x that
 * moe_combine / moe_combine_add_rmsnorm gather.
 *
 *   expand_x       [rows, H] int8 device, 16-byte aligned (moe_dispatch, quant_mode 1 or 2)
 *   dyn_scales     [rows] f32 device: each row's dequantization factor (the
 *                  dispatch's mode-2 dyn_scales; a constant array for mode 1)
 *   expert_offsets [E+1] int32 device (moe_dispatch's output): a non-decreasing
 *                  run in [0, rows]
 *   weight         [E, N, H] int8 device, 16-byte aligned: each output channel's
 *                  H weights contiguous
 *   weight_scales  [E, N] f32 device
 *   out            [rows, N] bf16 device, 16-byte aligned; rows outside
 *                  [expert_offsets[0], expert_offsets[E]) are left untouched
 *   workspace      device, moe_grouped_matmul_workspace_size bytes, 16-byte aligned
 *
 * Host errors: MOE_ERR_INVALID_ARG for sizes outside the limits or NULL /
 * misaligned pointers, MOE_ERR_WORKSPACE, MOE_ERR_CUDA if a tensor map cannot
 * be encoded or a launch is refused.  Device errors: offsets that are not a
 * non-decreasing run in [0, rows] set MOE_DEV_BAD_ID and nothing is written;
 * a bounded wait that gives up sets MOE_DEV_TIMEOUT.
 */
MOE_API moe_status moe_grouped_matmul(const moe_gmm_params *p, const void *expand_x, const float *dyn_scales,
                                      const int32_t *expert_offsets, const void *weight,
                                      const float *weight_scales, void *out, void *workspace,
                                      size_t workspace_bytes, void *cuda_stream);

/*
 * The same step on mxfp8 rows (moe_dispatch quant_mode 4) and mxfp8 weights,
 * on the block-scaled tensor-core path:
 *   out[r][n] = sum_h dec(expand_x[r][h]) * 2^(x_sf[r][h/32] - 127)
 *                    * dec(weight[e][n][h]) * 2^(weight_sf[e][n][h/32] - 127)
 * where dec is the E4M3 value of a code; the sum is formed by the tensor
 * cores in fp32 and rounded to bf16 once.
 *
 *   expand_x   [rows, H] E4M3 codes (uint8) device, 16-byte aligned
 *   x_sf       [rows, H/32] uint8 E8M0 device, 4-byte aligned (the dispatch's mode-4 dyn_scales)
 *   weight     [E, N, H] E4M3 codes device, 16-byte aligned
 *   weight_sf  [E, N, H/32] uint8 E8M0 device, 4-byte aligned
 * Other arguments, limits and errors as moe_grouped_matmul, plus H % 128 == 0
 * (each 128-element step reads one 4-byte word of factors per row).
 */
MOE_API moe_status moe_grouped_matmul_mx(const moe_gmm_params *p, const void *expand_x, const uint8_t *x_sf,
                                         const int32_t *expert_offsets, const void *weight,
                                         const uint8_t *weight_sf, void *out, void *workspace,
                                         size_t workspace_bytes, void *cuda_stream);

/* ------------------------------------------------------------------------ */
/* moe_dispatch_noalloc -- moe_dispatch without a caller-provided workspace  */
/* ------------------------------------------------------------------------ */

/* Size of the static scratch array behind moe_dispatch_noalloc (bytes), on
 * every GPU that loads the library.  It covers every call with one source
 * rank and any call of at most 8192 (token, k) copies; a call with several
 * source ranks past 8192 copies needs a larger workspace (its route table)
 * and moe_dispatch_noalloc refuses it with MOE_ERR_WORKSPACE, launching
 * nothing. */
#define MOE_NOALLOC_SCRATCH_BYTES MOE_MAX_WORKSPACE_BYTES

/*
 * The operator pages have no counterpart for this call; it exists for
 * callers that cannot allocate device memory of their own: runtimes that
 * hand a kernel only the tensors it reads and writes (no workspace), or that
 * run under a fixed memory plan where a cudaMalloc after start-up is not
 * allowed.  It does exactly what moe_dispatch does, with the same arguments
 * and results, but the workspace lives in a static device array inside the
 * library (MOE_NOALLOC_SCRATCH_BYTES per GPU, held by every GPU that loads
 * the library until the process exits).  It calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *
 *   device_error_out  optional device pointer (4 bytes, caller-owned): receives
 *                     this call's device error word (MOE_DEV_* bits) at its end.
 *
 * The first call on a device looks the array's device address up (with that
 * device current; several host threads may make it at once); make that first
 * call before any stream capture.  The address is kept until the process
 * exits and is not valid after cudaDeviceReset.  Each call zeroes the error
 * word first, and every call on a device shares the one array, so calls that
 * overlap on the GPU (other streams, other threads) race on it.  Returns
 * MOE_ERR_WORKSPACE, enqueuing nothing, if the call would need more scratch
 * than the array holds (see MOE_NOALLOC_SCRATCH_BYTES); other errors as
 * moe_dispatch.
 */
MOE_API moe_status moe_dispatch_noalloc(const moe_dispatch_params *p, const void *x, const int32_t *instance_ids,
                                        const uint8_t *mask, const float *smooth_scales, void *expand_x,
                                        void *dyn_scales, int32_t *expand_idx, int32_t *src_of_row,
                                        int32_t *expert_counts, int32_t *expert_offsets, uint32_t *device_error_out,
                                        void *cuda_stream);

/* ------------------------------------------------------------------------ */
/* Expert parallelism across GPUs: the AllToAllV of dispatch and of combine  */
/* ------------------------------------------------------------------------ */

/*
 * The pages' EP AllToAllV moves every quantized copy to the rank hosting its
 * instance (aclnnMoeDistributeDispatchV2, "功能说明", "计算公式": quantOut
 * then AllToAllV) and the expert outputs back (aclnnMoeDistributeCombineAddRmsNorm,
 * "计算公式": ataOut = AllToAllV).  Across G GPUs, GPU q owns the instances
 * [q * E / G, (q + 1) * E / G) (and so the simulated ranks that host them)
 * and every GPU is one source of its own bs tokens.  The rows of the group
 * are then exactly those of moe_dispatch with sources = G on one GPU,
 * ordered by (instance, source GPU, token, k); GPU q's receive buffer holds
 * the stretch of that order its instances own, so its row r is global row
 * base[q] + r.
 *
 * A layer on GPU g, fused form:
 *   1. moe_update_expert and moe_dispatch_route on its own tokens over all E
 *      instances (local rows, counts [E], offsets [E+1]; no row moved);
 *   2. the counts of every GPU gathered into counts_all [G][E] on every GPU
 *      (a collective of E ints per GPU, by the caller);
 *   3. moe_ep_plan, then moe_ep_dispatch: each token is quantized once and
 *      each copy (and its scales) stored straight into its owner's receive
 *      buffer through the owner's pointer;
 *   4. a group barrier (every row stored), then the expert step on the
 *      receive buffer (moe_ep_plan's recv_counts / recv_offsets describe it);
 *   5. a group barrier (every expert output written), then
 *      moe_ep_combine_add_rmsnorm: each copy's output read from its owner;
 *   6. a group barrier before the buffers are reused.
 * Two-step form: moe_dispatch into a local buffer in step 1, moe_ep_push in
 * step 3 (every local row stored into its owner's buffer), and in step 5
 * moe_ep_pull (each local row's output brought back in the local row order)
 * followed by moe_combine_add_rmsnorm with the local expand_idx.
 * The pointer tables hold, per GPU q, a pointer this GPU can dereference:
 * its own buffer for q = g, a peer mapping (moe_ipc_import, or any mapping
 * the caller set up) otherwise.  The copies are plain 16-byte loads and
 * stores by the SMs over NVLink; no TMA load reads peer memory.  With every
 * pointer in one GPU's memory (G buffers of one device), the calls emulate a
 * group of G on one GPU.
 */

#define MOE_EP_MAX_GPUS       64
#define MOE_IPC_HANDLE_BYTES  64

typedef struct {
    int32_t bs;             /* tokens of this GPU (one source), (0, 512] */
    int32_t top_k;          /* K, (0, 16] */
    int32_t num_instances;  /* E over the whole group, (0, 1024], a multiple of gpus */
    int32_t gpus;           /* G, [1, MOE_EP_MAX_GPUS] */
    int32_t rank;           /* this GPU, [0, G) */
    int32_t row_bytes;      /* bytes of one row moved: H for int8 / e4m3 rows, 2H for bf16 rows;
                               a multiple of 16 */
    int32_t scale_bytes;    /* bytes of one row's scales: 0 (quant modes 0, 1), 4 (2),
                               4 * ceil(H / 128) (3), H / 32 (4); push only */
    int32_t recv_rows;      /* rows of every GPU's receive (and expert output) buffer, >= 0 */
} moe_ep_params;

/* Workspace of the plan / push / pull calls of one layer (they share it:
 * the plan is stored there), 16-byte aligned, zeroed once. */
MOE_API moe_status moe_ep_workspace_size(const moe_ep_params *p, size_t *bytes);

/*
 * From the gathered counts, the global row of this GPU's first copy of
 * every instance (kept in the workspace for push and pull), and this GPU's
 * receive layout:
 *   counts_all    [G][E] int32 device: row g' = moe_dispatch's expert_counts on GPU g'
 *   recv_counts   [E/G]   int32 device, out: rows this GPU receives per own instance
 *   recv_offsets  [E/G+1] int32 device, out: their exclusive prefix; [E/G] = rows received
 * Device errors: more rows than recv_rows sets MOE_DEV_CAPACITY (push and
 * pull then drop the rows beyond it).
 */
MOE_API moe_status moe_ep_plan(const moe_ep_params *p, const int32_t *counts_all, int32_t *recv_counts,
                               int32_t *recv_offsets, void *workspace, size_t workspace_bytes, void *cuda_stream);

/*
 * Stores this GPU's dispatched rows into their owners' receive buffers:
 *   local_rows     [bs*K, row_bytes] device: moe_dispatch's expand_x
 *   local_scales   [bs*K, scale_bytes] device: its dyn_scales (NULL when scale_bytes = 0)
 *   local_offsets  [E+1], src_of_row [bs*K], expand_idx [bs, K], instance_ids [bs, K]:
 *                  moe_dispatch's outputs and its instance ids
 *   peer_rows      [G] device array of pointers: receive buffers, [recv_rows, row_bytes] each
 *   peer_scales    [G] device array of pointers, [recv_rows, scale_bytes] each (NULL when scale_bytes = 0)
 *   peer_src       [G] device array of pointers, optional: [recv_rows] int32 each,
 *                  receives every row's copy id in the group, (g * bs + i) * K + k
 *   global_idx     [bs, K] int32 device, out: every copy's global row (-1 if not sent)
 */
MOE_API moe_status moe_ep_push(const moe_ep_params *p, const void *local_rows, const void *local_scales,
                               const int32_t *local_offsets, const int32_t *src_of_row, const int32_t *expand_idx,
                               const int32_t *instance_ids, void *const *peer_rows, void *const *peer_scales,
                               int32_t *const *peer_src, int32_t *global_idx, void *workspace,
                               size_t workspace_bytes, void *cuda_stream);

/*
 * Brings every local row's expert output back from its owner:
 *   peer_rows   [G] device array of pointers: expert output buffers, [recv_rows, row_bytes] each
 *   local_offsets [E+1] int32 device: moe_dispatch's offsets on this GPU
 *   local_rows  [bs*K, row_bytes] device, out: the outputs in local row order
 *               (rows >= local_offsets[E] untouched)
 */
MOE_API moe_status moe_ep_pull(const moe_ep_params *p, void *const *peer_rows, const int32_t *local_offsets,
                               void *local_rows, void *workspace, size_t workspace_bytes, void *cuda_stream);

/*
 * Steps 1 and 3 fused: the rows are quantized once and stored straight into
 * their owners' receive buffers (no local expand_x), after moe_dispatch_route
 * and moe_ep_plan of the same layer on this GPU:
 *   p              the moe_dispatch parameters of the route call (sources = 1;
 *                  bs, top_k and num_instances equal to the EP parameters')
 *   x, instance_ids, mask, smooth_scales: as moe_dispatch
 *   expand_idx, expert_offsets: moe_dispatch_route's outputs
 *   peer_rows, peer_scales, peer_src, global_idx: as moe_ep_push (row_bytes
 *                  must be the mode's row size, scale_bytes its scale size)
 *   ep_workspace   the EP workspace the plan wrote
 * The receive buffers hold, row for row, what moe_dispatch with sources = G
 * writes on one GPU.  Host errors: MOE_ERR_INVALID_ARG for parameters that do
 * not agree or NULL / misaligned pointers, MOE_ERR_WORKSPACE.  Device errors
 * (in the EP workspace): MOE_DEV_BAD_ID for out-of-range ids or a plan that
 * does not match the routing, MOE_DEV_CAPACITY for rows past recv_rows
 * (dropped).
 */
MOE_API moe_status moe_ep_dispatch(const moe_dispatch_params *p, const moe_ep_params *ep, const void *x,
                                   const int32_t *instance_ids, const uint8_t *mask, const float *smooth_scales,
                                   const int32_t *expand_idx, const int32_t *expert_offsets,
                                   void *const *peer_rows, void *const *peer_scales, int32_t *const *peer_src,
                                   int32_t *global_idx, void *ep_workspace, size_t ep_workspace_bytes,
                                   void *cuda_stream);

/*
 * Steps 5 and the combine fused: moe_combine_add_rmsnorm whose top-K rows are
 * read from the GPUs that own them: copy (i, k) with global row
 * g = global_idx[i*K + k] reads row g - base[q] of peer_rows[q], q the owner
 * of g (the plan's base), through a plain load over NVLink.
 *   p           the combine parameters (sources = 1; bs and top_k equal to the EP parameters')
 *   ep          row_bytes = 2H (bf16 expert outputs)
 *   peer_rows   [G] device array of pointers: expert output buffers, [recv_rows, H] bf16 each
 *   global_idx  [bs, K] int32 device: moe_ep_dispatch's (or moe_ep_push's) output
 *   expert_scales, shared_x, residual_x, gamma, y, x_out, rstd_out: as moe_combine_add_rmsnorm
 * Errors as moe_combine_add_rmsnorm; device errors go to the EP workspace
 * (MOE_DEV_BAD_ID for a global row outside the group's rows).
 */
MOE_API moe_status moe_ep_combine_add_rmsnorm(const moe_combine_params *p, const moe_ep_params *ep,
                                              void *const *peer_rows, const int32_t *global_idx,
                                              const float *expert_scales, const void *shared_x,
                                              const void *residual_x, const void *gamma, void *y, void *x_out,
                                              float *rstd_out, void *ep_workspace, size_t ep_workspace_bytes,
                                              void *cuda_stream);

/*
 * Peer mappings for the pointer tables (CUDA IPC, no multicast object):
 * moe_ipc_export writes a MOE_IPC_HANDLE_BYTES handle (host memory) for the
 * device allocation that holds dev_ptr and dev_ptr's offset in it; another
 * process on the same node maps it with moe_ipc_import (base = the mapping to
 * give moe_ipc_close later, dev_ptr = base + offset).  The exporter keeps the
 * allocation alive until every importer has closed it.
 */
MOE_API moe_status moe_ipc_export(const void *dev_ptr, void *handle, uint64_t *offset);
MOE_API moe_status moe_ipc_import(const void *handle, uint64_t offset, void **base, void **dev_ptr);
MOE_API moe_status moe_ipc_close(void *base);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
