/*
 * moe_oracle.h -- plain, slow, obviously-correct CPU oracle for the MoE
 * update-expert / dispatch / combine+Add+RMSNorm path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library includes,
 * links or calls this code; only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark do.  It shares no code, header, table
 * or helper with the CUDA path.
 *
 * Sources (the operator pages this follows):
 *   [UE]  aclnnMoeUpdateExpert -- description (load balancing, expert
 *         pruning) and "Restriction on the shape format" (mapping table).
 *   [DV2] aclnnMoeDistributeDispatchV2 -- 计算公式 (formulas), cases 1..5
 *         (quantMode 0..4), and the quantMode constraints section.
 *   [CAR] aclnnMoeDistributeCombineAddRmsNorm -- 计算公式 (formula) and
 *         约束说明 item 4 (shape variables).
 *
 * Conventions: all arrays are row-major, host memory, caller-owned.
 * bf16 values travel as their raw 16-bit patterns (uint16_t).
 * Return values are bit masks of ORC_ERR_* (0 = clean).
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORC_ERR_BAD_ID    1u  /* an expert / instance id outside its range: item dropped */
#define ORC_ERR_BAD_TABLE 2u  /* mapping table violates its restrictions: every item dropped */

/* Largest fp8 e4m3 finite value and the exponent of its leading bit
 * (448 = 1.75 * 2^8), used by quantMode 4. */
#define ORC_E4M3_EMAX 8

/* Step 1: logical expert -> deployed instance, plus pruning.  [UE]
 * expert_scales and active_mask may be NULL.  prune_threshold <= 0 (or
 * expert_scales == NULL) disables threshold pruning. */
uint32_t orc_update_expert(int32_t bs, int32_t top_k, int32_t num_logical,
                           int32_t table_cols, int32_t ep_world_size,
                           const int32_t *expert_ids, const float *expert_scales,
                           const uint8_t *active_mask, float prune_threshold,
                           const int32_t *table,
                           int32_t *balanced_ids, uint8_t *balanced_mask);

/* Step 2: order the active (token, k) copies by destination instance and
 * quantize / copy them into the expert-major receive buffer.  [DV2]
 * quant_mode: 0 none (bf16 copy), 1 static int8, 2 per-token int8,
 * 3 per-128-tile int8, 4 mxfp8 (e4m3, 32-element blocks, E8M0 scale bytes).
 * smooth holds scales_len floats: modes 2/3 the (E, H) smooth scales (or
 * NULL); mode 1 the static scales, (1,), (H,) or (E, H).  mask may be NULL.
 * dyn_scales is ignored for modes 0 and 1. */
uint32_t orc_dispatch(int32_t bs, int32_t hidden, int32_t top_k,
                      int32_t num_instances, int32_t quant_mode,
                      const uint16_t *x_bf16, const int32_t *instance_ids,
                      const uint8_t *mask, const float *smooth, int64_t scales_len,
                      void *expand_x, void *dyn_scales,
                      int32_t *expand_idx, int32_t *src_of_row,
                      int32_t *expert_counts, int32_t *expert_offsets);

/* Step 3: gather, weighted top-K sum plus shared-expert term, residual add
 * and RMSNorm, all in double.  [CAR]
 * shared_x, y_bf16, x_out_bf16, rstd, y_f64, x_f64 may be NULL. */
void orc_combine_add_rmsnorm(int32_t bs, int32_t hidden, int32_t top_k,
                             const uint16_t *expand_x_bf16, const int32_t *expand_idx,
                             const float *expert_scales, const uint16_t *shared_x,
                             const uint16_t *residual_x, const uint16_t *gamma,
                             double norm_eps,
                             uint16_t *y_bf16, uint16_t *x_out_bf16, float *rstd,
                             double *y_f64, double *x_f64);

/* Exposed pieces, so the tests can pin them on their own. */
uint8_t orc_e4m3_encode(float v);   /* round-to-nearest-even, saturating */
uint16_t orc_bf16_from_double(double v); /* round-to-nearest-even */

/* The plain combine (CombineV2 series): combineOut only, no residual and no
 * RMSNorm.  out_bf16 / out_f64 may be NULL. */
void orc_combine(int32_t bs, int32_t hidden, int32_t top_k,
                 const uint16_t *expand_x_bf16, const int32_t *expand_idx,
                 const float *expert_scales, const uint16_t *shared_x,
                 uint16_t *out_bf16, double *out_f64);

/* The instances' grouped matmul between dispatch and combine (READING R24):
 * out[r][n] = (Sum_h q[r][h] * w[e][n][h]) * dyn_scales[r] * weight_scales[e][n]
 * for the rows r of instance e, [expert_offsets[e], expert_offsets[e+1]).
 * expand_x [rows, hidden] int8, weight [E, out_dim, hidden] int8,
 * weight_scales [E, out_dim] f32, out [rows, out_dim].  Returns
 * ORC_ERR_BAD_ID (and writes nothing) for offsets that are not a
 * non-decreasing sequence in [0, rows].  out_bf16 / out_f64 may be NULL. */
uint32_t orc_grouped_matmul(int32_t rows, int32_t hidden, int32_t out_dim, int32_t num_instances,
                            const int8_t *expand_x, const float *dyn_scales,
                            const int32_t *expert_offsets, const int8_t *weight,
                            const float *weight_scales, uint16_t *out_bf16, double *out_f64);

/* The same on mxfp8 rows and weights: E4M3 codes with one E8M0 factor per
 * 32-element block, x_sf [rows, hidden/32], weight_sf [E, out_dim, hidden/32];
 * the sum in binary64, rounded to bf16 once. */
uint32_t orc_grouped_matmul_mx(int32_t rows, int32_t hidden, int32_t out_dim, int32_t num_instances,
                               const uint8_t *expand_x, const uint8_t *x_sf,
                               const int32_t *expert_offsets, const uint8_t *weight,
                               const uint8_t *weight_sf, uint16_t *out_bf16, double *out_f64);
double orc_e4m3_decode(uint8_t c);  /* the value of an E4M3 code (NaN for S.1111.111) */

/* The TP domain of two ranks (READING R26; dispatch page 计算公式
 * expandXOut = AllGatherV(allToAllXOut), combine page 计算公式
 * rsOut = ReduceScatterV(expandX)), for localExpertNum = 1 (instance e is
 * EP rank e):
 * orc_tp_allgather: rank e's gathered rows are [TP domain 0's rows of e ;
 * TP domain 1's rows of e], in rank order.  d0 / d1 are the two domains'
 * AllToAllV outputs (rows of row_bytes, offsets off0 / off1 [E+1]); map0 /
 * map1 receive each domain row's row in out; tp_counts [E][2] the rows of
 * each (rank, domain).
 * orc_tp_reduce: the two TP ranks' partial expert outputs of the same rows,
 * summed exactly and rounded to bf16 (ties to even); the scatter half is
 * each domain reading its own rows. */
void orc_tp_allgather(int32_t num_instances, int64_t row_bytes, const uint8_t *d0, const int32_t *off0,
                      const uint8_t *d1, const int32_t *off1, uint8_t *out, int32_t *map0, int32_t *map1,
                      int32_t *tp_counts);
void orc_tp_reduce(int64_t n, const uint16_t *p0, const uint16_t *p1, uint16_t *out);

#ifdef __cplusplus
}
#endif
#endif
