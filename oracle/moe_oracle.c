/*
 * moe_oracle.c -- plain CPU oracle for MoE update-expert / dispatch /
 * combine+Add+RMSNorm.  TEST INFRASTRUCTURE ONLY (see moe_oracle.h): the
 * product never links or calls it.
 *
 * Written as the definitions read, loop by loop, with no blocking, fusion
 * or reordering.  Quantization runs in IEEE binary32 because the dispatch
 * page fixes it (CastToFp32); combine runs in binary64.  Build with
 * -O2 -fno-fast-math -ffp-contract=off so every float operation is one
 * correctly rounded IEEE operation.
 *
 * Readings where the pages are silent or garbled are marked READING(Rn);
 * the same numbering is used in the design notes.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORC_MAX_INSTANCES 1024 /* aclnnMoeUpdateExpert: total instances <= 1024 */

/* ---------------------------------------------------------------------- */
/* scalar helpers                                                          */
/* ---------------------------------------------------------------------- */

/* bf16 is the top half of a binary32: widening is exact. */
static float bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a double to the nearest bf16 (ties to even).  bf16 keeps 8
 * significant bits; below 2^-126 its grid is fixed at 2^-133. */
uint16_t orc_bf16_from_double(double v) {
    if (isnan(v)) return 0x7FC0;
    uint16_t s = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (a == 0.0) return s;
    int e;
    (void)frexp(a, &e);             /* a = m * 2^e, m in [0.5, 1) */
    int lsb = e - 8;                /* weight of the last kept bit */
    if (lsb < -133) lsb = -133;
    double q = rint(ldexp(a, -lsb)); /* exact scaling, then round half to even */
    double r = ldexp(q, lsb);
    if (r > 3.3895313892515355e38) return s | 0x7F80; /* past the largest bf16 */
    float f = (float)r;             /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return s | (uint16_t)((u >> 16) & 0x7FFF);
}

/* OCP FP8 E4M3 ("fn" variant): 1 sign, 4 exponent bits (bias 7), 3 mantissa
 * bits, no infinities, S.1111.111 = NaN, largest finite 1.75 * 2^8 = 448,
 * smallest normal 2^-6, subnormal step 2^-9.  Round to nearest even; values
 * beyond 448 saturate to +-448 (READING R12). */
uint8_t orc_e4m3_encode(float v) {
    uint8_t s = signbit(v) ? 0x80 : 0;
    if (isnan(v)) return s | 0x7F;
    float a = fabsf(v);
    if (a >= 448.0f) return s | 0x7E;
    if (a < 0.015625f) {                 /* subnormal range: multiples of 2^-9 */
        float m = rintf(a * 512.0f);     /* exact scaling; m in 0..8 (8 = 2^-6) */
        return s | (uint8_t)m;
    }
    int e;
    float fr = frexpf(a, &e);            /* a = fr * 2^e, fr in [0.5, 1) */
    int E = e - 1;                       /* a = (2 fr) * 2^E, 2 fr in [1, 2) */
    float m = rintf((2.0f * fr - 1.0f) * 8.0f); /* 3 fraction bits, RNE */
    if (m == 8.0f) { m = 0.0f; E += 1; }
    if (E > 8) return s | 0x7E;
    return s | (uint8_t)(((E + 7) << 3) | (int)m);
}

/* The value of an E4M3 ("fn") code: S.EEEE.MMM, exponent bias 7; E = 0 is
 * subnormal (M * 2^-9); S.1111.111 is NaN; no infinities. */
double orc_e4m3_decode(uint8_t c) {
    const int s = c >> 7, E = (c >> 3) & 15, M = c & 7;
    if (E == 15 && M == 7) return NAN;
    double v = E == 0 ? ldexp((double)M, -9) : ldexp(1.0 + M / 8.0, E - 7);
    return s ? -v : v;
}

/* ---------------------------------------------------------------------- */
/* Step 1: aclnnMoeUpdateExpert                                            */
/* ---------------------------------------------------------------------- */

/*
 * Mapping table [num_logical, table_cols]: column 0 = number of deployed
 * instances n_e (> 0), columns 1..n_e = the rank hosting each instance
 * ("Restriction on the shape format").  All instances together <= 1024 and
 * every rank hosts the same number L of them.
 *
 * READING R3: the output id is the deployed-instance id
 *   inst(e, j) = rank(e, j) * L + slot(e, j),
 * where slot(e, j) counts the instances of the same rank that come before
 * (e, j) in (e, j) order.  So rank = inst / L.
 * READING R2 (the page's formula is lost): token i uses replica
 * j = i mod n_e.
 * READING R4: a copy is pruned when its token's mask entry is false (the
 * (Bs,) mask broadcast to (Bs,K)) or when its expertScales entry is
 * strictly below the threshold.
 */
uint32_t orc_update_expert(int32_t bs, int32_t top_k, int32_t num_logical,
                           int32_t table_cols, int32_t ep_world_size,
                           const int32_t *expert_ids, const float *expert_scales,
                           const uint8_t *active_mask, float prune_threshold,
                           const int32_t *table,
                           int32_t *balanced_ids, uint8_t *balanced_mask) {
    uint32_t err = 0;
    const int F = table_cols;

    /* enumerate the instances (e, j) in (e, j) order and check the table */
    int valid = num_logical > 0 && ep_world_size > 0;
    int total = 0;
    for (int e = 0; valid && e < num_logical; ++e) {
        int n = table[(size_t)e * F];
        if (n < 1 || n > F - 1) { valid = 0; break; }
        for (int j = 0; j < n; ++j) {
            int r = table[(size_t)e * F + 1 + j];
            if (r < 0 || r >= ep_world_size) valid = 0;
        }
        total += n;
    }
    if (valid && (total > ORC_MAX_INSTANCES || total % ep_world_size != 0)) valid = 0;

    int *first = NULL, *inst = NULL, *per_rank = NULL;
    if (valid) {
        int L = total / ep_world_size;
        first = (int *)calloc((size_t)num_logical, sizeof(int));
        inst = (int *)calloc((size_t)total, sizeof(int));
        per_rank = (int *)calloc((size_t)ep_world_size, sizeof(int));
        int pos = 0;
        for (int e = 0; e < num_logical; ++e) {
            first[e] = pos;
            int n = table[(size_t)e * F];
            for (int j = 0; j < n; ++j) {
                int r = table[(size_t)e * F + 1 + j];
                int slot = per_rank[r]++;          /* earlier instances on rank r */
                inst[pos++] = r * L + slot;
            }
        }
        for (int r = 0; r < ep_world_size; ++r)
            if (per_rank[r] != L) valid = 0;     /* equal instances per rank */
    }

    for (int i = 0; i < bs; ++i) {
        for (int k = 0; k < top_k; ++k) {
            size_t ik = (size_t)i * top_k + k;
            if (!valid) {
                balanced_ids[ik] = -1;
                balanced_mask[ik] = 0;
                continue;
            }
            int e = expert_ids[ik];
            if (e < 0 || e >= num_logical) {
                err |= ORC_ERR_BAD_ID;
                balanced_ids[ik] = -1;
                balanced_mask[ik] = 0;
                continue;
            }
            int n = table[(size_t)e * F];
            int j = i % n;
            balanced_ids[ik] = inst[first[e] + j];
            int keep = active_mask ? (active_mask[i] != 0) : 1;
            if (expert_scales && prune_threshold > 0.0f && expert_scales[ik] < prune_threshold)
                keep = 0;
            balanced_mask[ik] = (uint8_t)keep;
        }
    }
    if (!valid) err |= ORC_ERR_BAD_TABLE;
    free(first);
    free(inst);
    free(per_rank);
    return err;
}

/* ---------------------------------------------------------------------- */
/* Step 2: aclnnMoeDistributeDispatchV2                                    */
/* ---------------------------------------------------------------------- */

typedef struct { int32_t id, i, k; } orc_item;

/* READING R15: rows are ordered by (instance, token i, k); instance ids are
 * rank-major, so each simulated rank's rows form one contiguous region. */
static int orc_item_cmp(const void *pa, const void *pb) {
    const orc_item *a = (const orc_item *)pa, *b = (const orc_item *)pb;
    if (a->id != b->id) return a->id < b->id ? -1 : 1;
    if (a->i != b->i) return a->i < b->i ? -1 : 1;
    if (a->k != b->k) return a->k < b->k ? -1 : 1;
    return 0;
}

/* Case 3 / case 4 (quantMode 2, 3): on one segment of a row,
 *   xFp32 = CastToFp32(X) * scales
 *   dynamicScales = dstTypeMax / Max(Abs(xFp32))
 *   quantOut = CastToInt8(xFp32 * dynamicScales)
 *   sent scale = 1.0 / dynamicScales
 * READING R6: dstTypeMax = 127, CastToInt8 rounds half to even and clamps to
 * [-127, 127].  READING R7: the sent scale is the fp32 quotient 1 / dyn.
 * READING R13: an all-zero segment gives codes 0 and scale 1/inf = 0.
 * READING R20: when 127 / amax overflows fp32 (amax < 127 / FLT_MAX) the
 * formula runs on dyn = +inf: CastToInt8 saturates +-inf to +-127 and maps the
 * NaN of 0 * inf to 0; the scale is again 1/inf = 0. */
static void orc_quant_int8_segment(const uint16_t *x, const float *smooth, int len,
                                   int8_t *q, float *scale_out) {
    float amax = 0.0f;
    for (int h = 0; h < len; ++h) {
        float xf = bf16_to_float(x[h]);
        if (smooth) xf = xf * smooth[h];
        float a = fabsf(xf);
        if (a > amax) amax = a;
    }
    float dyn = 127.0f / amax;           /* +inf when amax == 0 */
    *scale_out = 1.0f / dyn;
    for (int h = 0; h < len; ++h) {
        if (amax == 0.0f) { q[h] = 0; continue; }
        float xf = bf16_to_float(x[h]);
        if (smooth) xf = xf * smooth[h];
        float r = rintf(xf * dyn);
        if (isnan(r)) r = 0.0f;
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        q[h] = (int8_t)r;
    }
}

/* Case 5 (quantMode 4, mxfp8), on one 32-element block:
 *   sharedExp = Floor(log2(max(x))) - emax
 *   dynamicScales = 2^sharedExp
 *   quantOut = CastToFp8(X / dynamicScales)
 * READING R10: max over |x| of the block, e4m3 with emax = 8.
 * READING R11: the scale sent is the dequantization factor 2^sharedExp as
 * an E8M0 byte (sharedExp + 127), sharedExp clamped to [-127, 127]; an
 * all-zero block uses sharedExp = -127 (byte 0). */
static void orc_quant_mxfp8_block(const uint16_t *x, int len, uint8_t *q, uint8_t *e8m0) {
    float amax = 0.0f;
    for (int h = 0; h < len; ++h) {
        float a = fabsf(bf16_to_float(x[h]));
        if (a > amax) amax = a;
    }
    int se = -127;
    if (amax > 0.0f) {
        int e;
        (void)frexpf(amax, &e);          /* amax = m * 2^e, m in [0.5,1): floor(log2) = e-1 */
        se = (e - 1) - ORC_E4M3_EMAX;
        if (se < -127) se = -127;
        if (se > 127) se = 127;
    }
    *e8m0 = (uint8_t)(se + 127);
    float dyn = ldexpf(1.0f, se);        /* exact power of two */
    for (int h = 0; h < len; ++h)
        q[h] = orc_e4m3_encode(bf16_to_float(x[h]) / dyn);
}

/* Case 2 (quantMode 1, static quantization), one element:
 *   xFp32 = CastToFp32(X) * scales
 *   quantOut = Cast(xFp32, dstType)
 * READING R21: dstType is int8 and Cast rounds half to even, then saturates
 * to the int8 range [-128, 127]; a NaN product (0 * inf) casts to 0.  The
 * scales are one coefficient (1,), one per column (H,), or one row per
 * destination instance (E, H); nothing is sent besides the codes. */
static int8_t orc_static_int8(float xf) {
    float r = rintf(xf);
    if (isnan(r)) return 0;
    if (r > 127.0f) r = 127.0f;
    if (r < -128.0f) r = -128.0f;
    return (int8_t)r;
}

uint32_t orc_dispatch(int32_t bs, int32_t hidden, int32_t top_k,
                      int32_t num_instances, int32_t quant_mode,
                      const uint16_t *x_bf16, const int32_t *instance_ids,
                      const uint8_t *mask, const float *smooth, int64_t scales_len,
                      void *expand_x, void *dyn_scales,
                      int32_t *expand_idx, int32_t *src_of_row,
                      int32_t *expert_counts, int32_t *expert_offsets) {
    uint32_t err = 0;
    const int H = hidden;
    orc_item *items = (orc_item *)malloc(sizeof(orc_item) * (size_t)(bs * top_k + 1));
    int n = 0;

    /* the active copies: a 2-D mask entry of false means "not sent" */
    for (int i = 0; i < bs; ++i) {
        for (int k = 0; k < top_k; ++k) {
            size_t ik = (size_t)i * top_k + k;
            expand_idx[ik] = -1;
            if (mask && !mask[ik]) continue;
            int id = instance_ids[ik];
            if (id < 0 || id >= num_instances) { err |= ORC_ERR_BAD_ID; continue; }
            items[n].id = id;
            items[n].i = i;
            items[n].k = k;
            ++n;
        }
    }
    qsort(items, (size_t)n, sizeof(orc_item), orc_item_cmp);

    for (int e = 0; e < num_instances; ++e) expert_counts[e] = 0;
    for (int r = 0; r < n; ++r) {
        expert_counts[items[r].id] += 1;
        expand_idx[(size_t)items[r].i * top_k + items[r].k] = r;
        src_of_row[r] = items[r].i * top_k + items[r].k;
    }
    expert_offsets[0] = 0;
    for (int e = 0; e < num_instances; ++e) expert_offsets[e + 1] = expert_offsets[e] + expert_counts[e];

    /* the values of each received row: AllToAllV is a pure permutation here */
    const int tiles = (H + 127) / 128;
    for (int r = 0; r < n; ++r) {
        const uint16_t *xr = x_bf16 + (size_t)items[r].i * H;
        const float *sm = smooth ? smooth + (size_t)items[r].id * H : NULL; /* READING R9 */
        if (quant_mode == 0) {
            memcpy((uint16_t *)expand_x + (size_t)r * H, xr, sizeof(uint16_t) * (size_t)H);
        } else if (quant_mode == 1) {
            int8_t *q = (int8_t *)expand_x + (size_t)r * H;
            for (int h = 0; h < H; ++h) {
                float s;
                if (scales_len == 1) s = smooth[0];
                else if (scales_len == H) s = smooth[h];
                else s = smooth[(size_t)items[r].id * H + h];
                q[h] = orc_static_int8(bf16_to_float(xr[h]) * s);
            }
        } else if (quant_mode == 2) {
            orc_quant_int8_segment(xr, sm, H, (int8_t *)expand_x + (size_t)r * H,
                                   (float *)dyn_scales + r);
        } else if (quant_mode == 3) {
            for (int t = 0; t < tiles; ++t) {      /* READING R8: 128-element tiles */
                int h0 = t * 128;
                int len = H - h0 < 128 ? H - h0 : 128;
                orc_quant_int8_segment(xr + h0, sm ? sm + h0 : NULL, len,
                                       (int8_t *)expand_x + (size_t)r * H + h0,
                                       (float *)dyn_scales + (size_t)r * tiles + t);
            }
        } else if (quant_mode == 4) {
            for (int b = 0; b < H / 32; ++b)
                orc_quant_mxfp8_block(xr + b * 32, 32, (uint8_t *)expand_x + (size_t)r * H + b * 32,
                                      (uint8_t *)dyn_scales + (size_t)r * (H / 32) + b);
        }
    }
    free(items);
    return err;
}

/* ---------------------------------------------------------------------- */
/* Step 3: aclnnMoeDistributeCombineAddRmsNorm                             */
/* ---------------------------------------------------------------------- */

/*
 *   ataOut     = AllToAllV(expandX)       (here: row expand_idx[i][k])
 *   combineOut = Sum_k(expertScales * ataOut + expertScales * sharedExpertX)
 *   x          = combineOut + residualX
 *   y          = x / RMS(x) * gamma,  RMS(x) = sqrt(1/H * Sum_h x_h^2 + normEps)
 * READING R5: the formula is taken literally, so the shared-expert row is
 * weighted by every kept copy's scale.  READING R19: a pruned copy
 * (expand_idx == -1) contributes nothing.  READING R14: eps sits inside the
 * square root; y and x are rounded to bf16 only at the end.
 */
void orc_combine_add_rmsnorm(int32_t bs, int32_t hidden, int32_t top_k,
                             const uint16_t *expand_x_bf16, const int32_t *expand_idx,
                             const float *expert_scales, const uint16_t *shared_x,
                             const uint16_t *residual_x, const uint16_t *gamma,
                             double norm_eps,
                             uint16_t *y_bf16, uint16_t *x_out_bf16, float *rstd,
                             double *y_f64, double *x_f64) {
    const int H = hidden;
    double *x = (double *)malloc(sizeof(double) * (size_t)H);
    for (int i = 0; i < bs; ++i) {
        for (int h = 0; h < H; ++h) {
            double c = 0.0;
            for (int k = 0; k < top_k; ++k) {
                int row = expand_idx[(size_t)i * top_k + k];
                if (row < 0) continue;
                double s = (double)expert_scales[(size_t)i * top_k + k];
                double ata = (double)bf16_to_float(expand_x_bf16[(size_t)row * H + h]);
                double sh = shared_x ? (double)bf16_to_float(shared_x[(size_t)i * H + h]) : 0.0;
                c += s * ata + s * sh;
            }
            x[h] = c + (double)bf16_to_float(residual_x[(size_t)i * H + h]);
        }
        double ss = 0.0;
        for (int h = 0; h < H; ++h) ss += x[h] * x[h];
        double rms = sqrt(ss / H + norm_eps);
        if (rstd) rstd[i] = (float)(1.0 / rms);
        for (int h = 0; h < H; ++h) {
            double y = x[h] / rms * (double)bf16_to_float(gamma[h]);
            if (y_bf16) y_bf16[(size_t)i * H + h] = orc_bf16_from_double(y);
            if (y_f64) y_f64[(size_t)i * H + h] = y;
            if (x_out_bf16) x_out_bf16[(size_t)i * H + h] = orc_bf16_from_double(x[h]);
            if (x_f64) x_f64[(size_t)i * H + h] = x[h];
        }
    }
    free(x);
}

/* The plain combine paired with the dispatch (the CombineV2 series named on
 * the dispatch page; READING R23): the first line of the formula above and
 * nothing after it,
 *   combineOut = Sum_k(expertScales * ataOut + expertScales * sharedExpertX),
 * rounded to bf16 once. */
void orc_combine(int32_t bs, int32_t hidden, int32_t top_k,
                 const uint16_t *expand_x_bf16, const int32_t *expand_idx,
                 const float *expert_scales, const uint16_t *shared_x,
                 uint16_t *out_bf16, double *out_f64) {
    const int H = hidden;
    for (int i = 0; i < bs; ++i) {
        for (int h = 0; h < H; ++h) {
            double c = 0.0;
            for (int k = 0; k < top_k; ++k) {
                int row = expand_idx[(size_t)i * top_k + k];
                if (row < 0) continue;
                double s = (double)expert_scales[(size_t)i * top_k + k];
                double ata = (double)bf16_to_float(expand_x_bf16[(size_t)row * H + h]);
                double sh = shared_x ? (double)bf16_to_float(shared_x[(size_t)i * H + h]) : 0.0;
                c += s * ata + s * sh;
            }
            if (out_bf16) out_bf16[(size_t)i * H + h] = orc_bf16_from_double(c);
            if (out_f64) out_f64[(size_t)i * H + h] = c;
        }
    }
}

/* ---------------------------------------------------------------------- */
/* Between dispatch and combine: the instances' grouped matmul             */
/* ---------------------------------------------------------------------- */

/*
 * READING R24.  The pages name the expert step only by its place, between
 * the dispatch and the combine ("AllToAllV" out and back), and do not define
 * it.  Taken here as the one contraction that consumes the dispatch's output:
 * deployed instance e applies its own weight to the rows it received,
 * rows [expert_offsets[e], expert_offsets[e+1]) of expand_x.  The rows hold
 * int8 codes q with one dequantization factor each (quantMode 2:
 * x ~= q * dyn_scale); the weight is int8 w with one factor per output
 * channel (W[e][n][h] ~= w[e][n][h] * w_scale[e][n]).  Then
 *   acc[r][n] = Sum_h q[r][h] * w[e][n][h]            (an exact integer)
 *   out[r][n] = acc[r][n] * dyn_scale[r] * w_scale[e][n],  rounded to bf16 once.
 * Offsets must satisfy 0 <= off[0] <= ... <= off[E] <= rows; otherwise
 * nothing is written and ORC_ERR_BAD_ID is returned.  Rows outside
 * [off[0], off[E]) are not written.
 */
uint32_t orc_grouped_matmul(int32_t rows, int32_t hidden, int32_t out_dim, int32_t num_instances,
                            const int8_t *expand_x, const float *dyn_scales,
                            const int32_t *expert_offsets, const int8_t *weight,
                            const float *weight_scales, uint16_t *out_bf16, double *out_f64) {
    const int H = hidden, N = out_dim, E = num_instances;
    if (expert_offsets[0] < 0 || expert_offsets[E] > rows) return ORC_ERR_BAD_ID;
    for (int e = 0; e < E; ++e)
        if (expert_offsets[e + 1] < expert_offsets[e]) return ORC_ERR_BAD_ID;
    for (int e = 0; e < E; ++e) {
        const int8_t *w = weight + (size_t)e * N * H;
        for (int r = expert_offsets[e]; r < expert_offsets[e + 1]; ++r) {
            const int8_t *q = expand_x + (size_t)r * H;
            for (int n = 0; n < N; ++n) {
                int64_t acc = 0;
                for (int h = 0; h < H; ++h) acc += (int64_t)q[h] * (int64_t)w[(size_t)n * H + h];
                double v = (double)acc * (double)dyn_scales[r] * (double)weight_scales[(size_t)e * N + n];
                if (out_bf16) out_bf16[(size_t)r * N + n] = orc_bf16_from_double(v);
                if (out_f64) out_f64[(size_t)r * N + n] = v;
            }
        }
    }
    return 0;
}

/*
 * The same step on mxfp8 rows (quantMode 4, READING R24): the rows are E4M3
 * codes with one E8M0 factor 2^(b - 127) per 32-element block
 * (x_sf [rows, H/32], the dispatch's dynamicScales bytes), and so is the
 * weight (weight_sf [E, N, H/32]):
 *   out[r][n] = Sum_j 2^(x_sf[r][j] - 127) 2^(weight_sf[e][n][j] - 127) Sum_{h in block j} dec(q[r][h]) dec(w[e][n][h])
 * summed in binary64 and rounded to bf16 once.  Each block's sum is exact in
 * binary64 (32 products of two E4M3 values: multiples of 2^-18 below 2^18)
 * and the factors are powers of two, so only the sum over blocks rounds.
 * Offsets as above.
 */
uint32_t orc_grouped_matmul_mx(int32_t rows, int32_t hidden, int32_t out_dim, int32_t num_instances,
                               const uint8_t *expand_x, const uint8_t *x_sf,
                               const int32_t *expert_offsets, const uint8_t *weight,
                               const uint8_t *weight_sf, uint16_t *out_bf16, double *out_f64) {
    const int H = hidden, N = out_dim, E = num_instances, B = hidden / 32;
    if (expert_offsets[0] < 0 || expert_offsets[E] > rows) return ORC_ERR_BAD_ID;
    for (int e = 0; e < E; ++e)
        if (expert_offsets[e + 1] < expert_offsets[e]) return ORC_ERR_BAD_ID;
    double dec[256];  /* the value of every code */
    for (int c = 0; c < 256; ++c) dec[c] = orc_e4m3_decode((uint8_t)c);
    for (int e = 0; e < E; ++e) {
        for (int r = expert_offsets[e]; r < expert_offsets[e + 1]; ++r) {
            const uint8_t *q = expand_x + (size_t)r * H;
            for (int n = 0; n < N; ++n) {
                const size_t wr = (size_t)e * N + n;
                const uint8_t *w = weight + wr * H;
                double acc = 0.0;
                for (int j = 0; j < B; ++j) {
                    double blk = 0.0;
                    for (int h = 32 * j; h < 32 * j + 32; ++h) blk += dec[q[h]] * dec[w[h]];
                    acc += ldexp(blk, (int)x_sf[(size_t)r * B + j] + (int)weight_sf[wr * B + j] - 254);
                }
                if (out_bf16) out_bf16[(size_t)r * N + n] = orc_bf16_from_double(acc);
                if (out_f64) out_f64[(size_t)r * N + n] = acc;
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* TP domain of two ranks (READING R26)                                    */
/* ---------------------------------------------------------------------- */

/* AllGatherV over the TP pair (dispatch page, 计算公式): both TP ranks of EP
 * rank e end with the rows each of them received from its own EP domain,
 * domain 0's first.  With one instance per rank the ranks are the
 * instances, taken in order. */
void orc_tp_allgather(int32_t num_instances, int64_t row_bytes, const uint8_t *d0, const int32_t *off0,
                      const uint8_t *d1, const int32_t *off1, uint8_t *out, int32_t *map0, int32_t *map1,
                      int32_t *tp_counts) {
    int64_t o = 0;
    for (int32_t e = 0; e < num_instances; ++e) {
        for (int t = 0; t < 2; ++t) {
            const uint8_t *d = t ? d1 : d0;
            const int32_t *off = t ? off1 : off0;
            int32_t *map = t ? map1 : map0;
            for (int32_t r = off[e]; r < off[e + 1]; ++r, ++o) {
                if (row_bytes > 0) memcpy(out + o * row_bytes, d + (int64_t)r * row_bytes, (size_t)row_bytes);
                if (map) map[r] = (int32_t)o;
            }
            if (tp_counts) tp_counts[2 * e + t] = off[e + 1] - off[e];
        }
    }
}

/* ReduceScatterV over the TP pair (combine page, 计算公式): the sum of the two
 * partial bf16 outputs of a row, exact in binary64, rounded once to bf16. */
void orc_tp_reduce(int64_t n, const uint16_t *p0, const uint16_t *p1, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_bf16_from_double((double)bf16_to_float(p0[i]) + (double)bf16_to_float(p1[i]));
}
