/*
 * sbl_oracle.c -- plain, slow, obviously-correct CPU oracle of the
 * Sparse-BitLinear layer (Sparse-BitNet, "1.58-bit LLMs are Naturally
 * Friendly to Semi-Structured Sparsity", arXiv 2603.05168).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only tests/, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header or table with the CUDA
 * library; it computes every step straight from the written definitions,
 * one element at a time, in the order the definitions state.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (no FMA contraction, IEEE round-to-nearest-even, no flush-to-zero).
 *
 * Sources (page titles; sections / equations on them):
 *  [P1] paper-graph-ui summary of arXiv 2603.05168, "Sparse-BitNet",
 *       section 3.4 "Ternary Quantization in Sparse-BitNet" (gamma and
 *       RoundClip equations), "N:M Mask Generation", "Composition Order",
 *       "The Dual Straight-Through Estimator", "The Full Sparse-BitLinear
 *       Layer: Forward and Backward Pass".
 *  [P5] paper-graph-ui summary of arXiv 2504.12285, "BitNet b1.58 2B4T",
 *       section 3.4 "Weight Quantization: Absolute Mean", "Activation
 *       Quantization: Per-Token Absmax to 8-Bit Integers", "Inference
 *       Implementation: GPU (Custom CUDA Kernels)" (2-bit packing).
 *
 * Readings where the pages are silent, garbled or at odds (the same
 * R-numbers are used throughout this repository):
 *  R1  sum of |W|: fp64, pairwise tree in flat row-major order, zero-padded
 *      to a power of two (split at the largest power of two below n).
 *  R2  gamma = (float)(S / (double)(d_out*d_in)); no epsilon; gamma == 0
 *      gives W_q = 0 everywhere.
 *  R3  W_q = clamp(rint_half_even(fl32(W / gamma)), -1, 1).
 *  R4  mask: keep rank < n where rank counts strictly larger |W| plus equal
 *      |W| at a lower index (lower index wins ties; -0 ties +0).
 *  R5  the mask ranks the master weights and is applied after ternarisation;
 *      gamma is taken over all weights, masked ones included.
 *  R6  activation: a = max|x|; a == 0 -> q = 0, d = 0; otherwise
 *      r = fl32(127 / a), q = clamp(rint_half_even(fl32(x * r)), -128, 127),
 *      d = fl32(a / 127).
 *  R7  output: c_t = fl32(gamma * d_t), y = fl32(fl32(acc) * c_t), bf16 by
 *      round-to-nearest-even.
 *  R8  Dual-STE backward: identity through mask and quantiser, no clip
 *      window: dX = gamma * dY * W_eff.
 *  R9  dW = dY^T * Xtilde with Xtilde = d_t * q (the forward's operand).
 * The later readings (R10-R24) cover the packed formats, the statistics,
 * the ablation arms, the epilogue and the norm; each function below names
 * the one it follows.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ---------------------------------------------------------------- gamma -- */

/* Pairwise tree sum of |w[lo .. lo+n)| in fp64 (reading R1).  The tree over
 * n leaves is the tree over the next power of two with +0.0 padding; adding
 * +0.0 to a non-negative sum is exact, so the split point is the largest
 * power of two strictly below n. */
static double abs_sum_tree(const float *w, int64_t lo, int64_t n)
{
    if (n <= 0) return 0.0;
    if (n == 1) return fabs((double)w[lo]);
    int64_t h = 1;
    while (h * 2 < n) h *= 2;
    double left = abs_sum_tree(w, lo, h);
    double right = abs_sum_tree(w, lo + h, n - h);
    return left + right;
}

double sbl_oracle_abs_sum(const float *w, int64_t count)
{
    return abs_sum_tree(w, 0, count);
}

/* [P1] 3.4, equation for gamma: mean absolute value over all d_out*d_in
 * weights, masked ones included ([P1] "Composition Order"). */
float sbl_oracle_gamma(const float *w, int64_t d_out, int64_t d_in)
{
    int64_t count = d_out * d_in;
    double s = sbl_oracle_abs_sum(w, count);
    return (float)(s / (double)count);
}

/* ------------------------------------------------------------ ternarise -- */

/* [P1] 3.4 RoundClip equation; Algorithm 2's (w / scale).round().clamp(-1, 1)
 * as restated on [P1]; reading R3. */
void sbl_oracle_ternarize(const float *w, int64_t count, float gamma, int8_t *wq)
{
    for (int64_t i = 0; i < count; ++i) {
        if (gamma == 0.0f) { wq[i] = 0; continue; }
        float r = w[i] / gamma;          /* correctly rounded fp32 division */
        float q = nearbyintf(r);         /* current mode: to nearest, ties even */
        if (q > 1.0f) q = 1.0f;
        if (q < -1.0f) q = -1.0f;
        wq[i] = (int8_t)q;
    }
}

/* ----------------------------------------------------------------- mask -- */

/* [P1] "N:M Mask Generation": per contiguous group of m weights along the
 * input dimension keep the n with the largest |W| of the master weights
 * (reading R5).  Reading R4 for ties. */
void sbl_oracle_nm_mask(const float *w, int64_t d_out, int64_t d_in,
                        int n, int m, uint8_t *mask)
{
    for (int64_t o = 0; o < d_out; ++o) {
        for (int64_t g = 0; g < d_in / m; ++g) {
            const float *grp = w + o * d_in + g * m;
            for (int i = 0; i < m; ++i) {
                float ki = fabsf(grp[i]);
                int rank = 0;
                for (int j = 0; j < m; ++j) {
                    float kj = fabsf(grp[j]);
                    if (kj > ki || (kj == ki && j < i)) rank++;
                }
                mask[o * d_in + g * m + i] = (uint8_t)(rank < n ? 1 : 0);
            }
        }
    }
}

/* [P1] "Composition Order": W_eff = W_q (elementwise) M, the mask applied
 * after ternarisation (reading R5). */
void sbl_oracle_apply_mask(const int8_t *wq, const uint8_t *mask, int64_t count,
                           int8_t *weff)
{
    for (int64_t i = 0; i < count; ++i)
        weff[i] = (int8_t)(mask[i] ? wq[i] : 0);
}

/* ------------------------------------------------- ablation variants -- */

/* Pairwise tree of R1 over the flat row-major array with |w| at kept
 * positions and +0.0 at dropped ones. */
static double abs_sum_tree_masked(const float *w, const uint8_t *mask, int64_t lo, int64_t n)
{
    if (n <= 0) return 0.0;
    if (n == 1) return mask[lo] ? fabs((double)w[lo]) : 0.0;
    int64_t h = 1;
    while (h * 2 < n) h *= 2;
    double left = abs_sum_tree_masked(w, mask, lo, h);
    double right = abs_sum_tree_masked(w, mask, lo + h, n - h);
    return left + right;
}

/* Mask-then-quant ([P1] "Composition Order": W_eff = Q_t(W * M), the scale
 * taken over the surviving weights alone; reading R18): gamma = mean |W|
 * over the kept positions,
 * the sum over the same tree as gamma (zeros at dropped positions) divided
 * by the number of kept positions. */
float sbl_oracle_gamma_survivors(const float *w, const uint8_t *mask, int64_t d_out, int64_t d_in)
{
    int64_t count = d_out * d_in, kept = 0;
    for (int64_t i = 0; i < count; ++i) kept += mask[i] ? 1 : 0;
    if (kept == 0) return 0.0f;
    double s = abs_sum_tree_masked(w, mask, 0, count);
    return (float)(s / (double)kept);
}

/* Mask from the quantized weights ([P1] "Composition Order", "Where the mask
 * is computed"; reading R19): the same top-n rule ranking |W_q| in {0, 1}
 * instead of |W|; ties (nearly all) go to the lower index. */
void sbl_oracle_nm_mask_quantized(const int8_t *wq, int64_t d_out, int64_t d_in, int n, int m, uint8_t *mask)
{
    for (int64_t o = 0; o < d_out; ++o)
        for (int64_t g = 0; g < d_in / m; ++g) {
            const int8_t *grp = wq + o * d_in + g * m;
            for (int i = 0; i < m; ++i) {
                int ki = grp[i] != 0;
                int rank = 0;
                for (int j = 0; j < m; ++j) {
                    int kj = grp[j] != 0;
                    if (kj > ki || (kj == ki && j < i)) rank++;
                }
                mask[o * d_in + g * m + i] = (uint8_t)(rank < n ? 1 : 0);
            }
        }
}

/* -------------------------------------------------------------- packing -- */

/* 2-bit code of a ternary value: {-1, 0, +1} -> {0, 1, 2} ([P5] "Inference
 * Implementation: GPU", packing of four ternaries per byte). */
static uint8_t code_of(int8_t v) { return (uint8_t)(v + 1); }

static int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

int64_t sbl_oracle_pk2_row_bytes(int64_t d_in) { return round_up(d_in / 4, 16); }

/* PK2 (reading R12): weight k of a row at bits 2*(k%4) of byte k/4; padding
 * bytes hold code 1 in every slot (0x55, i.e. zero weights). */
void sbl_oracle_pack_pk2(const int8_t *weff, int64_t d_out, int64_t d_in, uint8_t *out)
{
    int64_t rb = sbl_oracle_pk2_row_bytes(d_in);
    for (int64_t o = 0; o < d_out; ++o) {
        uint8_t *row = out + o * rb;
        for (int64_t b = 0; b < rb; ++b) row[b] = 0x55;
        for (int64_t k = 0; k < d_in; ++k) {
            int64_t b = k / 4;
            int sh = (int)(2 * (k % 4));
            row[b] = (uint8_t)((row[b] & ~(3u << sh)) | ((unsigned)code_of(weff[o * d_in + k]) << sh));
        }
    }
}

int64_t sbl_oracle_nm_value_row_bytes(int64_t d_in, int n, int m)
{
    int64_t codes = d_in / m * n;
    return round_up((codes + 3) / 4, 16);
}

int64_t sbl_oracle_nm_bitmap_row_bytes(int64_t d_in) { return round_up(d_in / 8, 16); }

/* NM: the kept positions' 2-bit codes in ascending position order, four per
 * byte LSB-first (padding codes = 1), plus a keep-bitmap with bit k%8 of byte
 * k/8 set when position k is kept (padding bits = 0). */
void sbl_oracle_pack_nm(const int8_t *weff, const uint8_t *mask, int64_t d_out,
                        int64_t d_in, int n, int m, uint8_t *vals, uint8_t *bitmap)
{
    int64_t vb = sbl_oracle_nm_value_row_bytes(d_in, n, m);
    int64_t bb = sbl_oracle_nm_bitmap_row_bytes(d_in);
    for (int64_t o = 0; o < d_out; ++o) {
        uint8_t *vrow = vals + o * vb;
        uint8_t *brow = bitmap + o * bb;
        for (int64_t b = 0; b < vb; ++b) vrow[b] = 0x55;
        for (int64_t b = 0; b < bb; ++b) brow[b] = 0;
        int64_t slot = 0;
        for (int64_t k = 0; k < d_in; ++k) {
            if (!mask[o * d_in + k]) continue;
            brow[k / 8] = (uint8_t)(brow[k / 8] | (1u << (k % 8)));
            int sh = (int)(2 * (slot % 4));
            uint8_t *p = &vrow[slot / 4];
            *p = (uint8_t)((*p & ~(3u << sh)) | ((unsigned)code_of(weff[o * d_in + k]) << sh));
            slot++;
        }
    }
}

int64_t sbl_oracle_sp24_value_row_bytes(int64_t d_in) { return round_up(d_in / 2, 16); }

int64_t sbl_oracle_sp24_meta_row_bytes(int64_t d_in) { return round_up(d_in / 8, 16); }

/* SP24 (reading R14): W_eff as the 2:4-compressed operand of the sparse
 * tensor-core MMA (two stored values per group of four positions plus their
 * 2-bit indices).
 * For group g of a row (positions 4g .. 4g+3) the two positions i0 < i1 are
 * the group's kept positions, completed, when fewer than two are kept, with
 * the smallest positions of the group that are not kept.  Values: int8
 * W_eff at 4g+i0 and 4g+i1 in bytes 2g and 2g+1 of the value row.
 * Metadata: the nibble i0 | (i1 << 2) at bits 4*(g%2) of byte g/2 of the
 * metadata row.  Padding bytes are 0.  Returns -1 (writing nothing further)
 * when a group keeps more than two positions: such a mask is not 2:4. */
int sbl_oracle_pack_sp24(const int8_t *weff, const uint8_t *mask, int64_t d_out, int64_t d_in,
                         int8_t *vals, uint8_t *meta)
{
    int64_t vb = sbl_oracle_sp24_value_row_bytes(d_in);
    int64_t mb = sbl_oracle_sp24_meta_row_bytes(d_in);
    for (int64_t o = 0; o < d_out; ++o) {
        int8_t *vrow = vals + o * vb;
        uint8_t *mrow = meta + o * mb;
        for (int64_t b = 0; b < vb; ++b) vrow[b] = 0;
        for (int64_t b = 0; b < mb; ++b) mrow[b] = 0;
        for (int64_t g = 0; g < d_in / 4; ++g) {
            int idx[2];
            int count = 0;
            for (int i = 0; i < 4; ++i) {
                if (!mask[o * d_in + 4 * g + i]) continue;
                if (count == 2) return -1;
                idx[count++] = i;
            }
            /* complete with the smallest positions not kept */
            for (int i = 0; i < 4 && count < 2; ++i) {
                if (mask[o * d_in + 4 * g + i]) continue;
                if (count == 1 && idx[0] == i) continue;
                idx[count++] = i;
            }
            if (idx[0] > idx[1]) {
                int t = idx[0];
                idx[0] = idx[1];
                idx[1] = t;
            }
            vrow[2 * g] = weff[o * d_in + 4 * g + idx[0]];
            vrow[2 * g + 1] = weff[o * d_in + 4 * g + idx[1]];
            unsigned nib = (unsigned)idx[0] | ((unsigned)idx[1] << 2);
            mrow[g / 2] = (uint8_t)(mrow[g / 2] | (nib << (4 * (g % 2))));
        }
    }
    return 0;
}

int64_t sbl_oracle_t24_lo_row_bytes(int64_t d_in) { return round_up(d_in / 8, 16); }

int64_t sbl_oracle_t24_hi_row_bytes(int64_t d_in) { return round_up(d_in / 16, 16); }

/* T24: W_eff of a layer whose groups of four hold at most two nonzeros (2:4,
 * 1:4, 2:8, 1:8 masks) in 6 bits per group -- a denser form of the 2-bit
 * packing of [P5] "Inference Implementation: GPU" (no page gives a layout:
 * reading R24).  Group g (positions 4g .. 4g+3) with nonzero positions
 * p < q and sign bits s = 1 for -1, 0 for +1:
 *   no nonzero   code 0
 *   one (p)      code 1 + 2p + s_p                        (1 .. 8)
 *   two (p, q)   code 9 + 4k + 2 s_p + s_q, k the index of (p, q) in
 *                (0,1) (0,2) (0,3) (1,2) (1,3) (2,3)       (9 .. 32)
 * Low plane: code & 15 at bits 4 (g % 2) of byte g / 2 of the row; high
 * plane: code >> 4 at bits 2 (g % 4) of byte g / 4.  Padding bytes 0.
 * Returns -1 when a group has more than two nonzeros. */
int sbl_oracle_pack_t24(const int8_t *weff, int64_t d_out, int64_t d_in, uint8_t *lo, uint8_t *hi)
{
    static const int pair_index[4][4] = {{-1, 0, 1, 2}, {-1, -1, 3, 4}, {-1, -1, -1, 5}, {-1, -1, -1, -1}};
    int64_t lb = sbl_oracle_t24_lo_row_bytes(d_in), hb = sbl_oracle_t24_hi_row_bytes(d_in);
    for (int64_t o = 0; o < d_out; ++o) {
        uint8_t *lrow = lo + o * lb, *hrow = hi + o * hb;
        for (int64_t b = 0; b < lb; ++b) lrow[b] = 0;
        for (int64_t b = 0; b < hb; ++b) hrow[b] = 0;
        for (int64_t g = 0; g < d_in / 4; ++g) {
            const int8_t *w = weff + o * d_in + 4 * g;
            int pos[4], count = 0;
            for (int i = 0; i < 4; ++i)
                if (w[i] != 0) pos[count++] = i;
            unsigned code;
            if (count == 0) {
                code = 0;
            } else if (count == 1) {
                code = 1u + 2u * (unsigned)pos[0] + (w[pos[0]] < 0 ? 1u : 0u);
            } else if (count == 2) {
                code = 9u + 4u * (unsigned)pair_index[pos[0]][pos[1]] + (w[pos[0]] < 0 ? 2u : 0u) +
                       (w[pos[1]] < 0 ? 1u : 0u);
            } else {
                return -1;
            }
            lrow[g / 2] = (uint8_t)(lrow[g / 2] | ((code & 15u) << (4 * (g % 2))));
            hrow[g / 4] = (uint8_t)(hrow[g / 4] | ((code >> 4) << (2 * (g % 4))));
        }
    }
    return 0;
}

/* ------------------------------------------------------ mask statistics -- */

/* Mask flip count between consecutive steps ([P1] "Dynamic Mask
 * Recomputation at Every Training Step", flip rate r_t; reading R15): the
 * number of positions whose keep bit differs between the two masks, so that
 * r_t = flips / count.  Masks are one byte per position (0 or 1). */
int64_t sbl_oracle_mask_flips(const uint8_t *mask_prev, const uint8_t *mask, int64_t count)
{
    int64_t flips = 0;
    for (int64_t i = 0; i < count; ++i)
        if ((mask_prev[i] != 0) != (mask[i] != 0)) flips++;
    return flips;
}

/* Near-zero mass ([P1] "Polarization analysis": the share of weights with
 * |W| / gamma under 0.5; reading R16), as a count:
 * #{ fl32(|w| / gamma) < 0.5 }; every weight counts when gamma == 0 (all
 * weights are then 0 and quantise to 0). */
int64_t sbl_oracle_near_zero(const float *w, int64_t count, float gamma)
{
    if (!(gamma > 0.0f)) return count;
    int64_t c = 0;
    for (int64_t i = 0; i < count; ++i) {
        float r = fabsf(w[i]) / gamma;
        if (r < 0.5f) c++;
    }
    return c;
}

/* Per-block pruning threshold ([P1] "Magnitude stratification", threshold
 * t; reading R17): for row o
 * and group g, the largest |W| among the group's positions the mask drops,
 * which is the (n+1)-th largest |W| of the group; 0 when n == m (nothing is
 * dropped).  Output fp32 [d_out, d_in / m]. */
void sbl_oracle_block_threshold(const float *w, const uint8_t *mask, int64_t d_out, int64_t d_in,
                                int m, float *t)
{
    for (int64_t o = 0; o < d_out; ++o)
        for (int64_t g = 0; g < d_in / m; ++g) {
            float best = 0.0f;
            for (int i = 0; i < m; ++i) {
                int64_t k = o * d_in + g * m + i;
                if (mask[k]) continue;
                float a = fabsf(w[k]);
                if (a > best) best = a;
            }
            t[o * (d_in / m) + g] = best;
        }
}

/* ------------------------------------------------- activation quantiser -- */

static float bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* [P1] 3.4 activation quantisation equation; [P5] "Activation Quantization:
 * Per-Token Absmax": one scale per token, 127 / max|x|, rounding to the
 * nearest integer; reading R6. */
void sbl_oracle_quantize_act(const uint16_t *x, int64_t tokens, int64_t d_in,
                             int8_t *q, float *d)
{
    for (int64_t t = 0; t < tokens; ++t) {
        const uint16_t *row = x + t * d_in;
        float a = 0.0f;
        for (int64_t k = 0; k < d_in; ++k) {
            float v = fabsf(bf16_to_f32(row[k]));
            if (v > a) a = v;
        }
        if (a == 0.0f) {
            for (int64_t k = 0; k < d_in; ++k) q[t * d_in + k] = 0;
            d[t] = 0.0f;
            continue;
        }
        float r = 127.0f / a;
        for (int64_t k = 0; k < d_in; ++k) {
            float s = bf16_to_f32(row[k]) * r;
            float v = nearbyintf(s);
            if (v > 127.0f) v = 127.0f;
            if (v < -128.0f) v = -128.0f;
            q[t * d_in + k] = (int8_t)v;
        }
        d[t] = a / 127.0f;
    }
}

/* ------------------------------------------------------------- forward -- */

/* [P1] "The Full Sparse-BitLinear Layer", forward step 5: the integer
 * product of the masked ternary weights and the int8 activations.
 * Returns 0, or -1 when a sum does not fit int32. */
int sbl_oracle_gemm_acc(const int8_t *q, const int8_t *weff, int64_t tokens,
                        int64_t d_out, int64_t d_in, int32_t *acc)
{
    int status = 0;
    for (int64_t t = 0; t < tokens; ++t) {
        for (int64_t o = 0; o < d_out; ++o) {
            int64_t s = 0;
            for (int64_t k = 0; k < d_in; ++k)
                s += (int64_t)q[t * d_in + k] * (int64_t)weff[o * d_in + k];
            if (s > INT32_MAX || s < INT32_MIN) status = -1;
            acc[t * d_out + o] = (int32_t)s;
        }
    }
    return status;
}

/* Round-to-nearest-even fp32 -> bf16 (NaN kept quiet). */
static uint16_t f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* [P1] forward step 5: one scalar absorbs the weight scale gamma and the
 * token scale max|x|/127; reading R7. */
void sbl_oracle_dequant(const int32_t *acc, int64_t tokens, int64_t d_out,
                        float gamma, const float *d, float *y, uint16_t *y_bf16)
{
    for (int64_t t = 0; t < tokens; ++t) {
        float c = gamma * d[t];
        for (int64_t o = 0; o < d_out; ++o) {
            float v = (float)acc[t * d_out + o] * c;
            if (y) y[t * d_out + o] = v;
            if (y_bf16) y_bf16[t * d_out + o] = f32_to_bf16(v);
        }
    }
}

/* Pairwise tree (R1's shape) over the squares of a row of bf16 values, fp64:
 * each square of a bf16 value is exact in fp64. */
static double square_sum_tree(const uint16_t *x, int64_t lo, int64_t n)
{
    if (n <= 0) return 0.0;
    if (n == 1) {
        double v = (double)bf16_to_f32(x[lo]);
        return v * v;
    }
    int64_t h = 1;
    while (h * 2 < n) h *= 2;
    double left = square_sum_tree(x, lo, h);
    double right = square_sum_tree(x, lo + h, n - h);
    return left + right;
}

/* The norm before the activation quantiser ([P1] forward step 1:
 * x~ = Q_a(Norm(x)), Norm being RMSNorm) fused with it:
 *   r   = fl32(1 / sqrt(S / K + eps)) in fp64, S = the pairwise tree of
 *         x_k^2 over the row in flat order;
 *   u_k = fl32(fl32(x_k * r) * g_k)   (g: bf16 gains, 1 when absent);
 * then the quantiser of sbl_oracle_quantize_act on the fp32 u (a = max|u|,
 * q = clamp(rint(fl32(u * fl32(127 / a)))), d = fl32(a / 127); a == 0 gives
 * q = 0, d = 0).  Reading R23. */
void sbl_oracle_rmsnorm_quantize_act(const uint16_t *x, int64_t tokens, int64_t d_in, const uint16_t *g,
                                     float eps, int8_t *q, float *d)
{
    for (int64_t t = 0; t < tokens; ++t) {
        const uint16_t *row = x + t * d_in;
        double s = square_sum_tree(row, 0, d_in);
        float r = (float)(1.0 / sqrt(s / (double)d_in + (double)eps));
        float a = 0.0f;
        for (int64_t k = 0; k < d_in; ++k) {
            float u = bf16_to_f32(row[k]) * r;
            if (g) u = u * bf16_to_f32(g[k]);
            if (fabsf(u) > a) a = fabsf(u);
        }
        if (a == 0.0f) {
            for (int64_t k = 0; k < d_in; ++k) q[t * d_in + k] = 0;
            d[t] = 0.0f;
            continue;
        }
        float rq = 127.0f / a;
        for (int64_t k = 0; k < d_in; ++k) {
            float u = bf16_to_f32(row[k]) * r;
            if (g) u = u * bf16_to_f32(g[k]);
            float v = nearbyintf(u * rq);
            if (v > 127.0f) v = 127.0f;
            if (v < -128.0f) v = -128.0f;
            q[t * d_in + k] = (int8_t)v;
        }
        d[t] = a / 127.0f;
    }
}

/* Output epilogue after the layer ("Squared ReLU Activation in the
 * Feed-Forward Network" of the BitNet b1.58 2B4T summary: ReLU^2(x) =
 * max(0, x)^2, applied to the projection's output; and a residual add):
 *   v = y                      (the fp32 output of sbl_oracle_dequant)
 *   v = v > 0 ? fl32(v * v) : 0   when relu2
 *   v = fl32(v + r)            when a residual r (bf16 [T, O]) is given
 * written as fp32 and as bf16 (round to nearest even).  Reading R22. */
void sbl_oracle_epilogue(const float *y, int64_t tokens, int64_t d_out, int relu2, const uint16_t *res,
                         float *out, uint16_t *out_bf16)
{
    for (int64_t i = 0; i < tokens * d_out; ++i) {
        float v = y[i];
        if (relu2) v = v > 0.0f ? v * v : 0.0f;
        if (res) v = v + bf16_to_f32(res[i]);
        if (out) out[i] = v;
        if (out_bf16) out_bf16[i] = f32_to_bf16(v);
    }
}

/* ------------------------------------------------------------ backward -- */

/* [P1] "The Dual Straight-Through Estimator" (dL/dW ~= dL/dW_eff) and the
 * backward walk-through (gradient flows through mask and quantiser as
 * identity); readings R8 and R9, evaluated in fp64.
 *   dX[t,k] = gamma * sum_o dY[t,o] * W_eff[o,k]
 *   dW[o,k] = sum_t dY[t,o] * d_t * q[t,k]     (unmasked) */
void sbl_oracle_backward(const uint16_t *dy, const int8_t *weff, float gamma,
                         const int8_t *q, const float *d, int64_t tokens,
                         int64_t d_out, int64_t d_in, double *dx, double *dw)
{
    if (dx) {
        for (int64_t t = 0; t < tokens; ++t)
            for (int64_t k = 0; k < d_in; ++k) {
                double s = 0.0;
                for (int64_t o = 0; o < d_out; ++o)
                    s += (double)bf16_to_f32(dy[t * d_out + o]) * (double)weff[o * d_in + k];
                dx[t * d_in + k] = (double)gamma * s;
            }
    }
    if (dw) {
        for (int64_t o = 0; o < d_out; ++o)
            for (int64_t k = 0; k < d_in; ++k) {
                double s = 0.0;
                for (int64_t t = 0; t < tokens; ++t)
                    s += (double)bf16_to_f32(dy[t * d_out + o]) * (double)d[t] *
                         (double)q[t * d_in + k];
                dw[o * d_in + k] = s;
            }
    }
}

/* Sampled variants: the same definitions evaluated at chosen output
 * coordinates only, so full-size launches can be checked one output at a
 * time.  acc at (t, o); dX at (t, k); dW at (o, k). */
void sbl_oracle_acc_samples(const int8_t *q, const int8_t *weff, int64_t d_in,
                            const int64_t *idx_t, const int64_t *idx_o,
                            int64_t n_samples, int64_t *out)
{
    for (int64_t s = 0; s < n_samples; ++s) {
        int64_t t = idx_t[s], o = idx_o[s];
        int64_t acc = 0;
        for (int64_t k = 0; k < d_in; ++k)
            acc += (int64_t)q[t * d_in + k] * (int64_t)weff[o * d_in + k];
        out[s] = acc;
    }
}

void sbl_oracle_dx_samples(const uint16_t *dy, const int8_t *weff, float gamma,
                           int64_t d_out, int64_t d_in, const int64_t *idx_t,
                           const int64_t *idx_k, int64_t n_samples, double *out)
{
    for (int64_t s = 0; s < n_samples; ++s) {
        int64_t t = idx_t[s], k = idx_k[s];
        double acc = 0.0;
        for (int64_t o = 0; o < d_out; ++o)
            acc += (double)bf16_to_f32(dy[t * d_out + o]) * (double)weff[o * d_in + k];
        out[s] = (double)gamma * acc;
    }
}

void sbl_oracle_dw_samples(const uint16_t *dy, const int8_t *q, const float *d,
                           int64_t tokens, int64_t d_out, int64_t d_in,
                           const int64_t *idx_o, const int64_t *idx_k,
                           int64_t n_samples, double *out)
{
    for (int64_t s = 0; s < n_samples; ++s) {
        int64_t o = idx_o[s], k = idx_k[s];
        double acc = 0.0;
        for (int64_t t = 0; t < tokens; ++t)
            acc += (double)bf16_to_f32(dy[t * d_out + o]) * (double)d[t] *
                   (double)q[t * d_in + k];
        out[s] = acc;
    }
}

int sbl_oracle_rounding_is_nearest(void) { return fegetround() == FE_TONEAREST; }
