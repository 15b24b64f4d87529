/*
 * Oracle for the NVFP4 KV-cache append and block-causal chunk attention path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or constant generator
 * with the CUDA library.
 *
 * What it follows:
 *  - "NVlabs/LongLive 2.0: NVFP4 parallel infrastructure for long video
 *    generation", section "NVFP4, sequence parallel and the async decode path":
 *    the KV cache is stored in the same 4-bit NVFP4 format as the W4A4
 *    generator, and the listed optimisations include in-place quantized KV
 *    updates and FP4 KV dequantization.
 *  - "NVlabs LongLive" (refft.com), Core Analysis block "How do KV-cache
 *    relative RoPE and TriAttention work together": positions are assigned
 *    relative to the cache, so appended chunks do not drift.
 *  - The workload contract of the tiny reference case (2 heads, head_dim 128,
 *    8x8 tokens per frame): E2M1 element codes, one E4M3 scale per 16
 *    contiguous elements, a per-head FP32 global scale equal to the first
 *    chunk's amax divided by 6*448, round-to-nearest-even everywhere,
 *    saturation at +-6 and 448, keys cached before RoPE, 3D RoPE split
 *    44/42/42 over (frame, h, w) with base 10000.
 *
 * Precision: the scale arithmetic is FP32 as the contract fixes it (each FP32
 * operation is evaluated in double and rounded once to float, which is exact
 * IEEE single rounding for one +,-,*,/ because 53 >= 2*24+2); everything after
 * dequantization (RoPE, logits, softmax, weighted sum) is fp64.
 *
 * Compile with -ffp-contract=off and without -ffast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- FP32 ops */

static float f32_mul(float a, float b) { return (float)((double)a * (double)b); }
static float f32_div(float a, float b) { return (float)((double)a / (double)b); }

/* ------------------------------------------------------------ E2M1 format */

/* E2M1: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.
 * Exponent 0 is subnormal: value = m * 0.5.  Otherwise 2^(e-1) * (1 + m/2). */
double oracle_e2m1_decode(uint8_t code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* Nearest E2M1 magnitude by exhaustive search over the eight magnitude codes;
 * a tie goes to the even code (mantissa bit 0).  Magnitudes above 6 saturate
 * to 6 (stated explicitly: for huge values the fp64 distances to 4 and 6
 * would compare equal).  A value whose magnitude rounds to zero is stored as
 * 0x0 (no negative zero). */
uint8_t oracle_e2m1_encode(float y)
{
    double a = fabs((double)y);
    int best = 0;
    double best_err = INFINITY;
    if (a > 6.0) return (uint8_t)(y < 0.0f ? 0xF : 0x7);
    for (int c = 0; c < 8; ++c) {
        double err = fabs(oracle_e2m1_decode((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_err = err;
        }
    }
    if (best != 0 && y < 0.0f) best |= 8;
    return (uint8_t)best;
}

/* ------------------------------------------------------------ E4M3 format */

/* E4M3 ("fn" variant): bit 7 sign, bits 6..3 exponent (bias 7), bits 2..0
 * mantissa.  Exponent 0 is subnormal: m * 2^-9.  S.1111.111 is NaN, there is
 * no infinity, the largest finite value is 1.75 * 2^8 = 448. */
double oracle_e4m3_decode(uint8_t b)
{
    int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Nearest non-negative finite E4M3 value by exhaustive search over codes
 * 0x00..0x7E; a tie goes to the even code.  The caller clamps at 448 first,
 * as the block-scale rule does. */
uint8_t oracle_e4m3_encode(float t)
{
    double a = (double)t;
    int best = 0;
    double best_err = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double err = fabs(oracle_e4m3_decode((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)best;
}

/* ---------------------------------------------------------- NVFP4 scales */

/* Per-head global scale: s_g = fl32(amax / (6 * 448)).  A zero amax (or one
 * so small that s_g would not be a normal float) gives s_g = 1. */
float oracle_global_scale(float amax)
{
    float s = f32_div(amax, 2688.0f);
    if (!(s >= 1.17549435e-38f)) s = 1.0f;
    return s;
}

/* amax over n values (bf16 values carried as float). */
float oracle_amax(const float *x, int64_t n)
{
    float m = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > m) m = a;
    }
    return m;
}

/* One 16-element block:
 *   amax16 = max |x_i|
 *   t      = fl32(amax16 / fl32(6 * s_g))
 *   s_b    = 448 if t >= 448, else E4M3_RNE(t)
 *   y_i    = fl32(x_i / fl32(s_b * s_g)),   q_i = E2M1_RNE_sat(y_i)
 * s_b = 0 (zero block or scale underflow) gives sixteen zero codes.
 * Element 2i goes to the low nibble of byte i, element 2i+1 to the high one. */
void oracle_quantize_block16(const float *x, float s_g, uint8_t *codes8, uint8_t *scale)
{
    float amax16 = oracle_amax(x, 16);
    float t = f32_div(amax16, f32_mul(6.0f, s_g));
    uint8_t sb = (t >= 448.0f) ? (uint8_t)0x7E : oracle_e4m3_encode(t);
    float s_b = (float)oracle_e4m3_decode(sb);
    *scale = sb;
    memset(codes8, 0, 8);
    if (s_b == 0.0f) return;
    float d = f32_mul(s_b, s_g);
    for (int i = 0; i < 16; ++i) {
        uint8_t q = oracle_e2m1_encode(f32_div(x[i], d));
        codes8[i >> 1] |= (uint8_t)(q << ((i & 1) * 4));
    }
}

/* Quantize n_rows rows of 128 elements (one token-head each) with one global
 * scale: codes [n_rows][64], scales [n_rows][8]. */
void oracle_quantize_rows(const float *x, int64_t n_rows, float s_g, uint8_t *codes, uint8_t *scales)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r)
        for (int blk = 0; blk < 8; ++blk)
            oracle_quantize_block16(x + r * 128 + blk * 16, s_g, codes + r * 64 + blk * 8,
                                    scales + r * 8 + blk);
}

/* Dequantize rows: value = e2m1(code) * s_b * s_g, in fp64 (exact). */
void oracle_dequant_rows(const uint8_t *codes, const uint8_t *scales, int64_t n_rows, float s_g,
                         double *out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_rows; ++r)
        for (int i = 0; i < 128; ++i) {
            uint8_t byte = codes[r * 64 + i / 2];
            uint8_t q = (i & 1) ? (byte >> 4) : (byte & 15);
            double s_b = oracle_e4m3_decode(scales[r * 8 + i / 16]);
            out[r * 128 + i] = oracle_e2m1_decode(q) * s_b * (double)s_g;
        }
}

/* ------------------------------------------------------------------ RoPE */

/* 3D RoPE on one 128-channel vector, in place, fp64.  Channels are split in
 * three consecutive segments of widths split[0..2] for the (frame, h, w)
 * axes.  Inside a segment of width d, pair i is channels (2i, 2i+1) of the
 * segment, rotated by angle pos * base^(-2i/d):
 *   (x, y) -> (x cos a - y sin a, x sin a + y cos a). */
void oracle_rope3d(double *x, const int *pos3, const int *split, double base)
{
    int off = 0;
    for (int ax = 0; ax < 3; ++ax) {
        int d = split[ax];
        for (int i = 0; i < d / 2; ++i) {
            double theta = pow(base, -2.0 * i / (double)d);
            double a = (double)pos3[ax] * theta;
            double c = cos(a), s = sin(a);
            double x0 = x[off + 2 * i], x1 = x[off + 2 * i + 1];
            x[off + 2 * i] = x0 * c - x1 * s;
            x[off + 2 * i + 1] = x0 * s + x1 * c;
        }
        off += d;
    }
}

/* ------------------------------------------------------------- Attention */

/* Chunk attention for one (batch, head), fp64.
 *   q      [Lq][128]   query values (bf16 inputs as float), before RoPE
 *   k, v   [Lk][128]   dequantized cached keys (before RoPE) and values
 *   k_frame_pos [Lk]   RoPE frame index of each key (its order in the cache)
 *   k_tok  [Lk]        token index of each key inside its frame
 *   q_frame_pos [Lq]   RoPE frame index of each query row
 *   q_tok  [Lq]        token index of each query row inside its frame
 *   rows   [n_rows]    which query rows to compute (all keys are visible to
 *                      every listed row; masking is done by the caller's
 *                      choice of keys)
 *   out    [n_rows][128], lse [n_rows] (natural log of the softmax sum,
 *                      including the max)
 * Logits are (R q) . (R k) / sqrt(128); softmax with max subtraction. */
void oracle_attention_rows(const float *q, const double *k, const double *v, int64_t Lk,
                           const int *k_frame_pos, const int *k_tok, const int *q_frame_pos,
                           const int *q_tok, const int64_t *rows, int64_t n_rows, int grid_w,
                           const int *split, double base, double *out, double *lse)
{
    double *kr = (double *)malloc(sizeof(double) * (size_t)Lk * 128);
    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < Lk; ++j) {
        int pos3[3] = {k_frame_pos[j], k_tok[j] / grid_w, k_tok[j] % grid_w};
        memcpy(kr + j * 128, k + j * 128, sizeof(double) * 128);
        oracle_rope3d(kr + j * 128, pos3, split, base);
    }
    const double scale = 1.0 / sqrt(128.0);
    #pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        #pragma omp for schedule(dynamic, 1)
        for (int64_t ri = 0; ri < n_rows; ++ri) {
            int64_t r = rows[ri];
            double qr[128];
            for (int i = 0; i < 128; ++i) qr[i] = (double)q[r * 128 + i];
            int pos3[3] = {q_frame_pos[r], q_tok[r] / grid_w, q_tok[r] % grid_w};
            oracle_rope3d(qr, pos3, split, base);
            double m = -INFINITY;
            for (int64_t j = 0; j < Lk; ++j) {
                double s = 0.0;
                for (int i = 0; i < 128; ++i) s += qr[i] * kr[j * 128 + i];
                logit[j] = s * scale;
                if (logit[j] > m) m = logit[j];
            }
            double acc[128];
            for (int i = 0; i < 128; ++i) acc[i] = 0.0;
            double l = 0.0;
            for (int64_t j = 0; j < Lk; ++j) {
                double p = exp(logit[j] - m);
                l += p;
                for (int i = 0; i < 128; ++i) acc[i] += p * v[j * 128 + i];
            }
            for (int i = 0; i < 128; ++i) out[ri * 128 + i] = (Lk > 0) ? acc[i] / l : 0.0;
            if (lse) lse[ri] = (Lk > 0) ? m + log(l) : -INFINITY;
        }
        free(logit);
    }
    free(kr);
}

/* ------------------------------------- block-scaled FP4 Q K^T (a reading) */

/* A reading of "NVFP4 quantization end to end" (evermx.com, heading "NVFP4
 * Quantization End-to-End": the KV cache is held in the same 4-bit format as
 * the W4A4 generator) for the logits: Q K^T taken on FP4 operands, as a
 * block-scaled tensor-core contraction would, instead of on dequantized K.
 * The pages give no such kernel; the steps below are the plainest reading
 * that keeps the relative 3D RoPE ("NVlabs LongLive", refft.com, Core
 * Analysis block on KV-cache relative RoPE) exact:
 *  1. At append, K's spatial pairs (h and w segments) are rotated at the
 *     token's (h, w); its frame segment is stored unrotated.  The rotated row
 *     is quantized with the cache's NVFP4 rules (s_g from the first chunk's
 *     amax of the rotated rows).
 *  2. A query row at frame index f_q and (h_q, w_q) meets the keys of a frame
 *     at index f_k through Q_fk: its frame segment rotated by the relative
 *     index f_q - f_k, its spatial segments at (h_q, w_q).  Then
 *     Q_fk . K' = R(f_q, h_q, w_q) q . R(f_k, h_k, w_k) k exactly in real
 *     arithmetic, since the frame rotations of q and k combine to their
 *     difference and K' carries k's spatial rotation.
 *  3. Q_fk is quantized with the NVFP4 rules, one global scale per query row
 *     that holds for every rotation: s_gq = fl32(p / 2688) with p the row's
 *     largest pair magnitude fl32(sqrt(fl32(fl32(x^2) + fl32(y^2)))) (a
 *     rotation keeps each pair's magnitude, so no element of any Q_fk exceeds
 *     it but by rounding, which the 448 and 6 clamps absorb).
 *  4. The logit is the dot product of the dequantized Q_fk and K' rows, over
 *     sqrt(128); the softmax and the weighted sum of V are unchanged.
 * Precision: the rotations feed a quantizer whose codes are integers, so
 * they are fixed in float: cos and sin of the fp64 angle pos * base^(-2i/d),
 * each rounded once to float, and (fl32(fl32(x c) - fl32(y s)),
 * fl32(fl32(x s) + fl32(y c))).  Everything after dequantization is fp64. */

static float f32_add(float a, float b) { return (float)((double)a + (double)b); }
static float f32_sub(float a, float b) { return (float)((double)a - (double)b); }

/* cos and sin of pair i of a RoPE segment of width d at integer position pos,
 * each rounded once to float. */
void oracle_rope_cs_f32(int pos, int i, int d, double base, float *c, float *s)
{
    double a = (double)pos * pow(base, -2.0 * i / (double)d);
    *c = (float)cos(a);
    *s = (float)sin(a);
}

/* One pair (x, y) rotated in float with the rounded cos c and sin s. */
static void rot_pair_f32(float *x, float *y, float c, float s)
{
    float x0 = *x, y0 = *y;
    *x = f32_sub(f32_mul(x0, c), f32_mul(y0, s));
    *y = f32_add(f32_mul(x0, s), f32_mul(y0, c));
}

/* Rotate the channels of one 128-vector in float, segment by segment, at
 * positions pos3 (frame, h, w); a position of 0 leaves its segment as is. */
void oracle_rope3d_f32(float *x, const int *pos3, const int *split, double base)
{
    int off = 0;
    for (int ax = 0; ax < 3; ++ax) {
        int d = split[ax];
        if (pos3[ax] != 0)
            for (int i = 0; i < d / 2; ++i) {
                float c, s;
                oracle_rope_cs_f32(pos3[ax], i, d, base, &c, &s);
                rot_pair_f32(&x[off + 2 * i], &x[off + 2 * i + 1], c, s);
            }
        off += d;
    }
}

/* Step 1: K rows (bf16 values as float) with their spatial segments rotated
 * at each row's token (h = tok / grid_w, w = tok % grid_w), in place. */
void oracle_k_spatial_rope_f32(float *k, int64_t n, const int *tok, int grid_w, const int *split,
                               double base)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        int pos3[3] = {0, tok[r] / grid_w, tok[r] % grid_w};
        oracle_rope3d_f32(k + r * 128, pos3, split, base);
    }
}

/* Step 3: the per-row global scale of Q (1 if not a normal float). */
float oracle_q_row_global_scale(const float *q)
{
    float p = 0.0f;
    for (int i = 0; i < 64; ++i) {
        float x = q[2 * i], y = q[2 * i + 1];
        float m = (float)sqrt((double)f32_add(f32_mul(x, x), f32_mul(y, y)));
        if (m > p) p = m;
    }
    float s = f32_div(p, 2688.0f);
    if (!(s >= 1.17549435e-38f)) s = 1.0f;
    return s;
}

/* Steps 2 and 3 for one query row and one relative frame index dpos:
 * Q_fk quantized (codes [64], scales [8]) with the row's global scale. */
void oracle_q_for_frame(const float *q, int dpos, int q_tok, int grid_w, const int *split,
                        double base, float s_gq, uint8_t *codes, uint8_t *scales)
{
    float x[128];
    memcpy(x, q, sizeof(x));
    int pos3[3] = {dpos, q_tok / grid_w, q_tok % grid_w};
    oracle_rope3d_f32(x, pos3, split, base);
    oracle_quantize_rows(x, 1, s_gq, codes, scales);
}

/* The block form of one FP4 logit as a block-scaled contraction forms it:
 * per 16-element block the integer sum of code products (E2M1 values are
 * multiples of 1/2, so 4 times each product is an integer), times the two
 * block scales; then the global scales.  Equal to the dot product of the
 * dequantized rows up to fp64 rounding. */
double oracle_fp4_dot(const uint8_t *ca, const uint8_t *sa, float ga, const uint8_t *cb,
                      const uint8_t *sb, float gb)
{
    double acc = 0.0;
    for (int blk = 0; blk < 8; ++blk) {
        long long isum = 0;
        for (int i = blk * 16; i < blk * 16 + 16; ++i) {
            uint8_t qa = (ca[i / 2] >> ((i & 1) * 4)) & 15, qb = (cb[i / 2] >> ((i & 1) * 4)) & 15;
            isum += (long long)llround(4.0 * oracle_e2m1_decode(qa) * oracle_e2m1_decode(qb));
        }
        acc += (double)isum * 0.25 * oracle_e4m3_decode(sa[blk]) * oracle_e4m3_decode(sb[blk]);
    }
    return acc * (double)ga * (double)gb;
}

/* Step 4: chunk attention of one (batch, head) on the listed query rows with
 * FP4 logits.  q [Lq][128] pre-RoPE query values; kd [Lk][128] the cached K'
 * rows dequantized (step 1; exact in fp64); v [Lk][128] dequantized values;
 * positions as in oracle_attention_rows.  Q_fk is formed once per distinct
 * key frame index; quantize_q = 0 keeps it in float (no step 3), which the
 * tests use to check the RoPE split on its own.  out [n_rows][128], lse
 * [n_rows]. */
void oracle_attention_rows_fp4qk(const float *q, const double *kd, const double *v, int64_t Lk,
                                 const int *k_frame_pos, const int *q_frame_pos, const int *q_tok,
                                 const int64_t *rows, int64_t n_rows, int grid_w, const int *split,
                                 double base, int quantize_q, double *out, double *lse)
{
    int max_pos = 0;
    for (int64_t j = 0; j < Lk; ++j)
        if (k_frame_pos[j] > max_pos) max_pos = k_frame_pos[j];
    const double scale = 1.0 / sqrt(128.0);
    #pragma omp parallel
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        double *qd = (double *)malloc(sizeof(double) * (size_t)(max_pos + 1) * 128);
        char *have = (char *)malloc((size_t)max_pos + 1);
        #pragma omp for schedule(dynamic, 1)
        for (int64_t ri = 0; ri < n_rows; ++ri) {
            int64_t r = rows[ri];
            const float *qr = q + r * 128;
            float s_gq = oracle_q_row_global_scale(qr);
            memset(have, 0, (size_t)max_pos + 1);
            double m = -INFINITY;
            for (int64_t j = 0; j < Lk; ++j) {
                int fk = k_frame_pos[j];
                if (!have[fk]) {
                    if (quantize_q) {
                        uint8_t c[64], sc[8];
                        oracle_q_for_frame(qr, q_frame_pos[r] - fk, q_tok[r], grid_w, split,
                                           base, s_gq, c, sc);
                        oracle_dequant_rows(c, sc, 1, s_gq, qd + (size_t)fk * 128);
                    } else {
                        float x[128];
                        memcpy(x, qr, sizeof(x));
                        int pos3[3] = {q_frame_pos[r] - fk, q_tok[r] / grid_w, q_tok[r] % grid_w};
                        oracle_rope3d_f32(x, pos3, split, base);
                        for (int i = 0; i < 128; ++i) qd[(size_t)fk * 128 + i] = (double)x[i];
                    }
                    have[fk] = 1;
                }
                double s = 0.0;
                for (int i = 0; i < 128; ++i) s += qd[(size_t)fk * 128 + i] * kd[j * 128 + i];
                logit[j] = s * scale;
                if (logit[j] > m) m = logit[j];
            }
            double acc[128];
            for (int i = 0; i < 128; ++i) acc[i] = 0.0;
            double l = 0.0;
            for (int64_t j = 0; j < Lk; ++j) {
                double p = exp(logit[j] - m);
                l += p;
                for (int i = 0; i < 128; ++i) acc[i] += p * v[j * 128 + i];
            }
            for (int i = 0; i < 128; ++i) out[ri * 128 + i] = (Lk > 0) ? acc[i] / l : 0.0;
            if (lse) lse[ri] = (Lk > 0) ? m + log(l) : -INFINITY;
        }
        free(have);
        free(qd);
        free(logit);
    }
}

/* ------------------------------------------------------ array entry points */

/* Block-scale code for a scale ratio t (the clamp at 448 included). */
uint8_t oracle_block_scale_code(float t)
{
    return (t >= 448.0f) ? (uint8_t)0x7E : oracle_e4m3_encode(t);
}

void oracle_e2m1_encode_array(const float *y, int64_t n, uint8_t *out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_encode(y[i]);
}

void oracle_block_scale_code_array(const float *t, int64_t n, uint8_t *out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_block_scale_code(t[i]);
}
