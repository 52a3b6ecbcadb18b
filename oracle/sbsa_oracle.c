/*
 * CPU oracle for dynamic block-sparse self-attention -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference arm
 * may load or run this file.  The product path (the sm_100a library under
 * video_dit_dynamic_b200/) shares no code with it and never calls it.
 *
 * What it computes is the plain definition of the method, step by step, in fp64:
 *
 *   [Card]  = page "知识卡片：600倍加速，720p视频实时生成！单卡也能带的动14B模型",
 *             section 方法/产品要点, bullet 动态稀疏量化注意力
 *   [Guide] = page "单卡 RTX 5090 跑 Wan2.2-A14B：720p 视频生成只要 3.8 秒",
 *             section 四步拆解, item 3 动态稀疏注意力
 *
 *   1. pool    ([Card], [Guide]): block-level MEANS of Query and of Key are the
 *              cheap importance estimate.  Mean over the valid tokens of a block.
 *   2. select  ([Card], [Guide]): keep only ~10-20% of the key blocks for each query
 *              block.  Reading taken here: score(i,j) = <qmean_i, kmean_j>, the
 *              diagonal block j == i is always kept and counts toward k, the other
 *              k-1 are the largest scores, ties broken by the lower block index.
 *              The kept list is written in ascending block order.
 *   3. attend  ([Guide]): the kept blocks are computed densely.  Softmax attention
 *              of each query row over exactly the valid keys of its kept blocks,
 *              non-causal, scale 1/sqrt(d) unless given.  Two-pass softmax (max,
 *              then exp-sums), not the online form.
 *
 *   0. rope    (next step on the path, fused with 1 in the library) [Card] bullet
 *              高效推理算子 and [Guide] item 4 融合内核: 3D RoPE runs as a fused kernel.
 *              The pages give no frequencies; the reading taken here is the usual 3D
 *              split of the head dimension into rotation pairs (2p, 2p+1): the first
 *              P_t = d/2 - 2*P_h pairs rotate with the frame index, the next
 *              P_h = floor(d/6) with the row index, the last P_w = P_h with the column
 *              index of the token on the (T, H, W) latent grid (row-major); pair q of an
 *              axis with P pairs turns by angle pos * theta^(-q/P), theta = 10000.
 *
 *   fp8     (next step: the FP8 path of [Card], same bullet, and [Guide] item 3: the
 *              sparse mask feeds an FP8 attention in the style of SageAttention2).  The
 *              pages give no quantization detail; the reading taken here: K is first
 *              smoothed by subtracting a per-(b,h) channel vector (the sequence mean of
 *              K), which leaves softmax unchanged; then every block of Q and of K gets
 *              one scale, amax/448 over its valid tokens, and its values become e4m3
 *              codes (round to nearest even, saturating at +-448).  The code decision is
 *              taken in fp32 arithmetic, the same operations the GPU performs, so codes
 *              and scales match bit for bit.  Attention then runs on the dequantized
 *              Q and K (code value * block scale) with V as given.
 *
 *   nvfp4   (next step: the linear layers around the attention, [Card] bullets NVFP4
 *              量化感知训练 and 高效推理算子, and page "单卡 RTX 5090 跑 Wan2.2-A14B：720p 视频
 *              生成只要 3.8 秒", 四步拆解 item 2: both GEMM operands in NVFP4 -- E2M1 values,
 *              one FP8 E4M3 scale per 16 consecutive elements, one FP32 scale per tensor --
 *              with FP32 accumulation, BF16 output and a column bias added in the epilogue).
 *              The pages give no formula for the scales; the reading taken here: the
 *              tensor scale s = 2688 / amax (2688 = 6 * 448, so the largest block scale
 *              is 448 and its largest element 6); each block of 16 along a row gets
 *              sf = e4m3((block amax / 6) * s); each element the e2m1 code of
 *              x * (s / sf), nearest with ties to the even code, saturating at +-6.  All of
 *              it in fp32 operations, the same the GPU performs.  A value decodes to
 *              code * sf / s, and the GEMM is C = A_dec * B_dec^T + bias (per column).
 *
 * Inputs are read as fp32, bf16 (raw 16-bit patterns, converted exactly) or fp64.
 * Tensors are row-major [B][H][Lp][d]; means are [B][H][nb][d]; col_idx is
 * [B][H][nb][k].  Padded tokens t >= L are ignored as keys and their query rows
 * produce 0.
 *
 * Parity pins live in tests/test_oracle_pins.py.  Every function below is pinned there.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F64 = 2 };

static int g_threads = 0; /* 0: OpenMP default */

void oracle_set_threads(int n) { g_threads = n; }

int oracle_threads_used(void) {
#ifdef _OPENMP
    return g_threads > 0 ? g_threads : omp_get_max_threads();
#else
    return 1;
#endif
}

static double elem(const void *x, int dtype, size_t i) {
    if (dtype == ORC_F32) return (double)((const float *)x)[i];
    if (dtype == ORC_BF16) {
        uint32_t bits = (uint32_t)((const uint16_t *)x)[i] << 16;
        float f;
        memcpy(&f, &bits, sizeof f);
        return (double)f;
    }
    return ((const double *)x)[i];
}

/* Step 1: block means over valid tokens.  out[(bh*nb + i)*d + c]. */
void oracle_pool(int B, int H, int L, int Lp, int d, int blk,
                 const void *x, int dtype, double *out) {
    int nb = Lp / blk;
    long rows = (long)B * H * nb;
#pragma omp parallel for schedule(static) num_threads(oracle_threads_used())
    for (long r = 0; r < rows; ++r) {
        long bh = r / nb;
        int i = (int)(r % nb);
        int t0 = i * blk;
        int t1 = t0 + blk < L ? t0 + blk : L;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            for (int t = t0; t < t1; ++t)
                s += elem(x, dtype, ((size_t)bh * Lp + t) * d + c);
            out[r * d + c] = t1 > t0 ? s / (double)(t1 - t0) : 0.0;
        }
    }
}

/* Step 0: 3D RoPE of one tensor [B][H][Lp][d] over the (gt, gh, gw) grid, in fp64.
 * Token t < L = gt*gh*gw is rotated by its grid position t -> (t / (gh*gw),
 * (t / gw) % gh, t % gw); padded tokens (t >= L) have no position and are copied
 * unrotated.  out has the input's shape. */
void oracle_rope(int B, int H, int Lp, int d, int gt, int gh, int gw, double theta,
                 const void *x, int dtype, double *out) {
    const int half = d / 2, ph = d / 6, pw = d / 6, pt = half - ph - pw;
    const long L = (long)gt * gh * gw;
    long rows = (long)B * H * Lp;
#pragma omp parallel for schedule(static) num_threads(oracle_threads_used())
    for (long r = 0; r < rows; ++r) {
        long t = r % Lp;
        if (t >= L) {
            for (int c = 0; c < d; ++c) out[(size_t)r * d + c] = elem(x, dtype, (size_t)r * d + c);
            continue;
        }
        long pos[3] = {t / ((long)gh * gw), (t / gw) % gh, t % gw};
        for (int p = 0; p < half; ++p) {
            int axis = p < pt ? 0 : (p < pt + ph ? 1 : 2);
            int q = axis == 0 ? p : (axis == 1 ? p - pt : p - pt - ph);
            int np = axis == 0 ? pt : (axis == 1 ? ph : pw);
            double ang = (double)pos[axis] * pow(theta, -(double)q / (double)np);
            double c = cos(ang), sn = sin(ang);
            double a = elem(x, dtype, (size_t)r * d + 2 * p);
            double b = elem(x, dtype, (size_t)r * d + 2 * p + 1);
            out[(size_t)r * d + 2 * p] = a * c - b * sn;
            out[(size_t)r * d + 2 * p + 1] = a * sn + b * c;
        }
    }
}

/* e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities; the
 * largest finite value is 448) -> value.  Code 0x7F / 0xFF (NaN) decode to NaN. */
double oracle_e4m3_decode(int code) {
    int sgn = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);                 /* subnormal: m/8 * 2^-6 */
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return sgn ? -v : v;
}

/* float -> e4m3 code, round to nearest (ties to even), saturating at +-448. */
int oracle_e4m3_encode(float x) {
    int sgn = signbit(x) ? 1 : 0;
    double a = fabs((double)x);
    if (a >= 448.0) return (sgn << 7) | 0x7E;
    /* quantum: 2^(E-3) for a normal value in [2^E, 2^(E+1)), 2^-9 below 2^-6 */
    int E = a > 0.0 ? (int)floor(log2(a)) : -7;
    if (E < -6) E = -6;
    double quantum = ldexp(1.0, E - 3);
    double n = nearbyint(a / quantum);                   /* ties to even (default mode) */
    double r = n * quantum;
    if (r > 448.0) r = 448.0;
    /* encode r */
    if (r < ldexp(1.0, -6)) return (sgn << 7) | (int)(r / ldexp(1.0, -9));
    int e = (int)floor(log2(r));
    int m = (int)((r / ldexp(1.0, e) - 1.0) * 8.0);
    return (sgn << 7) | ((e + 7) << 3) | m;
}

/* FP8 quantization of one tensor [B][H][Lp][d] per block of blk tokens.  smooth is
 * [B*H][d] fp32 (or NULL): y = x - smooth[bh] in fp32 for valid tokens, 0 for padded
 * ones; amax = max |y| over the block; inv = 448 / amax and scale = amax / 448 in fp32
 * (inv = scale = 1 for an all-zero block); code = e4m3(y * inv) in fp32.  codes has
 * the input's shape; scales is [B*H*nb] fp32. */
void oracle_quantize_fp8(int B, int H, int L, int Lp, int d, int blk, const void *x, int dtype,
                         const float *smooth, uint8_t *codes, float *scales) {
    int nb = Lp / blk;
    long units = (long)B * H * nb;
#pragma omp parallel for schedule(static) num_threads(oracle_threads_used())
    for (long u = 0; u < units; ++u) {
        long bh = u / nb;
        int t0 = (int)(u % nb) * blk;
        float amax = 0.0f;
        for (int t = t0; t < t0 + blk && t < L; ++t)
            for (int c = 0; c < d; ++c) {
                float y = (float)elem(x, dtype, ((size_t)bh * Lp + t) * d + c) - (smooth ? smooth[bh * d + c] : 0.0f);
                float ay = fabsf(y);
                if (ay > amax) amax = ay;
            }
        float inv = amax > 0.0f ? 448.0f / amax : 1.0f;
        scales[u] = amax > 0.0f ? amax / 448.0f : 1.0f;
        for (int t = t0; t < t0 + blk; ++t)
            for (int c = 0; c < d; ++c) {
                size_t i = ((size_t)bh * Lp + t) * d + c;
                if (t >= L) {
                    codes[i] = 0;
                    continue;
                }
                float y = (float)elem(x, dtype, i) - (smooth ? smooth[bh * d + c] : 0.0f);
                codes[i] = (uint8_t)oracle_e4m3_encode(y * inv);
            }
    }
}

/* e2m1 (1 sign, 2 exponent bits with bias 1, 1 mantissa bit, no infinities or NaN):
 * magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 for codes 0..7; bit 3 is the sign. */
double oracle_e2m1_decode(int code) {
    int sgn = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = e == 0 ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return sgn ? -v : v;
}

/* float -> e2m1 code: nearest grid value, a tie going to the even code (mantissa bit
 * 0), saturating at +-6.  The grid step is 0.5 below 2, 1 in [2, 4) and 2 in [4, 6];
 * inside each range the code is (range offset) + n with n = value / step, so the even
 * n of nearbyint (ties to even in the default rounding mode) is the even code. */
int oracle_e2m1_encode(float x) {
    int sgn = signbit(x) ? 1 : 0;
    double a = fabs((double)x);
    if (a >= 6.0) return (sgn << 3) | 7;
    double step = a < 2.0 ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
    double r = nearbyint(a / step) * step;
    int code;
    if (r < 2.0) code = (int)(r * 2.0);      /* 0, 0.5, 1, 1.5 -> 0..3 */
    else if (r < 4.0) code = (int)r + 2;     /* 2, 3 -> 4, 5 */
    else if (r < 6.0) code = 6;              /* 4 */
    else code = 7;                           /* 6 */
    return (sgn << 3) | code;
}

/* Byte offset of the scale of (row r, 16-element block kb) in a scale array for K
 * columns: atoms of 128 rows x 4 blocks (512 bytes), the atoms of one 128-row group
 * consecutive along K, and inside an atom row r at (r % 32) * 16 + ((r % 128) / 32) * 4,
 * block kb at + kb % 4. */
size_t oracle_nvfp4_sf_offset(int r, int kb, int K) {
    size_t atom = (size_t)(r / 128) * (size_t)(K / 64) + (size_t)(kb / 4);
    return atom * 512 + (size_t)(r % 32) * 16 + (size_t)((r % 128) / 32) * 4 + (size_t)(kb % 4);
}

/* NVFP4 quantization of a row-major [rows][K] matrix (K a multiple of 64).  codes is
 * [rows][K/2]: element 2i of a row in the low nibble of byte i, 2i+1 in the high
 * nibble.  sf holds ceil(rows/128)*128 * K/16 bytes in the layout of
 * oracle_nvfp4_sf_offset; rows beyond `rows` get scale 0.  amax is max |x| over these rows,
 * or amax_in when that is >= 0 (rows sampled from a larger tensor).  Returns the tensor
 * scale s = 2688 / amax (1 when the tensor is all zero). */
float oracle_nvfp4_quantize(int rows, int K, const void *x, int dtype, float amax_in, uint8_t *codes, uint8_t *sf) {
    float amax = 0.0f;
    for (size_t i = 0; i < (size_t)rows * K; ++i) {
        float a = fabsf((float)elem(x, dtype, i));
        if (a > amax) amax = a;
    }
    if (amax_in >= 0.0f) amax = amax_in; /* rows sampled from a larger tensor: its amax */
    const float s = amax > 0.0f ? 2688.0f / amax : 1.0f;
    const int rows_p = (rows + 127) / 128 * 128;
    memset(sf, 0, (size_t)rows_p * (K / 16));
#pragma omp parallel for schedule(static) num_threads(oracle_threads_used())
    for (int r = 0; r < rows; ++r) {
        for (int kb = 0; kb < K / 16; ++kb) {
            float bmax = 0.0f;
            for (int c = kb * 16; c < kb * 16 + 16; ++c) {
                float a = fabsf((float)elem(x, dtype, (size_t)r * K + c));
                if (a > bmax) bmax = a;
            }
            float scaled = (bmax / 6.0f) * s;
            int code_sf = oracle_e4m3_encode(scaled);
            sf[oracle_nvfp4_sf_offset(r, kb, K)] = (uint8_t)code_sf;
            float sf_f = (float)oracle_e4m3_decode(code_sf);
            float inv = sf_f > 0.0f ? s / sf_f : 0.0f;
            for (int c = kb * 16; c < kb * 16 + 16; c += 2) {
                int lo = oracle_e2m1_encode((float)elem(x, dtype, (size_t)r * K + c) * inv);
                int hi = oracle_e2m1_encode((float)elem(x, dtype, (size_t)r * K + c + 1) * inv);
                codes[((size_t)r * K + c) / 2] = (uint8_t)(lo | (hi << 4));
            }
        }
    }
    return s;
}

/* Decoded NVFP4 matrix in fp64: out[r][c] = e2m1(code) * e4m3(sf) / s. */
void oracle_nvfp4_dequantize(int rows, int K, const uint8_t *codes, const uint8_t *sf, float s, double *out) {
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < K; ++c) {
            uint8_t byte = codes[((size_t)r * K + c) / 2];
            int code = (c & 1) ? (byte >> 4) : (byte & 15);
            double scale = oracle_e4m3_decode(sf[oracle_nvfp4_sf_offset(r, c / 16, K)]);
            out[(size_t)r * K + c] = oracle_e2m1_decode(code) * scale / (double)s;
        }
}

/* Step 2, part a: one row of the block-score matrix, s_j = sum_c qm[i,c]*km[j,c],
 * and a_j = sum_c |qm[i,c]*km[j,c]| (the magnitude that bounds its rounding error). */
void oracle_score_row(int nb, int d, const double *qmean_bh, const double *kmean_bh,
                      int i, double *score, double *absum) {
    for (int j = 0; j < nb; ++j) {
        double s = 0.0, a = 0.0;
        for (int c = 0; c < d; ++c) {
            double p = qmean_bh[(size_t)i * d + c] * kmean_bh[(size_t)j * d + c];
            s += p;
            a += fabs(p);
        }
        score[j] = s;
        if (absum) absum[j] = a;
    }
}

typedef struct { double s; int j; } cand_t;

/* Descending score; equal scores: lower block index first. */
static int by_score_desc(const void *pa, const void *pb) {
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

static int by_int_asc(const void *pa, const void *pb) {
    int a = *(const int *)pa, b = *(const int *)pb;
    return (a > b) - (a < b);
}

/* Step 2, part b: diagonal plus the top k-1 of the rest, written ascending.
 * kth_score (nullable) receives, per row, the score of the last kept non-diagonal
 * block (or -inf when k == 1). */
int oracle_select(int B, int H, int nb, int d, int k,
                  const double *qmean, const double *kmean,
                  int32_t *col_idx, double *kth_score) {
    if (k < 1 || k > nb) return 1;
    long rows = (long)B * H * nb;
    int fail = 0;
#pragma omp parallel num_threads(oracle_threads_used())
    {
        double *score = (double *)malloc(sizeof(double) * (size_t)nb);
        cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)nb);
        int *keep = (int *)malloc(sizeof(int) * (size_t)k);
        if (!score || !cand || !keep) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(static)
            for (long r = 0; r < rows; ++r) {
                long bh = r / nb;
                int i = (int)(r % nb);
                oracle_score_row(nb, d, qmean + (size_t)bh * nb * d,
                                 kmean + (size_t)bh * nb * d, i, score, NULL);
                int n = 0;
                for (int j = 0; j < nb; ++j)
                    if (j != i) { cand[n].s = score[j]; cand[n].j = j; ++n; }
                qsort(cand, (size_t)n, sizeof(cand_t), by_score_desc);
                keep[0] = i;
                for (int q = 0; q < k - 1; ++q) keep[q + 1] = cand[q].j;
                qsort(keep, (size_t)k, sizeof(int), by_int_asc);
                for (int q = 0; q < k; ++q) col_idx[r * k + q] = keep[q];
                if (kth_score) kth_score[r] = k > 1 ? cand[k - 2].s : -INFINITY;
            }
        }
        free(score);
        free(cand);
        free(keep);
    }
    return fail ? 2 : 0;
}

/* Step 3: attention of one (b,h,query block) unit over its kept blocks.
 * out: [blk][d]; rows t >= L are 0.  Two passes: the max, then the exp sums. */
static void attend_unit(int L, int Lp, int d, int blk, long bh, int i,
                        const void *q, const void *kx, const void *v, int dtype,
                        const int32_t *cols, int ncols, double scale,
                        double *logit, double *out) {
    int nkeys = ncols * blk;
    for (int r = 0; r < blk; ++r) {
        int t = i * blk + r;
        double *o = out + (size_t)r * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        if (t >= L) continue;
        size_t qrow = ((size_t)bh * Lp + t) * d;
        double m = -INFINITY;
        for (int n = 0; n < nkeys; ++n) {
            int u = cols[n / blk] * blk + n % blk;
            logit[n] = -INFINITY;
            if (u >= L) continue;
            size_t krow = ((size_t)bh * Lp + u) * d;
            double s = 0.0;
            for (int c = 0; c < d; ++c)
                s += elem(q, dtype, qrow + c) * elem(kx, dtype, krow + c);
            logit[n] = s * scale;
            if (logit[n] > m) m = logit[n];
        }
        if (m == -INFINITY) continue; /* no valid key kept: output stays 0 */
        double den = 0.0;
        for (int n = 0; n < nkeys; ++n) {
            if (logit[n] == -INFINITY) continue;
            int u = cols[n / blk] * blk + n % blk;
            size_t vrow = ((size_t)bh * Lp + u) * d;
            double p = exp(logit[n] - m);
            den += p;
            for (int c = 0; c < d; ++c) o[c] += p * elem(v, dtype, vrow + c);
        }
        for (int c = 0; c < d; ++c) o[c] /= den;
    }
}

/* Step 3 over a list of units (unit = bh*nb + i), or all units when units == NULL.
 * CSR: row_ptr[unit]..row_ptr[unit+1] index col_idx.  out: [n_units][blk][d]. */
int oracle_attention(int B, int H, int L, int Lp, int d, int blk,
                     const void *q, const void *k, const void *v, int dtype,
                     const int32_t *row_ptr, const int32_t *col_idx, double scale,
                     long n_units, const int64_t *units, double *out) {
    int nb = Lp / blk;
    if (scale == 0.0) scale = 1.0 / sqrt((double)d);
    if (!units) n_units = (long)B * H * nb;
    int maxcols = 0;
    for (long u = 0; u < (long)B * H * nb; ++u) {
        int n = row_ptr[u + 1] - row_ptr[u];
        if (n > maxcols) maxcols = n;
    }
    int fail = 0;
#pragma omp parallel num_threads(oracle_threads_used())
    {
        double *logit = (double *)malloc(sizeof(double) * (size_t)(maxcols > 0 ? maxcols : 1) * blk);
        if (!logit) {
#pragma omp atomic write
            fail = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long n = 0; n < n_units; ++n) {
                long unit = units ? (long)units[n] : n;
                long bh = unit / nb;
                int i = (int)(unit % nb);
                int a = row_ptr[unit], b = row_ptr[unit + 1];
                attend_unit(L, Lp, d, blk, bh, i, q, k, v, dtype, col_idx + a, b - a,
                            scale, logit, out + (size_t)n * blk * d);
            }
        }
        free(logit);
    }
    return fail ? 2 : 0;
}
