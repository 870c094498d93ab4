/*
 * sia_oracle.c -- plain, slow CPU oracle for indexed sparse attention over paged caches.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this file:
 * only tests/, __graft_entry__.smoke() and the cpu_baseline / reference legs of bench.py use
 * it.  It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes follows the naive five-step decode chain printed in "Day 0 Inference
 * Adaptation and Performance Optimization for Hybrid Sparse Attention LLMs" (section
 * "Operator Fusion and Multi-Stream Scheduling"): score every historical position, weight and
 * sum the heads, pick the Top-K positions, gather those rows of the primary paged KV cache and
 * run softmax attention over them.  The index score is fixed as
 *      I[t,s] = sum_h w[t,h] * ReLU(q[t,h] . k[s])
 * (one index key per position shared by all heads), ties in Top-K go to the lower position,
 * and every floating-point value is carried in fp64.
 *
 * Readings of points the pages leave open:
 *   - causal: query j of sequence b at position p sees positions 0..p (itself included);
 *   - quantised index cache: value = e4m3 code decoded exactly, times its per-token scale
 *     ("high-precision computation + low-precision cache": dequantise, then compute);
 *   - Top-K output: the selected positions in ascending order, padded with -1 when fewer
 *     than K positions are visible;
 *   - the Top-K decision is taken on scores rounded to fp32, the precision the GPU ranks in
 *     (for the integer-valued inputs used in tests that rounding is exact);
 *   - attention (MLA absorbed form): logits use all DL+DR dims of the latent row, the output
 *     is the softmax-weighted sum of the first DL dims; lse is the natural-log sum-exp.
 *
 * Parity pins: tests/test_oracle.py checks every function here against closed forms,
 * brute force and special cases that do not reuse this code.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_INPUT 1

/* ---- element decoding (from the format definitions) -------------------------------------- */

/* bfloat16: the upper 16 bits of an IEEE-754 binary32. */
double oracle_bf16_value(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP FP8 E4M3 ("fn" variant): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
 * no infinities, S.1111.111 is NaN.  Exponent field 0 encodes subnormals 2^-6 * m/8. */
double oracle_e4m3_value(uint8_t bits) {
    int sign = (bits >> 7) & 1;
    int e = (bits >> 3) & 15;
    int m = bits & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m / 8.0, 1 - 7);
    else mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* OCP Microscaling (MX) E8M0 shared scale: an 8-bit exponent with bias 127, value 2^(e-127);
 * the code 0xFF is NaN.  No sign, no mantissa. */
double oracle_e8m0_value(uint8_t bits) {
    if (bits == 0xFF) return NAN;
    return ldexp(1.0, (int)bits - 127);
}

static double elem_value(const void* base, long idx, int fp8) {
    if (fp8) return oracle_e4m3_value(((const uint8_t*)base)[idx]);
    return oracle_bf16_value(((const uint16_t*)base)[idx]);
}

/* ---- step a1: page-table translation ---------------------------------------------------- */

/* Physical row (page * P + offset) holding logical position s of sequence b, or -1 when the
 * page id is outside the pool. */
static long physical_row(const int32_t* page_table, int max_pages, int P, int num_pages,
                         int b, int s) {
    int page = page_table[(long)b * max_pages + s / P];
    if (page < 0 || page >= num_pages) return -1;
    return (long)page * P + (s % P);
}

static int query_position(const int32_t* seq_lens, const int32_t* q_pos, int J, int b, int j) {
    if (q_pos) return q_pos[(long)b * J + j];
    return seq_lens[b] - J + j;
}

/* ---- steps a2-a4: relevance scoring, head-weighted aggregation, causal mask --------------- */

/*
 * scores[(b*J + j) * Lpad + s] for s <= p (p = the query's position), NaN elsewhere, with
 * Lpad = max_pages * P.  n_visible[b*J + j] = p + 1 (0 when p < 0).
 * rows: optional list of flattened (b*J + j) rows to compute (NULL = all of them).
 */
int oracle_index_scores(int B, int J, int H, int D, int P, int max_pages, int num_pages,
                        int fp8, const void* q, const float* q_scale, const float* w,
                        const void* k_cache, const float* k_scale,
                        const int32_t* page_table, const int32_t* seq_lens,
                        const int32_t* q_pos, const int32_t* rows, int n_rows,
                        double* scores, int32_t* n_visible) {
    long Lpad = (long)max_pages * P;
    int total = rows ? n_rows : B * J;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int r = 0; r < total; ++r) {
        int bj = rows ? rows[r] : r;
        int b = bj / J, j = bj % J;
        int p = query_position(seq_lens, q_pos, J, b, j);
        double* out = scores + (long)bj * Lpad;
        for (long s = 0; s < Lpad; ++s) out[s] = NAN;
        if (p >= seq_lens[b] || p >= Lpad) { bad = 1; n_visible[bj] = 0; continue; }
        n_visible[bj] = p + 1 > 0 ? p + 1 : 0;
        double qs = q_scale ? (double)q_scale[bj] : 1.0;
        for (int s = 0; s <= p; ++s) {
            long row = physical_row(page_table, max_pages, P, num_pages, b, s);
            if (row < 0) { bad = 1; continue; }
            double ks = k_scale ? (double)k_scale[row] : 1.0;
            double total_score = 0.0;
            for (int h = 0; h < H; ++h) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d) {
                    double qv = elem_value(q, ((long)bj * H + h) * D + d, fp8) * qs;
                    double kv = elem_value(k_cache, row * D + d, fp8) * ks;
                    dot += qv * kv;
                }
                double relu = dot > 0.0 ? dot : 0.0;
                total_score += (double)w[(long)bj * H + h] * relu;
            }
            out[s] = total_score;
        }
    }
    return bad ? ORACLE_BAD_INPUT : ORACLE_OK;
}

/*
 * MXFP8 index path (NEXT row; oracle only so far): "Rapid Adaptation and Inference
 * Optimization" (tiered quantization table: index Q/K in MXFP8, per group of 32) and "Day 0
 * Inference Adaptation..." (section 5.1: every 32 elements share one scaling factor).  q holds
 * e4m3 codes [B, J, H, D] with one E8M0 scale per 32 consecutive elements of each head vector
 * (q_mx [B, J, H, D/32]); the key cache holds e4m3 codes [num_pages, P, D] with one E8M0
 * scale per 32 consecutive elements of each key (k_mx [num_pages, P, D/32]).  Each element is
 * dequantised (code times its group's scale) and the score is then the one above:
 *      I[t,s] = sum_h w[t,h] * ReLU(sum_d q[t,h,d] k[s,d]).
 * D must be a multiple of 32.  Output as for oracle_index_scores.
 */
#define MX_GROUP 32
int oracle_index_scores_mx(int B, int J, int H, int D, int P, int max_pages, int num_pages,
                           const uint8_t* q, const uint8_t* q_mx, const float* w,
                           const uint8_t* k_cache, const uint8_t* k_mx,
                           const int32_t* page_table, const int32_t* seq_lens,
                           const int32_t* q_pos, const int32_t* rows, int n_rows,
                           double* scores, int32_t* n_visible) {
    if (D % MX_GROUP != 0) return ORACLE_BAD_INPUT;
    int G = D / MX_GROUP;
    long Lpad = (long)max_pages * P;
    int total = rows ? n_rows : B * J;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int r = 0; r < total; ++r) {
        int bj = rows ? rows[r] : r;
        int b = bj / J, j = bj % J;
        int p = query_position(seq_lens, q_pos, J, b, j);
        double* out = scores + (long)bj * Lpad;
        for (long s = 0; s < Lpad; ++s) out[s] = NAN;
        if (p >= seq_lens[b] || p >= Lpad) { bad = 1; n_visible[bj] = 0; continue; }
        n_visible[bj] = p + 1 > 0 ? p + 1 : 0;
        for (int s = 0; s <= p; ++s) {
            long row = physical_row(page_table, max_pages, P, num_pages, b, s);
            if (row < 0) { bad = 1; continue; }
            double total_score = 0.0;
            for (int h = 0; h < H; ++h) {
                long qh = (long)bj * H + h;
                double dot = 0.0;
                for (int d = 0; d < D; ++d) {
                    double qv = oracle_e4m3_value(q[qh * D + d]) * oracle_e8m0_value(q_mx[qh * G + d / MX_GROUP]);
                    double kv = oracle_e4m3_value(k_cache[row * D + d]) *
                                oracle_e8m0_value(k_mx[row * G + d / MX_GROUP]);
                    dot += qv * kv;
                }
                double relu = dot > 0.0 ? dot : 0.0;
                total_score += (double)w[(long)bj * H + h] * relu;
            }
            out[s] = total_score;
        }
    }
    return bad ? ORACLE_BAD_INPUT : ORACLE_OK;
}

/* ---- step a5: Top-K selection ------------------------------------------------------------ */

typedef struct { double score; int32_t pos; } scored_pos;

/* Rank order: larger score first; equal scores -> lower position first.  -0.0 and +0.0
 * compare equal, so the position decides between them. */
static int by_score_desc_pos_asc(const void* a, const void* b) {
    const scored_pos* x = (const scored_pos*)a;
    const scored_pos* y = (const scored_pos*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->pos > y->pos) - (x->pos < y->pos);
}

static int by_int_asc(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* One query row: the K best of scores[0..n_visible) -> out[0..K), ascending, -1 padded. */
int oracle_topk_row(const double* scores, int n_visible, int K, int32_t* out) {
    int take = n_visible < K ? n_visible : K;
    scored_pos* all = (scored_pos*)malloc(sizeof(scored_pos) * (size_t)(n_visible > 0 ? n_visible : 1));
    if (!all) return ORACLE_BAD_INPUT;
    for (int s = 0; s < n_visible; ++s) {
        all[s].score = (double)(float)scores[s]; /* rank in the GPU's precision */
        all[s].pos = s;
    }
    qsort(all, (size_t)n_visible, sizeof(scored_pos), by_score_desc_pos_asc);
    for (int i = 0; i < take; ++i) out[i] = all[i].pos;
    qsort(out, (size_t)take, sizeof(int32_t), by_int_asc);
    for (int i = take; i < K; ++i) out[i] = -1;
    free(all);
    return ORACLE_OK;
}

/* Rows of a score matrix [n_rows_total, Lpad] -> topk [n_rows_total, K]. */
int oracle_topk(const double* scores, const int32_t* n_visible, long Lpad, int K,
                const int32_t* rows, int n_rows, int total_rows, int32_t* topk) {
    int total = rows ? n_rows : total_rows;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int r = 0; r < total; ++r) {
        int bj = rows ? rows[r] : r;
        bad |= oracle_topk_row(scores + (long)bj * Lpad, n_visible[bj], K, topk + (long)bj * K);
    }
    return bad ? ORACLE_BAD_INPUT : ORACLE_OK;
}

/* ---- steps a6-a7: gather the selected latent rows, softmax attention --------------------- */

/* Elements of one token's main-cache row that share a scale in the FP8 cache: "Rapid
 * Adaptation and Inference Optimization" (tiered quantization table) and "Day 0 Inference
 * Adaptation..." (section 5.2) quantize the main KV cache in blocks of 128 elements per token
 * and head.  The MLA row (DL latent + DR rope elements, one KV head) is read as consecutive
 * blocks [0,128), [128,256), ...; the last block may be shorter (the 64 rope elements). */
#define KV_QUANT_BLOCK 128

/* Element d of physical main-cache row `row`: a bf16 value, or (fp8) the e4m3 code decoded
 * exactly times the fp32 scale of its block -- dequantise, then compute in fp64. */
static double kv_value(const void* kv, const float* kv_scale, int fp8, int DC, long row, int d) {
    if (!fp8) return oracle_bf16_value(((const uint16_t*)kv)[row * DC + d]);
    int nblk = (DC + KV_QUANT_BLOCK - 1) / KV_QUANT_BLOCK;
    return oracle_e4m3_value(((const uint8_t*)kv)[row * DC + d]) *
           (double)kv_scale[row * nblk + d / KV_QUANT_BLOCK];
}

/*
 * q   bf16 [B, J, H, DL+DR];  kv [num_pages, P, DL+DR] (see kv_value);  topk int32 [B, J, K]
 * (-1 = none)
 * out [B, J, H, DL] = sum_s softmax_s(z) * c[s][0:DL],  z_s = scale * q[h] . c[s]
 * lse [B, J, H]     = log sum_s exp(z_s)  (-inf and out = 0 when the list is empty)
 */
static int sparse_attend_rows(int B, int J, int H, int DL, int DR, int P, int max_pages,
                              int num_pages, double scale, const uint16_t* q, const void* kv,
                              const float* kv_scale, int kv_fp8, const int32_t* page_table,
                              const int32_t* seq_lens, const int32_t* topk, int K,
                              const int32_t* rows, int n_rows, double* out, double* lse) {
    int DC = DL + DR;
    int total = rows ? n_rows : B * J;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int r = 0; r < total; ++r) {
        int bj = rows ? rows[r] : r;
        int b = bj / J;
        const int32_t* sel = topk + (long)bj * K;
        long* phys = (long*)malloc(sizeof(long) * (size_t)K);
        double* z = (double*)malloc(sizeof(double) * (size_t)K);
        int n = 0;
        for (int i = 0; i < K; ++i) {
            int s = sel[i];
            if (s < 0) continue;
            if (s >= seq_lens[b]) { bad = 1; continue; }
            long row = physical_row(page_table, max_pages, P, num_pages, b, s);
            if (row < 0) { bad = 1; continue; }
            phys[n++] = row;
        }
        for (int h = 0; h < H; ++h) {
            const uint16_t* qh = q + ((long)bj * H + h) * DC;
            double* oh = out + ((long)bj * H + h) * DL;
            double m = -INFINITY;
            for (int i = 0; i < n; ++i) {
                double dot = 0.0;
                for (int d = 0; d < DC; ++d)
                    dot += oracle_bf16_value(qh[d]) * kv_value(kv, kv_scale, kv_fp8, DC, phys[i], d);
                z[i] = scale * dot;
                if (z[i] > m) m = z[i];
            }
            double denom = 0.0;
            for (int i = 0; i < n; ++i) denom += exp(z[i] - m);
            for (int d = 0; d < DL; ++d) {
                double acc = 0.0;
                for (int i = 0; i < n; ++i) acc += exp(z[i] - m) * kv_value(kv, kv_scale, kv_fp8, DC, phys[i], d);
                oh[d] = n > 0 ? acc / denom : 0.0;
            }
            lse[(long)bj * H + h] = n > 0 ? m + log(denom) : -INFINITY;
        }
        free(phys);
        free(z);
    }
    return bad ? ORACLE_BAD_INPUT : ORACLE_OK;
}

/* bf16 main cache. */
int oracle_sparse_attend(int B, int J, int H, int DL, int DR, int P, int max_pages,
                         int num_pages, double scale, const uint16_t* q, const uint16_t* kv,
                         const int32_t* page_table, const int32_t* seq_lens,
                         const int32_t* topk, int K, const int32_t* rows, int n_rows,
                         double* out, double* lse) {
    return sparse_attend_rows(B, J, H, DL, DR, P, max_pages, num_pages, scale, q, kv, NULL, 0,
                              page_table, seq_lens, topk, K, rows, n_rows, out, lse);
}

/* FP8 main cache: kv holds e4m3 codes [num_pages, P, DL+DR]; kv_scale fp32
 * [num_pages, P, ceil((DL+DR) / 128)], one scale per block of the token's row. */
int oracle_sparse_attend_fp8kv(int B, int J, int H, int DL, int DR, int P, int max_pages,
                               int num_pages, double scale, const uint16_t* q, const uint8_t* kv,
                               const float* kv_scale, const int32_t* page_table,
                               const int32_t* seq_lens, const int32_t* topk, int K,
                               const int32_t* rows, int n_rows, double* out, double* lse) {
    return sparse_attend_rows(B, J, H, DL, DR, P, max_pages, num_pages, scale, q, kv, kv_scale, 1,
                              page_table, seq_lens, topk, K, rows, n_rows, out, lse);
}

/*
 * Second, independent formulation used to pin the first: dense attention of the query over
 * every causal position 0..p, with the logit of each position outside the allowed set forced
 * to -inf before the softmax.  allowed: uint8 [B*J, Lpad] (1 = take part).
 */
int oracle_dense_masked_attend(int B, int J, int H, int DL, int DR, int P, int max_pages,
                               int num_pages, double scale, const uint16_t* q,
                               const uint16_t* kv, const int32_t* page_table,
                               const int32_t* seq_lens, const int32_t* q_pos,
                               const uint8_t* allowed, double* out, double* lse) {
    int DC = DL + DR;
    long Lpad = (long)max_pages * P;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int bj = 0; bj < B * J; ++bj) {
        int b = bj / J, j = bj % J;
        int p = query_position(seq_lens, q_pos, J, b, j);
        double* logits = (double*)malloc(sizeof(double) * (size_t)(p + 1 > 0 ? p + 1 : 1));
        for (int h = 0; h < H; ++h) {
            const uint16_t* qh = q + ((long)bj * H + h) * DC;
            for (int s = 0; s <= p; ++s) {
                long row = physical_row(page_table, max_pages, P, num_pages, b, s);
                if (row < 0) { bad = 1; logits[s] = -INFINITY; continue; }
                if (!allowed[(long)bj * Lpad + s]) { logits[s] = -INFINITY; continue; }
                double dot = 0.0;
                for (int d = 0; d < DC; ++d)
                    dot += oracle_bf16_value(qh[d]) * oracle_bf16_value(kv[row * DC + d]);
                logits[s] = scale * dot;
            }
            double m = -INFINITY;
            for (int s = 0; s <= p; ++s) if (logits[s] > m) m = logits[s];
            double* oh = out + ((long)bj * H + h) * DL;
            if (m == -INFINITY) {
                for (int d = 0; d < DL; ++d) oh[d] = 0.0;
                lse[(long)bj * H + h] = -INFINITY;
                continue;
            }
            double denom = 0.0;
            for (int s = 0; s <= p; ++s) denom += exp(logits[s] - m);
            for (int d = 0; d < DL; ++d) {
                double acc = 0.0;
                for (int s = 0; s <= p; ++s) {
                    if (logits[s] == -INFINITY) continue;
                    long row = physical_row(page_table, max_pages, P, num_pages, b, s);
                    acc += exp(logits[s] - m) * oracle_bf16_value(kv[row * DC + d]);
                }
                oh[d] = acc / denom;
            }
            lse[(long)bj * H + h] = m + log(denom);
        }
        free(logits);
    }
    return bad ? ORACLE_BAD_INPUT : ORACLE_OK;
}

/* ---- paged cache append (NEXT row; oracle only so far) ---------------------------------- */

/* e4m3 encoding of an fp32 value, from the format definition: round to the nearest value of
 * the e4m3 grid (3 mantissa bits; below 2^-6 the subnormal step 2^-9), ties to the even
 * code; magnitudes at or above 448 give +-448 (saturation); NaN gives 0x7F. */
uint8_t oracle_e4m3_encode(float x) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double v = fabs((double)x);
    if (v >= 448.0) return sign | 0x7E;
    int e = v > 0.0 ? (int)floor(log2(v)) : -6;
    if (e < -6) e = -6;                       /* subnormal range: fixed step 2^-9 */
    while (ldexp(1.0, e) > v && e > -6) --e;  /* guard log2 rounding at binade edges */
    while (ldexp(1.0, e + 1) <= v) ++e;
    double step = ldexp(1.0, e - 3);
    double r = rint(v / step) * step;          /* v / step is exact; rint rounds half to even */
    if (r == 0.0) return sign;
    int re = (int)floor(log2(r));
    while (ldexp(1.0, re) > r) --re;
    while (ldexp(1.0, re + 1) <= r) ++re;
    if (re < -6) return sign | (uint8_t)(r / ldexp(1.0, -9));             /* subnormal code */
    return sign | (uint8_t)((re + 7) << 3) | (uint8_t)(r / ldexp(1.0, re - 3) - 8.0);
}

static float absmax_f(const float* x, int n) {
    float m = 0.0f;
    for (int i = 0; i < n; ++i) if (fabsf(x[i]) > m) m = fabsf(x[i]);
    return m;
}

/* Per-token FP8 index key: scale = the smallest power of two s with amax <= 448 s (1 for an
 * all-zero key); codes = e4m3(x / s), the division being exact. */
static float quantise_key_pow2(const float* x, int n, uint8_t* codes) {
    float amax = absmax_f(x, n);
    int e = 0;
    if (amax > 0.0f) {
        e = -160;
        while ((double)amax > 448.0 * ldexp(1.0, e)) ++e;
    }
    float s = (float)ldexp(1.0, e);
    for (int i = 0; i < n; ++i) codes[i] = oracle_e4m3_encode((float)ldexp((double)x[i], -e));
    return s;
}

/* FP8 main-cache block: scale = fp32(amax / 448) (1 for an all-zero block); codes =
 * e4m3(fp32(x / scale)), both divisions rounded to fp32 as a GPU computes them. */
static float quantise_block_amax(const float* x, int n, uint8_t* codes) {
    float amax = absmax_f(x, n);
    volatile float s = amax > 0.0f ? amax / 448.0f : 1.0f;
    for (int i = 0; i < n; ++i) {
        volatile float y = x[i] / s;
        codes[i] = oracle_e4m3_encode(y);
    }
    return s;
}

/* MX group (OCP Microscaling): shared exponent E = floor(log2 amax) - 8 (8 = the largest
 * e4m3 exponent), clamped to the E8M0 range [-127, 127]; scale code E + 127 (127 for an
 * all-zero group); codes = e4m3(x / 2^E), saturating. */
static uint8_t quantise_group_mx(const float* x, int n, uint8_t* codes) {
    float amax = absmax_f(x, n);
    int E = 0;
    if (amax > 0.0f) {
        int f = (int)floor(log2((double)amax));
        while (ldexp(1.0, f) > (double)amax) --f;
        while (ldexp(1.0, f + 1) <= (double)amax) ++f;
        E = f - 8;
        if (E < -127) E = -127;
        if (E > 127) E = 127;
    }
    for (int i = 0; i < n; ++i) codes[i] = oracle_e4m3_encode((float)ldexp((double)x[i], -E));
    return (uint8_t)(E + 127);
}

/*
 * Write the J new tokens of every sequence into the paged caches: token j of sequence b sits
 * at position p = seq_lens[b] - J + j (seq_lens counts the new tokens) and goes to row p % P
 * of page page_table[b][p / P].
 *   new_k  fp32 [B, J, D]      -> index cache, by k_mode:
 *          0: bf16 bits (k_cache uint16 [pages, P, D]; the input must already be bf16 values)
 *          1: e4m3 codes + per-token power-of-two scale (k_cache uint8, k_scale fp32 [pages, P])
 *          2: MXFP8 codes + one E8M0 code per 32 elements (k_scale read as uint8 [pages, P, D/32])
 *   new_kv fp32 [B, J, DC]     -> main cache, by kv_mode:
 *          0: bf16 bits (kv_cache uint16 [pages, P, DC])
 *          1: e4m3 codes + fp32 scale per 128-element block (kv_scale [pages, P, ceil(DC/128)])
 * Rows not written keep their contents.  A page id outside the pool skips the token and
 * reports ORACLE_BAD_INPUT.
 */
int oracle_cache_append(int B, int J, int D, int DC, int P, int max_pages, int num_pages,
                        const int32_t* page_table, const int32_t* seq_lens,
                        const float* new_k, int k_mode, void* k_cache, void* k_scale,
                        const float* new_kv, int kv_mode, void* kv_cache, float* kv_scale) {
    int bad = 0;
    int nblk = (DC + KV_QUANT_BLOCK - 1) / KV_QUANT_BLOCK;
    if (k_mode == 2 && D % MX_GROUP != 0) return ORACLE_BAD_INPUT;
    for (int b = 0; b < B; ++b) {
        for (int j = 0; j < J; ++j) {
            int p = seq_lens[b] - J + j;
            if (p < 0 || p >= max_pages * P) { bad = 1; continue; }
            long row = physical_row(page_table, max_pages, P, num_pages, b, p);
            if (row < 0) { bad = 1; continue; }
            const float* xk = new_k + ((long)b * J + j) * D;
            if (k_mode == 0) {
                for (int d = 0; d < D; ++d) {
                    uint32_t u;
                    memcpy(&u, &xk[d], sizeof u);
                    ((uint16_t*)k_cache)[row * D + d] = (uint16_t)(u >> 16);
                }
            } else if (k_mode == 1) {
                ((float*)k_scale)[row] = quantise_key_pow2(xk, D, (uint8_t*)k_cache + row * D);
            } else {
                for (int g = 0; g < D / MX_GROUP; ++g)
                    ((uint8_t*)k_scale)[row * (D / MX_GROUP) + g] =
                        quantise_group_mx(xk + g * MX_GROUP, MX_GROUP, (uint8_t*)k_cache + row * D + g * MX_GROUP);
            }
            const float* xv = new_kv + ((long)b * J + j) * DC;
            if (kv_mode == 0) {
                for (int d = 0; d < DC; ++d) {
                    uint32_t u;
                    memcpy(&u, &xv[d], sizeof u);
                    ((uint16_t*)kv_cache)[row * DC + d] = (uint16_t)(u >> 16);
                }
            } else {
                for (int g = 0; g < nblk; ++g) {
                    int lo = g * KV_QUANT_BLOCK, n = DC - lo < KV_QUANT_BLOCK ? DC - lo : KV_QUANT_BLOCK;
                    kv_scale[row * nblk + g] = quantise_block_amax(xv + lo, n, (uint8_t*)kv_cache + row * DC + lo);
                }
            }
        }
    }
    return bad ? ORACLE_BAD_INPUT : ORACLE_OK;
}

/* Number of threads the OpenMP runtime uses for the loops above (1 without OpenMP). */
#ifdef _OPENMP
#include <omp.h>
int oracle_num_threads(void) { return omp_get_max_threads(); }
void oracle_set_num_threads(int n) { omp_set_num_threads(n); }
#else
int oracle_num_threads(void) { return 1; }
void oracle_set_num_threads(int n) { (void)n; }
#endif
