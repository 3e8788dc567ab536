/*
 * oracle.c -- plain, slow, obviously-correct CPU oracle for one decode step of
 * attention over a paged KV cache.  TEST INFRASTRUCTURE ONLY: it is called by
 * the tests, by the package's smoke check and by the benchmark's CPU-baseline
 * leg, never by the product path.  It shares no code, header or constant
 * generator with the CUDA library.
 *
 * Sources (the three web pages this method is described on):
 *   [KVF]  "推理速度慢怎么办？KV Cache与Flash Attention如何加速大模型推理" (ipipp.com)
 *   [LES]  "KV缓存与Flash注意力" (FANDEX course lesson)
 *   [BLOG] "KV Cache:推理慢的真正原因" (cybercheems.top)
 *
 * Every floating-point quantity is computed in IEEE binary64.  fp16 / bf16
 * storage values are decoded exactly (every binary16 / bfloat16 value is a
 * binary64 value).  Nothing is blocked, fused or reordered beyond what the
 * definitions state.
 *
 * Functions and what pins them (tests/test_oracle_pins.py):
 *   orc_f16_to_f64 / orc_bf16_to_f64  -- numpy float16 / torch bfloat16 decoders
 *   orc_kv_bytes_per_token            -- worked numbers printed on [BLOG] and [LES]
 *   orc_append                        -- cached == naive toy decoder; canary pool
 *   orc_attend                        -- CPU float64 SDPA, independent brute force,
 *                                        closed forms, GQA == repeated-head MHA
 *   orc_attend_tiled                  -- equals orc_attend (flash is exact)
 *   orc_merge                         -- merge of disjoint partitions == one shot
 *   orc_e4m3_decode / orc_e4m3_encode -- torch float8_e4m3fn (all codes; RN ties)
 *   orc_quantize_fp8 / orc_append_fp8 -- round-trip bound, per-group scales,
 *                                        outlier isolation, == numpy re-derivation
 *   orc_attend_fp8                    -- CPU float64 SDPA on the dequantised cache
 *   orc_int8_decode / orc_int8_encode -- numpy int8 view; closed-form roundings
 *   orc_quantize_int8 / orc_append_int8 / orc_attend_int8
 *                                     -- half-step round trip, extreme -> +-127,
 *                                        CPU float64 SDPA on the dequantised cache
 *   orc_int4_decode / orc_int4_encode -- two's complement nibbles; closed-form roundings
 *   orc_quantize_int4 / orc_append_int4 / orc_attend_int4
 *                                     -- half-step round trip, extreme -> +-7, nibble
 *                                        order, CPU float64 SDPA on the dequantised cache
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* [BLOG] section "工程优化手段 / PagedAttention": the cache is cut into fixed
 * blocks of 16 tokens and a block table maps logical to physical blocks. */
#define ORC_PAGE_TOKENS 16

enum { ORC_F16 = 0, ORC_BF16 = 1 };
enum { ORC_OK = 0, ORC_ERR_ARGS = 1, ORC_ERR_RANGE = 2, ORC_ERR_NOMEM = 3 };

/* ---------------------------------------------------------------- decoding */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double orc_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double v;
    if (expo == 0) {
        v = ldexp((double)frac, -24);              /* subnormal: frac * 2^-24 */
    } else if (expo == 31) {
        v = frac ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + frac), expo - 25); /* (1.frac) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32 word. */
double orc_bf16_to_f64(uint16_t b)
{
    uint32_t bits = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double decode_elem(uint16_t x, int dtype)
{
    return dtype == ORC_BF16 ? orc_bf16_to_f64(x) : orc_f16_to_f64(x);
}

/* ------------------------------------------------------------ byte formula */

/* [BLOG] section "显存账": bytes per token = 2 (K and V) x dtype bytes x L x H x d_head.
 * [KVF] section "一、KV Cache" gives the same count times B and N. */
long long orc_kv_bytes_per_token(int layers, int heads, int d_head, int dtype_size)
{
    return 2LL * (long long)dtype_size * layers * heads * d_head;
}

/* ------------------------------------------------------------------ append */

/* [BLOG] section "缓存的是什么" (KVCache.append writes the new step's K/V at
 * position `length`), made paged by section "PagedAttention": the token at
 * logical position pos lives in physical block block_table[b][pos / 16] at
 * row pos % 16.  Cache layout [num_blocks][H_kv][16][d]; k_new, v_new
 * [B][H_kv][d]; storage words are copied verbatim.  slot[b] < 0 skips b. */
int orc_append(uint16_t *k_cache, uint16_t *v_cache, const int32_t *block_table,
               const int32_t *slot, const uint16_t *k_new, const uint16_t *v_new,
               int B, int H_kv, int d, int num_blocks, int max_blocks)
{
    if (!k_cache || !v_cache || !block_table || !slot || !k_new || !v_new) return ORC_ERR_ARGS;
    if (B < 0 || H_kv <= 0 || d <= 0 || num_blocks <= 0 || max_blocks <= 0) return ORC_ERR_ARGS;
    for (int b = 0; b < B; ++b) {
        int pos = slot[b];
        if (pos < 0) continue;
        int logical = pos / ORC_PAGE_TOKENS;
        int row = pos % ORC_PAGE_TOKENS;
        if (logical >= max_blocks) return ORC_ERR_RANGE;
        int phys = block_table[(size_t)b * max_blocks + logical];
        if (phys < 0 || phys >= num_blocks) return ORC_ERR_RANGE;
        for (int h = 0; h < H_kv; ++h) {
            size_t dst = (((size_t)phys * H_kv + h) * ORC_PAGE_TOKENS + row) * (size_t)d;
            size_t src = ((size_t)b * H_kv + h) * (size_t)d;
            memcpy(k_cache + dst, k_new + src, (size_t)d * sizeof(uint16_t));
            memcpy(v_cache + dst, v_new + src, (size_t)d * sizeof(uint16_t));
        }
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------- attention */

/* Address of token j of sequence b, KV head g, in the paged pool (or -1). */
static long long token_offset(const int32_t *block_table, int b, int j, int g,
                              int H_kv, int d, int num_blocks, int max_blocks)
{
    int logical = j / ORC_PAGE_TOKENS;
    if (logical >= max_blocks) return -1;
    int phys = block_table[(size_t)b * max_blocks + logical];
    if (phys < 0 || phys >= num_blocks) return -1;
    return (long long)((((size_t)phys * H_kv + g) * ORC_PAGE_TOKENS + (j % ORC_PAGE_TOKENS)) * (size_t)d);
}

static int check_common(const void *q, const void *kc, const void *vc, const int32_t *bt,
                        const int32_t *seq_lens, int B, int H_q, int H_kv, int d,
                        int num_blocks, int max_blocks, int dtype)
{
    if (!q || !kc || !vc || !bt || !seq_lens) return ORC_ERR_ARGS;
    if (B < 0 || H_q <= 0 || H_kv <= 0 || d <= 0 || num_blocks <= 0 || max_blocks <= 0) return ORC_ERR_ARGS;
    if (H_q % H_kv != 0) return ORC_ERR_ARGS;
    if (dtype != ORC_F16 && dtype != ORC_BF16) return ORC_ERR_ARGS;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] < 0 || seq_lens[b] > max_blocks * ORC_PAGE_TOKENS) return ORC_ERR_RANGE;
    return ORC_OK;
}

/*
 * One-shot attention of each query row over its cached tokens.
 *   [KVF] section "一、KV Cache" (forward_with_kv_cache): scores = q K^T * scale,
 *   softmax over all cached tokens including the one just appended, output =
 *   weights . V.  No causal mask: the decode query is the last position.
 *   [BLOG] section "工程优化手段 / GQA": several query heads share one KV head;
 *   query head hq reads KV head hq / (H_q / H_kv).
 * Token range per sequence: [lo[b], hi[b]) when lo/hi are given, else
 * [0, seq_lens[b]).  Per row: m = max_j s_j, w_j = exp(s_j - m),
 * out = sum_j w_j v_j / sum_j w_j, lse = m + ln sum_j w_j.  An empty range
 * gives out = 0 and lse = -inf.
 * q [B][H_q][d] storage words; out [B][H_q][d] and lse [B][H_q] binary64.
 */
int orc_attend(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
               const int32_t *block_table, const int32_t *seq_lens,
               const int32_t *lo, const int32_t *hi, double scale,
               int B, int H_q, int H_kv, int d, int num_blocks, int max_blocks, int dtype,
               double *out, double *lse, int nthreads)
{
    int rc = check_common(q, k_cache, v_cache, block_table, seq_lens, B, H_q, H_kv, d,
                          num_blocks, max_blocks, dtype);
    if (rc) return rc;
    if (!out) return ORC_ERR_ARGS;
    const int G = H_q / H_kv;
    int status = ORC_OK;
    long long rows = (long long)B * H_q;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (long long r = 0; r < rows; ++r) {
        int b = (int)(r / H_q), hq = (int)(r % H_q), g = hq / G;
        int j0 = lo ? lo[b] : 0;
        int j1 = hi ? hi[b] : seq_lens[b];
        double *o = out + (size_t)r * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        if (j0 < 0 || j1 > seq_lens[b]) { status = ORC_ERR_RANGE; continue; }
        if (j1 <= j0) { if (lse) lse[r] = -INFINITY; continue; }
        int n = j1 - j0;
        double *s = (double *)malloc((size_t)n * sizeof(double));
        double *qv = (double *)malloc((size_t)d * sizeof(double));
        if (!s || !qv) { free(s); free(qv); status = ORC_ERR_NOMEM; continue; }
        for (int i = 0; i < d; ++i) qv[i] = decode_elem(q[(size_t)r * d + i], dtype);
        int bad = 0;
        for (int j = j0; j < j1; ++j) {
            long long off = token_offset(block_table, b, j, g, H_kv, d, num_blocks, max_blocks);
            if (off < 0) { bad = 1; break; }
            double dot = 0.0;
            for (int i = 0; i < d; ++i) dot += qv[i] * decode_elem(k_cache[off + i], dtype);
            s[j - j0] = scale * dot;
        }
        if (bad) { free(s); free(qv); status = ORC_ERR_RANGE; continue; }
        double m = -INFINITY;
        for (int t = 0; t < n; ++t) if (s[t] > m) m = s[t];
        double den = 0.0;
        for (int j = j0; j < j1; ++j) {
            double w = exp(s[j - j0] - m);
            den += w;
            long long off = token_offset(block_table, b, j, g, H_kv, d, num_blocks, max_blocks);
            for (int i = 0; i < d; ++i) o[i] += w * decode_elem(v_cache[off + i], dtype);
        }
        for (int i = 0; i < d; ++i) o[i] /= den;
        if (lse) lse[r] = m + log(den);
        free(s);
        free(qv);
    }
    return status;
}

/*
 * Tiled online softmax, [LES] section "步骤2:分块softmax" (tiled_softmax_dot),
 * with the score scale of [KVF] added.  Walk the tokens in tiles of `tile`;
 * keep a running maximum m and a running sum s; on each tile rescale the
 * previous sum and output by exp(m_old - m_new) (zero before the first tile)
 * and add the tile's exp(score - m_new) terms.  Result out / s.  Used only to
 * show that tiling returns the one-shot result.
 */
int orc_attend_tiled(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                     const int32_t *block_table, const int32_t *seq_lens, double scale,
                     int B, int H_q, int H_kv, int d, int num_blocks, int max_blocks, int dtype,
                     int tile, double *out)
{
    int rc = check_common(q, k_cache, v_cache, block_table, seq_lens, B, H_q, H_kv, d,
                          num_blocks, max_blocks, dtype);
    if (rc) return rc;
    if (!out || tile <= 0) return ORC_ERR_ARGS;
    const int G = H_q / H_kv;
    double *qv = (double *)malloc((size_t)d * sizeof(double));
    double *acc = (double *)malloc((size_t)d * sizeof(double));
    double *sc = (double *)malloc((size_t)tile * sizeof(double));
    if (!qv || !acc || !sc) { free(qv); free(acc); free(sc); return ORC_ERR_NOMEM; }
    for (int b = 0; b < B; ++b) {
        for (int hq = 0; hq < H_q; ++hq) {
            int g = hq / G;
            size_t r = (size_t)b * H_q + hq;
            int n = seq_lens[b];
            for (int i = 0; i < d; ++i) { qv[i] = decode_elem(q[r * d + i], dtype); acc[i] = 0.0; }
            double m = -INFINITY, ssum = 0.0;
            for (int start = 0; start < n; start += tile) {
                int cnt = n - start < tile ? n - start : tile;
                double new_m = m;
                for (int t = 0; t < cnt; ++t) {
                    long long off = token_offset(block_table, b, start + t, g, H_kv, d, num_blocks, max_blocks);
                    if (off < 0) { free(qv); free(acc); free(sc); return ORC_ERR_RANGE; }
                    double dot = 0.0;
                    for (int i = 0; i < d; ++i) dot += qv[i] * decode_elem(k_cache[off + i], dtype);
                    sc[t] = scale * dot;
                    if (sc[t] > new_m) new_m = sc[t];
                }
                double exp_old = (m == -INFINITY) ? 0.0 : exp(m - new_m);
                double tile_sum = 0.0;
                for (int t = 0; t < cnt; ++t) { sc[t] = exp(sc[t] - new_m); tile_sum += sc[t]; }
                ssum = ssum * exp_old + tile_sum;
                for (int i = 0; i < d; ++i) {
                    double add = 0.0;
                    for (int t = 0; t < cnt; ++t) {
                        long long off = token_offset(block_table, b, start + t, g, H_kv, d, num_blocks, max_blocks);
                        add += sc[t] * decode_elem(v_cache[off + i], dtype);
                    }
                    acc[i] = acc[i] * exp_old + add;
                }
                m = new_m;
            }
            for (int i = 0; i < d; ++i) out[r * d + i] = n > 0 ? acc[i] / ssum : 0.0;
        }
    }
    free(qv); free(acc); free(sc);
    return ORC_OK;
}

/*
 * Merge of S partial results of one row, each the attention over a disjoint
 * part of the tokens: partial o_s (normalised) and lse_s = m_s + ln l_s.
 * Combining two running (max, sum, out) states is the rescale step of [LES]
 * "步骤2:分块softmax" applied to whole partitions:
 *   LSE = M + ln sum_s exp(lse_s - M), M = max_s lse_s,
 *   out = sum_s exp(lse_s - LSE) o_s.
 * Partitions with lse = -inf carry no weight; if all are empty, out = 0 and
 * LSE = -inf.  Layout: part_o [B][H_q][S][d], part_lse [B][H_q][S]; counts[b]
 * (nullable) limits sequence b to its first counts[b] partials.
 */
int orc_merge(const double *part_o, const double *part_lse, const int32_t *counts,
              int B, int H_q, int d, int S, double *out, double *lse)
{
    if (!part_o || !part_lse || !out || B < 0 || H_q <= 0 || d <= 0 || S <= 0) return ORC_ERR_ARGS;
    for (int b = 0; b < B; ++b) {
        int ns = counts ? counts[b] : S;
        if (ns < 0 || ns > S) return ORC_ERR_RANGE;
        for (int h = 0; h < H_q; ++h) {
            size_t r = (size_t)b * H_q + h;
            const double *L = part_lse + r * S;
            double M = -INFINITY;
            for (int s = 0; s < ns; ++s) if (L[s] > M) M = L[s];
            double *o = out + r * d;
            for (int i = 0; i < d; ++i) o[i] = 0.0;
            if (M == -INFINITY) { if (lse) lse[r] = -INFINITY; continue; }
            double tot = 0.0;
            for (int s = 0; s < ns; ++s) tot += exp(L[s] - M);
            double LSE = M + log(tot);
            for (int s = 0; s < ns; ++s) {
                double w = exp(L[s] - LSE);
                if (w == 0.0) continue;
                const double *po = part_o + (r * S + s) * d;
                for (int i = 0; i < d; ++i) o[i] += w * po[i];
            }
            if (lse) lse[r] = LSE;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------- 8-bit KV cache */

/* "KV Cache:推理慢的真正原因", section "工程优化手段 / 量化": the cache is stored in
 * 8 bits; because a few keys are very large, the scale is taken per channel
 * group rather than one for the whole tensor.  "KV缓存与Flash注意力", section
 * "实际应用" (serving with an fp8 KV cache).  Reading taken here: FP8 E4M3
 * codes with one fp32 scale per (token, KV head, group of 32 channels);
 * s = max|x| / 448 (448 = largest E4M3 value), code = E4M3(x / s) rounded to
 * nearest (ties to even), saturating at +-448; both divisions are IEEE fp32
 * (the precision the kernels use, since the fp32 quotient decides the code).
 * A group of zeros gets s = 0 and codes 0.  Dequantised value: s * E4M3(code). */
#define ORC_FP8_GROUP 32

/* E4M3 ("fn" variant): 1 sign, 4 exponent bits (bias 7), 3 fraction bits; no
 * infinities; exponent 15 with fraction 7 is NaN; subnormals fraction * 2^-9. */
double orc_e4m3_decode(uint8_t c)
{
    int sign = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp((double)(8 + m), e - 10);
    return sign ? -v : v;
}

uint8_t orc_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a < ldexp(1.0, -6)) {                 /* subnormal range: multiples of 2^-9 */
        double r = rint(a / ldexp(1.0, -9));  /* nearest, ties to even; 8 = smallest normal */
        return sign | (uint8_t)r;
    }
    int e2;
    frexp(a, &e2);                            /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;                           /* a = 1.xxx * 2^E */
    double r = rint(a / ldexp(1.0, E - 3));   /* in [8, 16] */
    if (r == 16.0) { r = 8.0; E += 1; }
    int biased = E + 7;
    int frac = (int)r - 8;
    if (biased > 15 || (biased == 15 && frac == 7)) return sign | 0x7E;   /* saturate at 448 */
    return sign | (uint8_t)((biased << 3) | frac);
}

/* Quantise n rows of d storage words (fp16/bf16) into codes [n][d] and
 * scales [n][d / 32]. */
int orc_quantize_fp8(const uint16_t *rows, int n, int d, int dtype, uint8_t *codes, float *scales)
{
    if (!rows || !codes || !scales || n < 0 || d <= 0 || d % ORC_FP8_GROUP) return ORC_ERR_ARGS;
    const int ng = d / ORC_FP8_GROUP;
    for (long long r = 0; r < n; ++r) {
        for (int g = 0; g < ng; ++g) {
            const uint16_t *x = rows + r * d + g * ORC_FP8_GROUP;
            float mx = 0.0f;
            for (int i = 0; i < ORC_FP8_GROUP; ++i) {
                float v = (float)fabs(decode_elem(x[i], dtype));
                if (v > mx) mx = v;
            }
            volatile float s = mx / 448.0f;
            scales[r * ng + g] = s;
            for (int i = 0; i < ORC_FP8_GROUP; ++i) {
                float v = (float)decode_elem(x[i], dtype);
                volatile float q = s == 0.0f ? 0.0f : v / s;
                codes[r * d + g * ORC_FP8_GROUP + i] = s == 0.0f ? 0 : orc_e4m3_encode(q);
            }
        }
    }
    return ORC_OK;
}

/* Append for an 8-bit cache: quantise k_new/v_new [B][H_kv][d] with `quant`
 * and write the codes and scales of row slot[b] % 16 of page
 * block_table[b][slot[b] / 16] (codes [NB][H_kv][16][d], scales
 * [NB][H_kv][16][d/32]). */
typedef int (*orc_quant_fn)(const uint16_t *, int, int, int, uint8_t *, float *);

/* row_bytes: bytes of codes per cache row (d for 8-bit codes, d / 2 for 4-bit). */
static int append_codes(uint8_t *k8, uint8_t *v8, float *ks, float *vs, const int32_t *block_table,
                        const int32_t *slot, const uint16_t *k_new, const uint16_t *v_new, int B,
                        int H_kv, int d, int row_bytes, int num_blocks, int max_blocks, int dtype,
                        orc_quant_fn quant)
{
    if (!k8 || !v8 || !ks || !vs || !block_table || !slot || !k_new || !v_new) return ORC_ERR_ARGS;
    if (d % ORC_FP8_GROUP) return ORC_ERR_ARGS;
    const int ng = d / ORC_FP8_GROUP;
    uint8_t *code = (uint8_t *)malloc((size_t)row_bytes);
    float *sc = (float *)malloc((size_t)ng * sizeof(float));
    if (!code || !sc) { free(code); free(sc); return ORC_ERR_NOMEM; }
    int rc = ORC_OK;
    for (int b = 0; b < B && rc == ORC_OK; ++b) {
        int pos = slot[b];
        if (pos < 0) continue;
        int logical = pos / ORC_PAGE_TOKENS, row = pos % ORC_PAGE_TOKENS;
        if (logical >= max_blocks) { rc = ORC_ERR_RANGE; break; }
        int phys = block_table[(size_t)b * max_blocks + logical];
        if (phys < 0 || phys >= num_blocks) { rc = ORC_ERR_RANGE; break; }
        for (int h = 0; h < H_kv; ++h) {
            size_t r = ((size_t)phys * H_kv + h) * ORC_PAGE_TOKENS + row;
            size_t src = ((size_t)b * H_kv + h) * (size_t)d;
            quant(k_new + src, 1, d, dtype, code, sc);
            memcpy(k8 + r * row_bytes, code, (size_t)row_bytes);
            memcpy(ks + r * ng, sc, (size_t)ng * sizeof(float));
            quant(v_new + src, 1, d, dtype, code, sc);
            memcpy(v8 + r * row_bytes, code, (size_t)row_bytes);
            memcpy(vs + r * ng, sc, (size_t)ng * sizeof(float));
        }
    }
    free(code);
    free(sc);
    return rc;
}

static int append_kv8(uint8_t *k8, uint8_t *v8, float *ks, float *vs, const int32_t *block_table,
                      const int32_t *slot, const uint16_t *k_new, const uint16_t *v_new, int B,
                      int H_kv, int d, int num_blocks, int max_blocks, int dtype, orc_quant_fn quant)
{
    return append_codes(k8, v8, ks, vs, block_table, slot, k_new, v_new, B, H_kv, d, d, num_blocks,
                        max_blocks, dtype, quant);
}

int orc_append_fp8(uint8_t *k8, uint8_t *v8, float *ks, float *vs, const int32_t *block_table,
                   const int32_t *slot, const uint16_t *k_new, const uint16_t *v_new, int B,
                   int H_kv, int d, int num_blocks, int max_blocks, int dtype)
{
    return append_kv8(k8, v8, ks, vs, block_table, slot, k_new, v_new, B, H_kv, d, num_blocks,
                      max_blocks, dtype, orc_quantize_fp8);
}

/* Attention over an 8-bit cache: exactly orc_attend's definition applied to
 * the dequantised values s * dec(code) (binary64).  q is fp16/bf16 words. */
typedef double (*orc_dec_fn)(uint8_t);

/* Value of channel i of cache row `row` (codes of `bits` bits: 8 -- one code
 * per byte, dec(byte); 4 -- two per byte, channel i in the low nibble of
 * byte i / 2 when i is even, in its high nibble when i is odd). */
static double code_value(const uint8_t *codes, long long row, int d, int i, int bits, orc_dec_fn dec)
{
    if (bits == 8) return dec(codes[row * d + i]);
    uint8_t byte = codes[row * (d / 2) + i / 2];
    return dec((uint8_t)((i % 2 == 0) ? (byte & 15) : (byte >> 4)));
}

static int attend_kv8(const uint16_t *q, const uint8_t *k8, const uint8_t *v8, const float *ks,
                      const float *vs, const int32_t *block_table, const int32_t *seq_lens,
                      double scale, int B, int H_q, int H_kv, int d, int num_blocks, int max_blocks,
                      int dtype, double *out, double *lse, int nthreads, orc_dec_fn dec, int bits)
{
    if (!q || !k8 || !v8 || !ks || !vs || !block_table || !seq_lens || !out) return ORC_ERR_ARGS;
    if (B < 0 || H_q <= 0 || H_kv <= 0 || H_q % H_kv || d <= 0 || d % ORC_FP8_GROUP) return ORC_ERR_ARGS;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] < 0 || seq_lens[b] > max_blocks * ORC_PAGE_TOKENS) return ORC_ERR_RANGE;
    const int G = H_q / H_kv, ng = d / ORC_FP8_GROUP;
    int status = ORC_OK;
    long long rows = (long long)B * H_q;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (long long r = 0; r < rows; ++r) {
        int b = (int)(r / H_q), hq = (int)(r % H_q), g = hq / G;
        int n = seq_lens[b];
        double *o = out + (size_t)r * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        if (n == 0) { if (lse) lse[r] = -INFINITY; continue; }
        double *s = (double *)malloc((size_t)n * sizeof(double));
        double *qv = (double *)malloc((size_t)d * sizeof(double));
        if (!s || !qv) { free(s); free(qv); status = ORC_ERR_NOMEM; continue; }
        for (int i = 0; i < d; ++i) qv[i] = decode_elem(q[(size_t)r * d + i], dtype);
        int bad = 0;
        for (int j = 0; j < n; ++j) {
            long long off = token_offset(block_table, b, j, g, H_kv, d, num_blocks, max_blocks);
            if (off < 0) { bad = 1; break; }
            const float *sk = ks + off / d * ng;
            double dot = 0.0;
            for (int i = 0; i < d; ++i)
                dot += qv[i] * ((double)sk[i / ORC_FP8_GROUP] * code_value(k8, off / d, d, i, bits, dec));
            s[j] = scale * dot;
        }
        if (bad) { free(s); free(qv); status = ORC_ERR_RANGE; continue; }
        double m = -INFINITY;
        for (int t = 0; t < n; ++t) if (s[t] > m) m = s[t];
        double den = 0.0;
        for (int j = 0; j < n; ++j) {
            double w = exp(s[j] - m);
            den += w;
            long long off = token_offset(block_table, b, j, g, H_kv, d, num_blocks, max_blocks);
            const float *sv = vs + off / d * ng;
            for (int i = 0; i < d; ++i)
                o[i] += w * ((double)sv[i / ORC_FP8_GROUP] * code_value(v8, off / d, d, i, bits, dec));
        }
        for (int i = 0; i < d; ++i) o[i] /= den;
        if (lse) lse[r] = m + log(den);
        free(s);
        free(qv);
    }
    return status;
}

int orc_attend_fp8(const uint16_t *q, const uint8_t *k8, const uint8_t *v8, const float *ks,
                   const float *vs, const int32_t *block_table, const int32_t *seq_lens,
                   double scale, int B, int H_q, int H_kv, int d, int num_blocks, int max_blocks,
                   int dtype, double *out, double *lse, int nthreads)
{
    return attend_kv8(q, k8, v8, ks, vs, block_table, seq_lens, scale, B, H_q, H_kv, d, num_blocks,
                      max_blocks, dtype, out, lse, nthreads, orc_e4m3_decode, 8);
}

/* Symmetric INT8 codes.  "KV Cache:推理慢的真正原因", section "工程优化手段 /
 * 量化" (int8 or int4 storage, scales per channel group because of outlier
 * keys); "推理速度慢怎么办？KV Cache与Flash Attention如何加速大模型推理", section
 * "三、实际落地" (the cache kept in INT8 or even INT4).  Reading taken here:
 * the same per-(token, KV head, 32-channel group) fp32 scale as the E4M3
 * cache with s = max|x| / 127 (fp32 division), code = x / s (fp32 division)
 * rounded to the nearest integer, ties to even, clamped to [-127, 127]; a
 * NaN quotient gives code 0; a group of zeros gets s = 0 and codes 0.
 * Dequantised value: s * code. */
double orc_int8_decode(uint8_t c)
{
    return (double)(int8_t)c;
}

uint8_t orc_int8_encode(float x)
{
    if (isnan(x)) return 0;
    double r = rint((double)x);               /* nearest, ties to even */
    if (r > 127.0) r = 127.0;
    if (r < -127.0) r = -127.0;
    return (uint8_t)(int8_t)r;
}

int orc_quantize_int8(const uint16_t *rows, int n, int d, int dtype, uint8_t *codes, float *scales)
{
    if (!rows || !codes || !scales || n < 0 || d <= 0 || d % ORC_FP8_GROUP) return ORC_ERR_ARGS;
    const int ng = d / ORC_FP8_GROUP;
    for (long long r = 0; r < n; ++r) {
        for (int g = 0; g < ng; ++g) {
            const uint16_t *x = rows + r * d + g * ORC_FP8_GROUP;
            float mx = 0.0f;
            for (int i = 0; i < ORC_FP8_GROUP; ++i) {
                float v = (float)fabs(decode_elem(x[i], dtype));
                if (v > mx) mx = v;
            }
            volatile float s = mx / 127.0f;
            scales[r * ng + g] = s;
            for (int i = 0; i < ORC_FP8_GROUP; ++i) {
                float v = (float)decode_elem(x[i], dtype);
                volatile float qt = s == 0.0f ? 0.0f : v / s;
                codes[r * d + g * ORC_FP8_GROUP + i] = s == 0.0f ? 0 : orc_int8_encode(qt);
            }
        }
    }
    return ORC_OK;
}

int orc_append_int8(uint8_t *k8, uint8_t *v8, float *ks, float *vs, const int32_t *block_table,
                    const int32_t *slot, const uint16_t *k_new, const uint16_t *v_new, int B,
                    int H_kv, int d, int num_blocks, int max_blocks, int dtype)
{
    return append_kv8(k8, v8, ks, vs, block_table, slot, k_new, v_new, B, H_kv, d, num_blocks,
                      max_blocks, dtype, orc_quantize_int8);
}

int orc_attend_int8(const uint16_t *q, const uint8_t *k8, const uint8_t *v8, const float *ks,
                    const float *vs, const int32_t *block_table, const int32_t *seq_lens,
                    double scale, int B, int H_q, int H_kv, int d, int num_blocks, int max_blocks,
                    int dtype, double *out, double *lse, int nthreads)
{
    return attend_kv8(q, k8, v8, ks, vs, block_table, seq_lens, scale, B, H_q, H_kv, d, num_blocks,
                      max_blocks, dtype, out, lse, nthreads, orc_int8_decode, 8);
}

/* Symmetric INT4 codes, two per byte.  "KV Cache:推理慢的真正原因", section
 * "工程优化手段 / 量化" (int4 storage, scales per channel group because of
 * outlier keys); "推理速度慢怎么办？KV Cache与Flash Attention如何加速大模型推理",
 * section "三、实际落地" (the cache kept in INT8 or even INT4).  Reading taken
 * here: the INT8 cache's definition with 7 in place of 127 -- one fp32 scale
 * per (token, KV head, 32-channel group), s = max|x| / 7 (fp32 division),
 * code = x / s (fp32 division) rounded to the nearest integer, ties to even,
 * clamped to [-7, 7]; a NaN quotient gives 0; a group of zeros gets s = 0 and
 * codes 0.  Packing: channel 2i is the low nibble of byte i and channel
 * 2i + 1 its high nibble, each a 4-bit two's complement integer.  Dequantised
 * value: s * code. */
double orc_int4_decode(uint8_t nib)
{
    int v = nib & 15;
    return (double)(v >= 8 ? v - 16 : v);
}

uint8_t orc_int4_encode(float x)
{
    if (isnan(x)) return 0;
    double r = rint((double)x);               /* nearest, ties to even */
    if (r > 7.0) r = 7.0;
    if (r < -7.0) r = -7.0;
    return (uint8_t)((int)r & 15);
}

/* Quantise n rows of d storage words into packed codes [n][d / 2] and
 * scales [n][d / 32]. */
int orc_quantize_int4(const uint16_t *rows, int n, int d, int dtype, uint8_t *codes, float *scales)
{
    if (!rows || !codes || !scales || n < 0 || d <= 0 || d % ORC_FP8_GROUP) return ORC_ERR_ARGS;
    const int ng = d / ORC_FP8_GROUP;
    for (long long r = 0; r < n; ++r) {
        for (int g = 0; g < ng; ++g) {
            const uint16_t *x = rows + r * d + g * ORC_FP8_GROUP;
            float mx = 0.0f;
            for (int i = 0; i < ORC_FP8_GROUP; ++i) {
                float v = (float)fabs(decode_elem(x[i], dtype));
                if (v > mx) mx = v;
            }
            volatile float s = mx / 7.0f;
            scales[r * ng + g] = s;
            for (int i = 0; i < ORC_FP8_GROUP; ++i) {
                float v = (float)decode_elem(x[i], dtype);
                volatile float qt = s == 0.0f ? 0.0f : v / s;
                uint8_t nib = s == 0.0f ? 0 : orc_int4_encode(qt);
                int ch = g * ORC_FP8_GROUP + i;          /* channel within the row */
                uint8_t *byte = codes + r * (d / 2) + ch / 2;
                if (ch % 2 == 0) *byte = (uint8_t)((*byte & 0xF0) | nib);
                else *byte = (uint8_t)((*byte & 0x0F) | (nib << 4));
            }
        }
    }
    return ORC_OK;
}

int orc_append_int4(uint8_t *k4, uint8_t *v4, float *ks, float *vs, const int32_t *block_table,
                    const int32_t *slot, const uint16_t *k_new, const uint16_t *v_new, int B,
                    int H_kv, int d, int num_blocks, int max_blocks, int dtype)
{
    if (d % 2) return ORC_ERR_ARGS;
    return append_codes(k4, v4, ks, vs, block_table, slot, k_new, v_new, B, H_kv, d, d / 2,
                        num_blocks, max_blocks, dtype, orc_quantize_int4);
}

int orc_attend_int4(const uint16_t *q, const uint8_t *k4, const uint8_t *v4, const float *ks,
                    const float *vs, const int32_t *block_table, const int32_t *seq_lens,
                    double scale, int B, int H_q, int H_kv, int d, int num_blocks, int max_blocks,
                    int dtype, double *out, double *lse, int nthreads)
{
    return attend_kv8(q, k4, v4, ks, vs, block_table, seq_lens, scale, B, H_q, H_kv, d, num_blocks,
                      max_blocks, dtype, out, lse, nthreads, orc_int4_decode, 4);
}

int orc_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
