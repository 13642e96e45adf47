/*
 * attention_ref.c -- plain fp64 CPU oracle for exact scaled-dot-product
 * attention forward (the standard, non-tiled definition).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline leg do.  It shares no code, header, table or constant with the
 * CUDA library.
 *
 * What is computed, and where the pages define it:
 *   S = scale * Q K^T, P = softmax(S), O = P V
 *     -- "PyTorch Transformer Flash Attention机制" section 1 (formulas for
 *        Attention_weights and Output); "FlashAttention算法原理与性能优化实战"
 *        section 1.1 (S, P, O).
 *   softmax is the three-pass safe softmax: m = max, d = sum e^{x-m},
 *   a = e^{x-m}/d
 *     -- "Flash Attention是怎么做到又快又省显存的？" section 时间复杂度
 *        (Safe Softmax, its three iterations).
 *   lse = m + ln(d) of the scaled scores: the per-row statistic the forward
 *   keeps for the backward pass
 *     -- Triton FA2 walkthrough (logsumexp L for backward);
 *        "FlashAttention算法原理与性能优化实战" section 2.2 (softmax_max and
 *        softmax_sum outputs of shape [B,H,S]).
 *   visibility (mask): key j is visible from query i iff
 *        j < L_k, (not causal or j <= i), (wl < 0 or j >= i - wl),
 *        (wr < 0 or j <= i + wr); indices are raw positions (top-left
 *        aligned).  pre_tokens / next_tokens of section 2.2 of
 *        "FlashAttention算法原理与性能优化实战" are wl / wr; a negative value
 *        means unbounded (their default is INT_MAX).
 *   GQA: query head h reads key/value head h / (H / H_kv)
 *     -- "FlashAttention算法原理与性能优化实战" section 1.3 (MQA/GQA).
 *   A row with no visible key has O = 0 and lse = -inf (the pages are
 *   silent; this is the stated reading).
 *
 * Inputs are raw bit patterns (fp16, bf16, or fp8 e4m3 codes widened to 16
 * bits); this file decodes them itself.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------------
 * Number formats (IEEE 754 binary16, and bfloat16 = the top 16 bits of
 * binary32).  Decoding is exact in double.
 * ------------------------------------------------------------------- */
double oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);               /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);   /* 1.m * 2^(e-15) */
    return sign ? -v : v;
}

double oracle_bf16_to_f64(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int e = (b >> 7) & 0xff;
    int m = b & 0x7f;
    double v;
    if (e == 0)
        v = ldexp((double)m, -133);              /* subnormal: m * 2^-133 */
    else if (e == 255)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(128 + m), e - 134);   /* 1.m * 2^(e-127) */
    return sign ? -v : v;
}

/* Round a double to the nearest representable value with ties to even,
 * for a format with `mbits` fraction bits and exponent bias `bias`
 * (normal exponents 1 .. 2*bias).  Returns the bit pattern. */
static uint16_t round_rne(double x, int mbits, int bias)
{
    const int ebits = (bias == 15) ? 5 : 8;
    const uint16_t inf_bits = (uint16_t)(((1u << ebits) - 1) << mbits);
    uint16_t sign = signbit(x) ? (uint16_t)(1u << 15) : 0;
    if (isnan(x))
        return (uint16_t)(inf_bits | (1u << (mbits - 1)));
    double a = fabs(x);
    if (isinf(a))
        return sign | inf_bits;
    if (a == 0.0)
        return sign;
    int E;
    frexp(a, &E);                 /* a = f * 2^E, f in [0.5, 1) */
    int ue = E - 1;               /* a in [2^ue, 2^(ue+1)) */
    const int emin = 1 - bias;    /* smallest normal exponent */
    int q_exp = (ue < emin ? emin : ue) - mbits;   /* quantum = 2^q_exp */
    double r = nearbyint(ldexp(a, -q_exp));        /* default mode: ties to even */
    if (ue < emin) {
        /* subnormal range; r == 2^mbits is exactly the smallest normal */
        return sign | (uint16_t)r;
    }
    if (r >= ldexp(1.0, mbits + 1)) {  /* carried into the next binade */
        r = ldexp(r, -1);
        ue += 1;
    }
    int eb = ue + bias;
    if (eb >= (1 << ebits) - 1)
        return sign | inf_bits;
    return sign | (uint16_t)(eb << mbits) | (uint16_t)((uint32_t)r - (1u << mbits));
}

/* FP8 E4M3 (the "fn" variant: no infinities, S.1111.111 is NaN, largest
 * finite 448): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
 * exponent field 0 holds the subnormals m * 2^-9.  The pages name fp8 as an
 * input type of FlashAttention-2 ("PyTorch Transformer Flash Attention机制",
 * section 5); the format itself is the standard OCP FP8 E4M3 encoding. */
double oracle_e4m3_to_f64(uint8_t x)
{
    int sign = (x >> 7) & 1;
    int e = (x >> 3) & 0xf;
    int m = x & 0x7;
    double v;
    if (e == 0xf && m == 0x7)
        v = NAN;
    else if (e == 0)
        v = ldexp((double)m, -9);                /* subnormal: m * 2^-9 */
    else
        v = ldexp((double)(8 + m), e - 10);      /* 1.m * 2^(e-7) */
    return sign ? -v : v;
}

uint16_t oracle_f64_to_f16(double x) { return round_rne(x, 10, 15); }
uint16_t oracle_f64_to_bf16(double x) { return round_rne(x, 7, 127); }

/* ---------------------------------------------------------------------
 * Softmax over one vector.
 * ------------------------------------------------------------------- */

/* Three-pass safe softmax ("Flash Attention是怎么做到又快又省显存的？",
 * Safe Softmax): pass 1 the maximum m, pass 2 d = sum e^{x_i - m},
 * pass 3 a_i = e^{x_i - m} / d.  Returns d and m through the pointers. */
void oracle_safe_softmax(const double *x, int64_t n, double *out,
                         double *d_out, double *m_out)
{
    double m = -INFINITY;
    for (int64_t i = 0; i < n; i++)
        if (x[i] > m) m = x[i];
    double d = 0.0;
    if (m != -INFINITY)
        for (int64_t i = 0; i < n; i++)
            d += exp(x[i] - m);
    for (int64_t i = 0; i < n; i++)
        out[i] = (m == -INFINITY) ? 0.0 : exp(x[i] - m) / d;
    if (d_out) *d_out = d;
    if (m_out) *m_out = m;
}

/* Online normaliser (same page, the Online normalizer derivation): one pass
 * keeps the running maximum m_i and d'_i = d'_{i-1} e^{m_{i-1} - m_i} +
 * e^{x_i - m_i}; a second pass forms a_i = e^{x_i - m_N} / d'_N.  The final
 * pass uses the global m_N for every element, as the derivation states. */
void oracle_online_softmax(const double *x, int64_t n, double *out,
                           double *d_out, double *m_out)
{
    double m = -INFINITY, d = 0.0;
    for (int64_t i = 0; i < n; i++) {
        double m_new = x[i] > m ? x[i] : m;
        if (m_new == -INFINITY)
            continue;                       /* nothing visible yet */
        d = d * exp(m - m_new) + exp(x[i] - m_new);
        m = m_new;
    }
    for (int64_t i = 0; i < n; i++)
        out[i] = (m == -INFINITY) ? 0.0 : exp(x[i] - m) / d;
    if (d_out) *d_out = d;
    if (m_out) *m_out = m;
}

/* ---------------------------------------------------------------------
 * Attention forward.
 * ------------------------------------------------------------------- */
static int visible(int64_t i, int64_t j, int64_t L_k, int causal,
                   int64_t wl, int64_t wr)
{
    if (j < 0 || j >= L_k) return 0;
    if (causal && j > i) return 0;
    if (wl >= 0 && j < i - wl) return 0;
    if (wr >= 0 && j > i + wr) return 0;
    return 1;
}

/* dtype 0 fp16, 1 bf16, 2 fp8 e4m3 (the code in the low byte). */
static void build_decode_table(int dtype, double *tab)
{
    for (uint32_t b = 0; b < 65536u; b++)
        tab[b] = dtype == 0 ? oracle_f16_to_f64((uint16_t)b)
               : dtype == 1 ? oracle_bf16_to_f64((uint16_t)b)
                            : oracle_e4m3_to_f64((uint8_t)(b & 0xff));
}

/* ---------------------------------------------------------------------
 * Forward with an optional attention mask and the two softmax statistics.
 *
 * The operator statement of "FlashAttention算法原理与性能优化实战" section 2.2
 * takes an optional attn_mask (fp16, fp32 or bool) and returns, beside the
 * output, softmax_max and softmax_sum of shape [B, H, S] for the backward.
 * The Triton FA2 walkthrough notes that mask (and dropout) act on S before
 * the softmax, as step MASK of FlashAttention's Algorithm 2.  The pages do
 * not spell out the mask's meaning; the reading taken here:
 *   - a float mask (fp16 / fp32) is added to the scaled scores:
 *       s_ij = scale * q_i . k_j + mask_ij   (-inf hides the key);
 *   - a bool mask hides the keys where it is true (nonzero byte), like the
 *     MASK step that sets those scores to -inf;
 *   - the causal / window visibility still applies on top;
 *   - element (b, h, i, j) of the mask is element
 *       b*stride_b + h*stride_h + i*stride_q + j  of the array,
 *     a stride of 0 broadcasts over that index;
 *   - softmax_max_i = max_j s_ij over the visible keys and
 *     softmax_sum_i = sum_j e^{s_ij - softmax_max_i}, so that
 *     lse_i = softmax_max_i + ln(softmax_sum_i); a row with no visible key
 *     has softmax_max = -inf and softmax_sum = 0.
 * mask_type: 0 none, 1 bool (uint8), 2 fp16, 3 fp32.
 * ------------------------------------------------------------------- */
static double mask_value(const void *mask, int mask_type, int64_t idx, int *hidden)
{
    *hidden = 0;
    if (mask_type == 1) {
        *hidden = ((const uint8_t *)mask)[idx] != 0;
        return 0.0;
    }
    if (mask_type == 2) return oracle_f16_to_f64(((const uint16_t *)mask)[idx]);
    if (mask_type == 3) return (double)((const float *)mask)[idx];
    return 0.0;
}


/*
 * Exact attention for a list of query rows.
 *   q    : [B, H,    L_q, D] bit patterns (dtype 0 = fp16, 1 = bf16)
 *   k, v : [B, H_kv, L_k, D]
 *   rows : flattened row ids r = (b*H + h)*L_q + i, or NULL for all rows
 *   out  : [n_rows, D] fp64;  lse : [n_rows] fp64 (may be NULL)
 *   wabs : [n_rows, D] fp64 (may be NULL): sum_j p_j |v_j[d]|, the softmax-
 *          weighted mean magnitude of V.  Not part of the attention result:
 *          it is the scale of the error that rounding the weights p_j to a
 *          t-bit format causes in O (at most 2^-t * wabs per element, first
 *          order), which the parity tests use in their tolerance.
 *   wrss : [n_rows, D] fp64 (may be NULL): sqrt(sum_j p_j^2 v_j[d]^2), the
 *          root of the sum of squares of the same terms.  Also not part of
 *          the result: when the rounding errors of the weights are
 *          independent, their effect on O[d] has a standard deviation of
 *          at most 2^-t / sqrt(3) * wrss, which the parity tests use for a
 *          tolerance that does not grow with the number of keys.
 *   mask, mask_type, stride_b/h/q : the optional mask (type 0 = none),
 *          read as stated above mask_value();
 *   smax, ssum : [n_rows] fp64 (may be NULL): softmax_max, softmax_sum.
 * Shared by oracle_attention_rows (no mask, no statistics) and
 * oracle_attention_rows_ex.
 * Returns the number of threads used, or a negative value on bad input.
 */
static int rows_core(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     int dtype, int64_t B, int64_t H, int64_t H_kv, int64_t L_q,
                     int64_t L_k, int64_t D, double scale, int causal,
                     int64_t window_left, int64_t window_right,
                     const void *mask, int mask_type, int64_t stride_b,
                     int64_t stride_h, int64_t stride_q, const int64_t *rows,
                     int64_t n_rows, double *out, double *lse, double *wabs,
                     double *wrss, double *smax, double *ssum, int n_threads)
{
    if (B < 1 || H < 1 || H_kv < 1 || L_q < 0 || L_k < 0 || D < 1)
        return -1;
    if (H % H_kv != 0 || dtype < 0 || dtype > 2)
        return -1;
    if (mask_type < 0 || mask_type > 3 || (mask_type != 0 && mask == NULL))
        return -1;
    if (rows == NULL)
        n_rows = B * H * L_q;
    const int64_t group = H / H_kv;
    double *tab = (double *)malloc(sizeof(double) * 65536);
    if (!tab) return -2;
    build_decode_table(dtype, tab);
    int used = 1;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#endif

#pragma omp parallel
    {
#ifdef _OPENMP
#pragma omp single
        used = omp_get_num_threads();
#endif
        double *qrow = (double *)malloc(sizeof(double) * (size_t)(D > 0 ? D : 1));
        double *s = (double *)malloc(sizeof(double) * (size_t)(L_k > 0 ? L_k : 1));
        double *p = (double *)malloc(sizeof(double) * (size_t)(L_k > 0 ? L_k : 1));
#pragma omp for schedule(dynamic, 4)
        for (int64_t t = 0; t < n_rows; t++) {
            int64_t r = rows ? rows[t] : t;
            int64_t bh = r / L_q, i = r % L_q;
            int64_t b = bh / H, h = bh % H;
            int64_t g = h / group;                       /* GQA head map */
            const uint16_t *qp = q + ((b * H + h) * L_q + i) * D;
            const uint16_t *kp = k + (b * H_kv + g) * L_k * D;
            const uint16_t *vp = v + (b * H_kv + g) * L_k * D;
            for (int64_t d = 0; d < D; d++)
                qrow[d] = tab[qp[d]];
            /* the full row of S, with masked entries at -inf */
            for (int64_t j = 0; j < L_k; j++) {
                int hidden = 0;
                double bias = 0.0;
                if (mask_type != 0)
                    bias = mask_value(mask, mask_type,
                                      b * stride_b + h * stride_h + i * stride_q + j, &hidden);
                if (hidden || !visible(i, j, L_k, causal, window_left, window_right)) {
                    s[j] = -INFINITY;
                    continue;
                }
                double acc = 0.0;
                for (int64_t d = 0; d < D; d++)
                    acc += qrow[d] * tab[kp[j * D + d]];
                s[j] = scale * acc;
                s[j] += bias;
            }
            double m, den;
            oracle_safe_softmax(s, L_k, p, &den, &m);
            double *o = out + t * D;
            for (int64_t d = 0; d < D; d++)
                o[d] = 0.0;
            for (int64_t j = 0; j < L_k; j++) {
                if (p[j] == 0.0) continue;
                for (int64_t d = 0; d < D; d++)
                    o[d] += p[j] * tab[vp[j * D + d]];
            }
            if (lse)
                lse[t] = (m == -INFINITY) ? -INFINITY : m + log(den);
            if (smax) smax[t] = m;
            if (ssum) ssum[t] = (m == -INFINITY) ? 0.0 : den;
            if (wabs) {
                double *w = wabs + t * D;
                for (int64_t d = 0; d < D; d++)
                    w[d] = 0.0;
                for (int64_t j = 0; j < L_k; j++) {
                    if (p[j] == 0.0) continue;
                    for (int64_t d = 0; d < D; d++)
                        w[d] += p[j] * fabs(tab[vp[j * D + d]]);
                }
            }
            if (wrss) {
                double *w = wrss + t * D;
                for (int64_t d = 0; d < D; d++)
                    w[d] = 0.0;
                for (int64_t j = 0; j < L_k; j++) {
                    if (p[j] == 0.0) continue;
                    for (int64_t d = 0; d < D; d++) {
                        const double term = p[j] * tab[vp[j * D + d]];
                        w[d] += term * term;
                    }
                }
                for (int64_t d = 0; d < D; d++)
                    w[d] = sqrt(w[d]);
            }
        }
        free(qrow);
        free(s);
        free(p);
    }
    free(tab);
    return used;
}

int oracle_attention_rows(const uint16_t *q, const uint16_t *k,
                          const uint16_t *v, int dtype, int64_t B, int64_t H,
                          int64_t H_kv, int64_t L_q, int64_t L_k, int64_t D,
                          double scale, int causal, int64_t window_left,
                          int64_t window_right, const int64_t *rows,
                          int64_t n_rows, double *out, double *lse,
                          double *wabs, int n_threads)
{
    return rows_core(q, k, v, dtype, B, H, H_kv, L_q, L_k, D, scale, causal,
                     window_left, window_right, NULL, 0, 0, 0, 0, rows, n_rows,
                     out, lse, wabs, NULL, NULL, NULL, n_threads);
}

/* The same with a mask and the two softmax statistics (wabs, wrss, smax,
 * ssum nullable), as stated above the mask helpers. */
int oracle_attention_rows_ex(const uint16_t *q, const uint16_t *k,
                             const uint16_t *v, int dtype, int64_t B, int64_t H,
                             int64_t H_kv, int64_t L_q, int64_t L_k, int64_t D,
                             double scale, int causal, int64_t window_left,
                             int64_t window_right, const void *mask,
                             int mask_type, int64_t stride_b, int64_t stride_h,
                             int64_t stride_q, const int64_t *rows,
                             int64_t n_rows, double *out, double *lse,
                             double *wabs, double *wrss, double *smax,
                             double *ssum, int n_threads)
{
    return rows_core(q, k, v, dtype, B, H, H_kv, L_q, L_k, D, scale, causal,
                     window_left, window_right, mask, mask_type, stride_b,
                     stride_h, stride_q, rows, n_rows, out, lse, wabs, wrss,
                     smax, ssum, n_threads);
}

/*
 * The same rows computed by the FA2 recurrence instead of the plain
 * definition: for one query row, walk the keys in blocks of `block`,
 * keep the running maximum m, the running normaliser l and an
 * unnormalised accumulator acc; when the maximum grows by a block,
 * scale l and acc by e^{m_old - m_new}; divide by l once at the end.
 *   -- Triton FA2 walkthrough (outer loop over Q, inner over K/V, the
 *      division by the softmax denominator moved to the end);
 *      "FlashAttention算法原理与性能优化实战" section 1.2.2, read as the plain
 *      FA1 update (the block-local correction factor is applied once).
 * Test infrastructure: it shows the tiled method reaches the definition.
 */
int oracle_attention_rows_online(const uint16_t *q, const uint16_t *k,
                                 const uint16_t *v, int dtype, int64_t B,
                                 int64_t H, int64_t H_kv, int64_t L_q,
                                 int64_t L_k, int64_t D, double scale,
                                 int causal, int64_t window_left,
                                 int64_t window_right, const int64_t *rows,
                                 int64_t n_rows, int64_t block, double *out,
                                 double *lse)
{
    if (B < 1 || H < 1 || H_kv < 1 || L_q < 0 || L_k < 0 || D < 1 || block < 1)
        return -1;
    if (H % H_kv != 0 || (dtype != 0 && dtype != 1))
        return -1;
    if (rows == NULL)
        n_rows = B * H * L_q;
    const int64_t group = H / H_kv;
    double *tab = (double *)malloc(sizeof(double) * 65536);
    double *acc = (double *)malloc(sizeof(double) * (size_t)D);
    double *sb = (double *)malloc(sizeof(double) * (size_t)block);
    if (!tab || !acc || !sb) { free(tab); free(acc); free(sb); return -2; }
    build_decode_table(dtype, tab);
    for (int64_t t = 0; t < n_rows; t++) {
        int64_t r = rows ? rows[t] : t;
        int64_t bh = r / L_q, i = r % L_q;
        int64_t b = bh / H, h = bh % H;
        int64_t g = h / group;
        const uint16_t *qp = q + ((b * H + h) * L_q + i) * D;
        const uint16_t *kp = k + (b * H_kv + g) * L_k * D;
        const uint16_t *vp = v + (b * H_kv + g) * L_k * D;
        double m = -INFINITY, l = 0.0;
        for (int64_t d = 0; d < D; d++) acc[d] = 0.0;
        for (int64_t j0 = 0; j0 < L_k; j0 += block) {
            int64_t nb = (L_k - j0 < block) ? (L_k - j0) : block;
            double m_blk = -INFINITY;
            for (int64_t c = 0; c < nb; c++) {
                int64_t j = j0 + c;
                if (!visible(i, j, L_k, causal, window_left, window_right)) {
                    sb[c] = -INFINITY;
                    continue;
                }
                double dot = 0.0;
                for (int64_t d = 0; d < D; d++)
                    dot += tab[qp[d]] * tab[kp[j * D + d]];
                sb[c] = scale * dot;
                if (sb[c] > m_blk) m_blk = sb[c];
            }
            if (m_blk == -INFINITY)
                continue;                     /* nothing visible in block */
            double m_new = m > m_blk ? m : m_blk;
            double alpha = exp(m - m_new);    /* 0 when m was -inf */
            l *= alpha;
            for (int64_t d = 0; d < D; d++) acc[d] *= alpha;
            for (int64_t c = 0; c < nb; c++) {
                if (sb[c] == -INFINITY) continue;
                double pc = exp(sb[c] - m_new);
                l += pc;
                for (int64_t d = 0; d < D; d++)
                    acc[d] += pc * tab[vp[(j0 + c) * D + d]];
            }
            m = m_new;
        }
        for (int64_t d = 0; d < D; d++)
            out[t * D + d] = (l > 0.0) ? acc[d] / l : 0.0;
        if (lse)
            lse[t] = (l > 0.0) ? m + log(l) : -INFINITY;
    }
    free(tab);
    free(acc);
    free(sb);
    return 1;
}

/* ---------------------------------------------------------------------
 * Attention on fp64 inputs, forward and backward.
 *
 * Backward: the pages keep only the softmax statistics from the forward and
 * recompute the attention matrix from Q, K, V when the gradients are taken
 * ("FlashAttention算法原理与性能优化实战" section 1.2.3, recomputation;
 * "Flash Attention是怎么做到又快又省显存的？" 总结, recomputation as a
 * tiling-based gradient checkpoint; the Triton FA2 walkthrough keeps the
 * logsumexp for the backward pass).  They print no gradient formulas, so
 * this is the plain definition: the gradient of sum(dO .* O) for
 * O = softmax(scale Q K^T + mask) V, by the chain rule,
 *     dV = P^T dO,  dP = dO V^T,  dS_ij = P_ij (dP_ij - delta_i),
 *     delta_i = sum_j P_ij dP_ij,  dQ = scale dS K,  dK = scale dS^T Q,
 * with P recomputed by the plain safe softmax of each row.  With GQA, the
 * gradient of a shared K/V head sums over the query heads that read it.
 * ------------------------------------------------------------------- */

/*
 * Forward on fp64 inputs (no rounding anywhere); layout as
 * oracle_attention_rows, all rows.  out [B,H,L_q,D], lse [B,H,L_q]
 * (nullable).  Returns 0, or -1 on bad sizes.
 */
int oracle_attention_f64(const double *q, const double *k, const double *v,
                         int64_t B, int64_t H, int64_t H_kv, int64_t L_q,
                         int64_t L_k, int64_t D, double scale, int causal,
                         int64_t wl, int64_t wr, double *out, double *lse)
{
    if (B < 1 || H < 1 || H_kv < 1 || L_q < 0 || L_k < 0 || D < 1 ||
        H % H_kv != 0)
        return -1;
    const int64_t group = H / H_kv;
    double *s = (double *)malloc(sizeof(double) * (size_t)(L_k > 0 ? L_k : 1));
    double *p = (double *)malloc(sizeof(double) * (size_t)(L_k > 0 ? L_k : 1));
    if (!s || !p) { free(s); free(p); return -2; }
    for (int64_t b = 0; b < B; b++)
        for (int64_t h = 0; h < H; h++) {
            const double *kp = k + (b * H_kv + h / group) * L_k * D;
            const double *vp = v + (b * H_kv + h / group) * L_k * D;
            for (int64_t i = 0; i < L_q; i++) {
                const int64_t row = (b * H + h) * L_q + i;
                const double *qi = q + row * D;
                for (int64_t j = 0; j < L_k; j++) {
                    if (!visible(i, j, L_k, causal, wl, wr)) { s[j] = -INFINITY; continue; }
                    double acc = 0.0;
                    for (int64_t d = 0; d < D; d++) acc += qi[d] * kp[j * D + d];
                    s[j] = scale * acc;
                }
                double m, den;
                oracle_safe_softmax(s, L_k, p, &den, &m);
                double *o = out + row * D;
                for (int64_t d = 0; d < D; d++) o[d] = 0.0;
                for (int64_t j = 0; j < L_k; j++)
                    for (int64_t d = 0; d < D; d++) o[d] += p[j] * vp[j * D + d];
                if (lse) lse[row] = (m == -INFINITY) ? -INFINITY : m + log(den);
            }
        }
    free(s);
    free(p);
    return 0;
}

/*
 * Backward on fp64 inputs: dq [B,H,L_q,D], dk and dv [B,H_kv,L_k,D] (all
 * written), for the upstream gradient dout [B,H,L_q,D].
 *
 * Optional error scales for the parity tests (each nullable; not part of
 * the gradient): given delta_err[row] >= 0, a bound on the error of the
 * delta_i the tested implementation uses,
 *   dv_abs = |P|^T |dO|,
 *   dk_abs = scale (|dS| + P e)^T |Q|,   dq_abs = scale (|dS| + P e) |K|,
 * with e_i = delta_err[i] (0 when delta_err is NULL): rounding P or dS to a
 * t-bit format moves a gradient by at most 2^-t times these (first order),
 * and an error e_i in delta_i moves dS_ij by P_ij e_i.
 * Threads run over (b, K/V head) so that each owns its dk / dv rows.
 * Returns the number of threads used, or a negative value on bad input.
 */
static int bwd_core(const double *q, const double *k, const double *v,
                    const double *dout, int64_t B, int64_t H, int64_t H_kv,
                    int64_t L_q, int64_t L_k, int64_t D, double scale,
                    int causal, int64_t wl, int64_t wr, const void *mask,
                    int mask_type, int64_t stride_b, int64_t stride_h,
                    int64_t stride_q, double *dq, double *dk, double *dv,
                    const double *delta_err, double *dq_abs, double *dk_abs,
                    double *dv_abs, int n_threads)
{
    if (B < 1 || H < 1 || H_kv < 1 || L_q < 0 || L_k < 0 || D < 1 ||
        H % H_kv != 0)
        return -1;
    if (mask_type < 0 || mask_type > 3 || (mask_type != 0 && mask == NULL))
        return -1;
    const int64_t group = H / H_kv;
    int used = 1;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#endif
#pragma omp parallel
    {
#ifdef _OPENMP
#pragma omp single
        used = omp_get_num_threads();
#endif
        const size_t nk = (size_t)(L_k > 0 ? L_k : 1);
        double *s = (double *)malloc(sizeof(double) * nk);
        double *p = (double *)malloc(sizeof(double) * nk);
        double *dp = (double *)malloc(sizeof(double) * nk);
        double *ds = (double *)malloc(sizeof(double) * nk);
#pragma omp for schedule(dynamic, 1)
        for (int64_t bg = 0; bg < B * H_kv; bg++) {
            const int64_t b = bg / H_kv, g = bg % H_kv;
            const double *kp = k + bg * L_k * D;
            const double *vp = v + bg * L_k * D;
            double *dkp = dk + bg * L_k * D;
            double *dvp = dv + bg * L_k * D;
            double *dka = dk_abs ? dk_abs + bg * L_k * D : NULL;
            double *dva = dv_abs ? dv_abs + bg * L_k * D : NULL;
            for (int64_t x = 0; x < L_k * D; x++) {
                dkp[x] = 0.0;
                dvp[x] = 0.0;
                if (dka) dka[x] = 0.0;
                if (dva) dva[x] = 0.0;
            }
            for (int64_t h = g * group; h < (g + 1) * group; h++)
                for (int64_t i = 0; i < L_q; i++) {
                    const int64_t row = (b * H + h) * L_q + i;
                    const double *qi = q + row * D;
                    const double *doi = dout + row * D;
                    /* recompute P_i (plain safe softmax of the scaled row) */
                    for (int64_t j = 0; j < L_k; j++) {
                        int hidden = 0;
                        double bias = 0.0;
                        if (mask_type != 0)
                            bias = mask_value(mask, mask_type, b * stride_b + h * stride_h +
                                                                   i * stride_q + j, &hidden);
                        if (hidden || !visible(i, j, L_k, causal, wl, wr)) { s[j] = -INFINITY; continue; }
                        double acc = 0.0;
                        for (int64_t d = 0; d < D; d++) acc += qi[d] * kp[j * D + d];
                        s[j] = scale * acc + bias;
                    }
                    double m, den;
                    oracle_safe_softmax(s, L_k, p, &den, &m);
                    /* dP_ij = dO_i . V_j, delta_i = sum_j P_ij dP_ij */
                    double delta = 0.0;
                    for (int64_t j = 0; j < L_k; j++) {
                        double acc = 0.0;
                        if (p[j] != 0.0)
                            for (int64_t d = 0; d < D; d++) acc += doi[d] * vp[j * D + d];
                        dp[j] = acc;
                        delta += p[j] * acc;
                    }
                    for (int64_t j = 0; j < L_k; j++)
                        ds[j] = p[j] * (dp[j] - delta);
                    const double e = delta_err ? delta_err[row] : 0.0;
                    double *dqi = dq + row * D;
                    double *dqa = dq_abs ? dq_abs + row * D : NULL;
                    for (int64_t d = 0; d < D; d++) {
                        dqi[d] = 0.0;
                        if (dqa) dqa[d] = 0.0;
                    }
                    for (int64_t j = 0; j < L_k; j++) {
                        if (p[j] == 0.0) continue;
                        const double wabs_j = fabs(ds[j]) + p[j] * e;
                        for (int64_t d = 0; d < D; d++) {
                            dqi[d] += scale * ds[j] * kp[j * D + d];
                            dkp[j * D + d] += scale * ds[j] * qi[d];
                            dvp[j * D + d] += p[j] * doi[d];
                            if (dqa) dqa[d] += scale * wabs_j * fabs(kp[j * D + d]);
                            if (dka) dka[j * D + d] += scale * wabs_j * fabs(qi[d]);
                            if (dva) dva[j * D + d] += p[j] * fabs(doi[d]);
                        }
                    }
                }
        }
        free(s);
        free(p);
        free(dp);
        free(ds);
    }
    return used;
}

/* The backward without a mask, and with one (read as the forward reads it,
 * see mask_value): P is the softmax of scale q.k + mask with hidden keys
 * removed; the mask is a constant, so the gradients keep their form. */
int oracle_attention_bwd_f64(const double *q, const double *k, const double *v,
                             const double *dout, int64_t B, int64_t H,
                             int64_t H_kv, int64_t L_q, int64_t L_k, int64_t D,
                             double scale, int causal, int64_t wl, int64_t wr,
                             double *dq, double *dk, double *dv,
                             const double *delta_err, double *dq_abs,
                             double *dk_abs, double *dv_abs, int n_threads)
{
    return bwd_core(q, k, v, dout, B, H, H_kv, L_q, L_k, D, scale, causal, wl, wr,
                    NULL, 0, 0, 0, 0, dq, dk, dv, delta_err, dq_abs, dk_abs, dv_abs,
                    n_threads);
}

int oracle_attention_bwd_f64_ex(const double *q, const double *k, const double *v,
                                const double *dout, int64_t B, int64_t H,
                                int64_t H_kv, int64_t L_q, int64_t L_k, int64_t D,
                                double scale, int causal, int64_t wl, int64_t wr,
                                const void *mask, int mask_type, int64_t stride_b,
                                int64_t stride_h, int64_t stride_q, double *dq,
                                double *dk, double *dv, const double *delta_err,
                                double *dq_abs, double *dk_abs, double *dv_abs,
                                int n_threads)
{
    return bwd_core(q, k, v, dout, B, H, H_kv, L_q, L_k, D, scale, causal, wl, wr,
                    mask, mask_type, stride_b, stride_h, stride_q, dq, dk, dv,
                    delta_err, dq_abs, dk_abs, dv_abs, n_threads);
}
