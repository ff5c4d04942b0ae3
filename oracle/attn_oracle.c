/*
 * Plain CPU oracle for causal scaled-dot-product attention, in fp64.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the bench's CPU-baseline leg load this
 * file's library; the CUDA product path never calls it, links it or shares code with it.
 *
 * What it computes is the plain definition, with no blocking, fusion or online rescaling:
 *
 *   for every batch b, query head h and query row i (kv head = h / (Hq / Hkv)):
 *     visible keys  V_i = { j : 0 <= j < Skv and (!causal or j <= i + (Skv - Sq)) }
 *     s_j   = scale * sum_d q[i,d] * k[j,d]                                  (step 1)
 *     m     = max_{j in V_i} s_j                                              (pass 1)
 *     l     = sum_{j in V_i} exp(s_j - m)                                     (pass 2)
 *     o[i,:]= sum_{j in V_i} exp(s_j - m) * v[j,:] / l ;  lse_i = m + ln(l)   (pass 3)
 *
 * Sources (page title, section):
 *  - "05 · Tích vô hướng, Softmax và toán của Attention", §1 (dot product as the relevance score;
 *    worked example (2,-1,0.5).(3,4,2) = 3), "Vì sao chia cho √128" (divide scores by sqrt(d)),
 *    §2 (softmax = exp then divide by the sum; subtract the row max first), §3 (one query against
 *    all keys -> scale -> softmax -> weighted sum of values).
 *  - "AI Infra 入门：RMSNorm、Softmax、Causal Mask、Sampling 的数学与底层优化", §2 (safe softmax:
 *    subtract the max M), §3 (causal mask adds -inf for j > i; softmax as three passes: max, then
 *    denominator, then result; LSE = m + ln(l) so that softmax(z_i) = exp(z_i - LSE)).
 *  - "Bộ 06 · Bên trong model", Q1 (softmax(x - c) = softmax(x)), Q2 (the mask adds -inf, whose
 *    exponential is exactly 0, so a masked key gets weight exactly 0).
 *  - "第11节：Attention 实现（Flash vs Fallback）", §3 (with a KV cache the triangular -inf mask is
 *    added to the LAST seq_len key columns only: key j is hidden from query i iff
 *    j - (Skv - Sq) > i), §4 (scores have shape [B, H, Q_len, K_len], heads-major), §5 (softmax
 *    in float, i.e. in a precision above the bf16 inputs).
 *
 * Readings where the pages leave a step open:
 *  - A masked key is left out of the max and of both sums. That is what adding -inf does, since
 *    exp(-inf) = 0; no finite stand-in such as -65504 is used.
 *  - GQA grouping is consecutive: query head h reads kv head h / (Hq / Hkv).
 *  - LSE is the natural logarithm of the sum over the SCALED scores.
 *  - Inputs are bf16 bit patterns widened exactly to double; `scale` is the fp32 value the GPU
 *    receives, widened exactly to double. All arithmetic is fp64.
 *  - causal with Sq > Skv is rejected (the cache-aligned mask leaves early rows with no key).
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARGS (-1)
#define ORACLE_ERR_NOMEM (-2)

/* bf16 -> double: a bf16 value is the upper 16 bits of an IEEE fp32 value, so the widening is exact. */
static double bf16_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* One query row: fills out[0..D) and *lse_out. `scores` is scratch of length Skv. */
static void oracle_row(const uint16_t *q_row, const uint16_t *k_head, const uint16_t *v_head,
                       int Skv, int D, int last_visible, double scale,
                       double *scores, double *out, double *lse_out)
{
    /* step 1: scaled dot products for the visible keys 0..last_visible */
    for (int j = 0; j <= last_visible; ++j) {
        const uint16_t *k_row = k_head + (size_t)j * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += bf16_to_double(q_row[d]) * bf16_to_double(k_row[d]);
        scores[j] = scale * dot;
    }
    (void)Skv;

    /* pass 1: row maximum over the visible keys */
    double m = -INFINITY;
    for (int j = 0; j <= last_visible; ++j)
        if (scores[j] > m)
            m = scores[j];

    /* pass 2: denominator */
    double l = 0.0;
    for (int j = 0; j <= last_visible; ++j)
        l += exp(scores[j] - m);

    /* pass 3: normalised weighted sum of the value rows, and the log-sum-exp */
    for (int d = 0; d < D; ++d)
        out[d] = 0.0;
    for (int j = 0; j <= last_visible; ++j) {
        double w = exp(scores[j] - m) / l;
        const uint16_t *v_row = v_head + (size_t)j * D;
        for (int d = 0; d < D; ++d)
            out[d] += w * bf16_to_double(v_row[d]);
    }
    *lse_out = m + log(l);
}

/*
 * q: [B, Hq, Sq, D], k/v: [B, Hkv, Skv, D], all bf16 bit patterns, contiguous.
 * rows: optional list of n_rows flat row ids r = (b * Hq + h) * Sq + i; NULL means every row in order.
 * o: [n_rows, D] fp64, lse: [n_rows] fp64.
 * n_threads <= 0 uses the OpenMP default.
 */
int oracle_attn(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                double *o, double *lse,
                int B, int Hq, int Hkv, int Sq, int Skv, int D,
                float scale, int causal,
                const int64_t *rows, int64_t n_rows, int n_threads)
{
    if (!q || !k || !v || !o || !lse)
        return ORACLE_ERR_ARGS;
    if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Skv < 1 || D < 1 || Hq % Hkv != 0)
        return ORACLE_ERR_ARGS;
    if (causal && Sq > Skv)
        return ORACLE_ERR_ARGS;
    const int64_t total_rows = (int64_t)B * Hq * Sq;
    if (rows == NULL)
        n_rows = total_rows;
    if (n_rows < 0)
        return ORACLE_ERR_ARGS;
    for (int64_t r = 0; rows && r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= total_rows)
            return ORACLE_ERR_ARGS;

    const int group = Hq / Hkv;
    const int offset = Skv - Sq; /* the mask covers the last Sq key columns */
    const double scale_d = (double)scale;
    int failed = 0;

#pragma omp parallel num_threads(n_threads > 0 ? n_threads : omp_get_max_threads())
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)Skv);
        if (!scores) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 8)
        for (int64_t r = 0; r < n_rows; ++r) {
            if (!scores)
                continue;
            const int64_t row = rows ? rows[r] : r;
            const int i = (int)(row % Sq);
            const int64_t bh = row / Sq;
            const int h = (int)(bh % Hq);
            const int b = (int)(bh / Hq);
            const int kvh = h / group;
            const int last_visible = causal ? i + offset : Skv - 1;
            const uint16_t *q_row = q + (size_t)row * D;
            const size_t kv_off = ((size_t)b * Hkv + kvh) * (size_t)Skv * D;
            oracle_row(q_row, k + kv_off, v + kv_off, Skv, D, last_visible, scale_d, scores,
                       o + (size_t)r * D, lse + r);
        }
        free(scores);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/*
 * Backward pass of the same operation, in fp64: given dO (the gradient of a loss with respect to
 * O), the gradients dQ, dK, dV.
 *
 * TEST INFRASTRUCTURE, like the forward above.
 *
 * The pages state only that the backward pass recomputes the softmax weights from the saved LSE
 * instead of storing them ("AI Infra 入门…", §3, LSE paragraph); the gradients below are the
 * textbook derivative of the forward definition above, written out with no blocking:
 *
 *   for every batch b, kv head g, every query head h of g's group and query row i:
 *     P_ij  = exp(s_ij - lse_i)                 (visible j; lse_i as in the forward: m + ln l)
 *     dP_ij = dO_i . v_j
 *     D_i   = sum_j P_ij dP_ij                  (equal to dO_i . O_i)
 *     dS_ij = P_ij (dP_ij - D_i)                (softmax derivative)
 *     dQ_i  = scale * sum_j dS_ij k_j
 *     dK_j += scale * dS_ij q_i                 (summed over rows and over the group's heads)
 *     dV_j += P_ij dO_i
 *
 * q: [B, Hq, Sq, D], k/v: [B, Hkv, Skv, D], dout: [B, Hq, Sq, D], all bf16 bit patterns.
 * dq: [B, Hq, Sq, D], dk/dv: [B, Hkv, Skv, D], fp64. Work is split over (b, kv head), so each
 * thread owns the dK/dV rows it accumulates.
 */
int oracle_attn_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                    double *dq, double *dk, double *dv,
                    int B, int Hq, int Hkv, int Sq, int Skv, int D,
                    float scale, int causal, int n_threads)
{
    if (!q || !k || !v || !dout || !dq || !dk || !dv)
        return ORACLE_ERR_ARGS;
    if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Skv < 1 || D < 1 || Hq % Hkv != 0)
        return ORACLE_ERR_ARGS;
    if (causal && Sq > Skv)
        return ORACLE_ERR_ARGS;
    const int group = Hq / Hkv;
    const int offset = Skv - Sq;
    const double scale_d = (double)scale;
    int failed = 0;

#pragma omp parallel num_threads(n_threads > 0 ? n_threads : omp_get_max_threads())
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)Skv);
        double *p = (double *)malloc(sizeof(double) * (size_t)Skv);
        double *dp = (double *)malloc(sizeof(double) * (size_t)Skv);
        if (!s || !p || !dp) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t bg = 0; bg < (int64_t)B * Hkv; ++bg) {
            if (!s || !p || !dp)
                continue;
            const int b = (int)(bg / Hkv);
            const int g = (int)(bg % Hkv);
            const size_t kv_off = ((size_t)b * Hkv + g) * (size_t)Skv * D;
            const uint16_t *k_head = k + kv_off;
            const uint16_t *v_head = v + kv_off;
            double *dk_head = dk + kv_off;
            double *dv_head = dv + kv_off;
            for (size_t e = 0; e < (size_t)Skv * D; ++e) {
                dk_head[e] = 0.0;
                dv_head[e] = 0.0;
            }
            for (int h = g * group; h < (g + 1) * group; ++h) {
                for (int i = 0; i < Sq; ++i) {
                    const size_t row = ((size_t)b * Hq + h) * Sq + i;
                    const uint16_t *q_row = q + row * D;
                    const uint16_t *do_row = dout + row * D;
                    double *dq_row = dq + row * D;
                    const int last = causal ? i + offset : Skv - 1;
                    /* scores, then lse exactly as the forward computes it */
                    double m = -INFINITY;
                    for (int j = 0; j <= last; ++j) {
                        double dot = 0.0;
                        for (int d = 0; d < D; ++d)
                            dot += bf16_to_double(q_row[d]) * bf16_to_double(k_head[(size_t)j * D + d]);
                        s[j] = scale_d * dot;
                        if (s[j] > m)
                            m = s[j];
                    }
                    double l = 0.0;
                    for (int j = 0; j <= last; ++j)
                        l += exp(s[j] - m);
                    const double lse = m + log(l);
                    /* weights, dP and D_i */
                    double Di = 0.0;
                    for (int j = 0; j <= last; ++j) {
                        p[j] = exp(s[j] - lse);
                        double dot = 0.0;
                        for (int d = 0; d < D; ++d)
                            dot += bf16_to_double(do_row[d]) * bf16_to_double(v_head[(size_t)j * D + d]);
                        dp[j] = dot;
                        Di += p[j] * dp[j];
                    }
                    /* gradients */
                    for (int d = 0; d < D; ++d)
                        dq_row[d] = 0.0;
                    for (int j = 0; j <= last; ++j) {
                        const double ds = p[j] * (dp[j] - Di);
                        for (int d = 0; d < D; ++d) {
                            dq_row[d] += scale_d * ds * bf16_to_double(k_head[(size_t)j * D + d]);
                            dk_head[(size_t)j * D + d] += scale_d * ds * bf16_to_double(q_row[d]);
                            dv_head[(size_t)j * D + d] += p[j] * bf16_to_double(do_row[d]);
                        }
                    }
                }
            }
        }
        free(s);
        free(p);
        free(dp);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/*
 * Attention over an FP8 (e4m3) K/V cache with per-channel scales, in fp64.
 *
 * TEST INFRASTRUCTURE, like the functions above.
 *
 * "MLA 矩阵乘法吸收的数值稳定性治理", §五: the KV cache may be stored in FP8 to save bandwidth,
 * with the products accumulated in higher precision; §二.1 of the same page scales each feature
 * channel by a coefficient. Reading taken here: one fp32 coefficient per (kv head, channel) for K
 * and one for V, and the cached value is code * coefficient:
 *
 *   k~[b,g,j,d] = e4m3(k8[b,g,j,d]) * k_scale[g,d],   v~[b,g,j,d] = e4m3(v8[b,g,j,d]) * v_scale[g,d]
 *
 * after which the result is the plain definition above with k~, v~ in place of k, v.
 *
 * e4m3 (the OCP 8-bit format with 4 exponent and 3 mantissa bits, bias 7, no infinities): bit 7
 * sign, bits 6-3 exponent e, bits 2-0 mantissa m. e = 0: (m / 8) * 2^-6; otherwise
 * (1 + m / 8) * 2^(e - 7), except e = 15 with m = 7, which is NaN. Largest finite value 448.
 */
static double e4m3_to_double(uint8_t code)
{
    const int sign = code >> 7;
    const int e = (code >> 3) & 15;
    const int m = code & 7;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* Decodes n e4m3 codes (exposed for the tests that pin the decoder). */
void oracle_decode_e4m3(const uint8_t *codes, double *out, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = e4m3_to_double(codes[i]);
}

/* One query row over the dequantised cache; n_vis keys (0..n_vis-1) are visible. */
static void fp8kv_row(const uint16_t *qv, const uint8_t *kc, const uint8_t *vc, const float *ks,
                      const float *vs, int D, int n_vis, double scale, double *sc, double *out,
                      double *lse_out)
{
    /* scaled scores against the dequantised keys k~ = e4m3(code) * ks[channel] */
    for (int j = 0; j < n_vis; ++j) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d) {
            const double kd = e4m3_to_double(kc[(size_t)j * D + d]) * (double)ks[d];
            acc += bf16_to_double(qv[d]) * kd;
        }
        sc[j] = acc * scale;
    }
    double mx = -INFINITY;
    for (int j = 0; j < n_vis; ++j)
        mx = sc[j] > mx ? sc[j] : mx;
    double den = 0.0;
    for (int j = 0; j < n_vis; ++j)
        den += exp(sc[j] - mx);
    for (int d = 0; d < D; ++d)
        out[d] = 0.0;
    for (int j = 0; j < n_vis; ++j) {
        const double wj = exp(sc[j] - mx) / den;
        for (int d = 0; d < D; ++d) {
            const double vd = e4m3_to_double(vc[(size_t)j * D + d]) * (double)vs[d];
            out[d] += wj * vd;
        }
    }
    *lse_out = mx + log(den);
}

/*
 * q: [B, Hq, Sq, D] bf16 bits; k8/v8: [B, Hkv, Skv, D] e4m3 codes; k_scale/v_scale: [Hkv, D] fp32.
 * rows, o, lse, n_threads: as oracle_attn.
 */
int oracle_attn_fp8kv(const uint16_t *q, const uint8_t *k8, const uint8_t *v8, const float *k_scale,
                      const float *v_scale, double *o, double *lse,
                      int B, int Hq, int Hkv, int Sq, int Skv, int D,
                      float scale, int causal,
                      const int64_t *rows, int64_t n_rows, int n_threads)
{
    if (!q || !k8 || !v8 || !k_scale || !v_scale || !o || !lse)
        return ORACLE_ERR_ARGS;
    if (B < 1 || Hq < 1 || Hkv < 1 || Sq < 1 || Skv < 1 || D < 1 || Hq % Hkv != 0)
        return ORACLE_ERR_ARGS;
    if (causal && Sq > Skv)
        return ORACLE_ERR_ARGS;
    const int64_t n_all = (int64_t)B * Hq * Sq;
    if (rows == NULL)
        n_rows = n_all;
    if (n_rows < 0)
        return ORACLE_ERR_ARGS;
    for (int64_t r = 0; rows && r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= n_all)
            return ORACLE_ERR_ARGS;
    int failed = 0;

#pragma omp parallel num_threads(n_threads > 0 ? n_threads : omp_get_max_threads())
    {
        double *sc = (double *)malloc(sizeof(double) * (size_t)Skv);
        if (!sc) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 8)
        for (int64_t r = 0; r < n_rows; ++r) {
            if (!sc)
                continue;
            const int64_t row = rows ? rows[r] : r;
            const int64_t bh = row / Sq;
            const int i = (int)(row - bh * Sq);
            const int b = (int)(bh / Hq);
            const int h = (int)(bh - (int64_t)b * Hq);
            const int g = h / (Hq / Hkv); /* kv head of query head h */
            const int n_vis = causal ? i + (Skv - Sq) + 1 : Skv;
            const size_t cache = ((size_t)b * Hkv + g) * (size_t)Skv * D;
            fp8kv_row(q + (size_t)row * D, k8 + cache, v8 + cache, k_scale + (size_t)g * D,
                      v_scale + (size_t)g * D, D, n_vis, (double)scale, sc, o + (size_t)r * D, lse + r);
        }
        free(sc);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}
