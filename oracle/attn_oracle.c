/*
 * attn_oracle.c -- plain FP64 CPU oracle for the scaled dot-product attention
 * forward.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * bench's CPU-baseline / reference arm may call it; the product path never
 * does.  It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (the definition, written out with no blocking, fusion or
 * reordering):
 *
 *   Attention(Q, K, V) = softmax(Q K^T / sqrt(d_k)) V
 *       -- rkmt.cn "GPU attention operator optimisation" page, section 1
 *          (the formula in the opening paragraph).
 *
 *   The three steps, in the order that page and the bjdmk.com.cn survey
 *   page (section 1, "Query-Key product, softmax normalisation, Value
 *   weighted sum") give them:
 *     1. S[i][j] = scale * sum_c Q[i][c] * K[j][c]          (scores)
 *        causal: S[i][j] = -inf for j > i + (s_k - s_q)    (mask; the
 *        intelliparadigm.com AVO page, section 2.2, fuses the mask into
 *        the softmax -- here it is simply applied to S.  The pages only
 *        use s_q = s_k, where this is j > i.  They never say how the mask
 *        lines up when s_q < s_k; the reading taken here aligns it to the
 *        bottom-right corner: the s_q queries are taken to be the LAST s_q
 *        positions of the key sequence, so the last query sees every key
 *        and s_q > s_k is refused, since a row would then see no key)
 *        sliding window (window_left >= 0, causal only): also
 *        S[i][j] = -inf for j < i + (s_k - s_q) - window_left, so row i
 *        sees the window_left + 1 keys ending at its diagonal.  The pages
 *        name a local-window variant without defining it; the reading
 *        taken is this one-sided window on top of the causal mask)
 *     2. m_i = max_j S[i][j];  E = exp(S - m_i);  l_i = sum_j E[i][j];
 *        P = E / l_i        (numerically stable softmax with the scale
 *        applied before the max, as in the AVO page, section 3.1 item 2)
 *     3. O[i][:] = sum_j P[i][j] V[j][:]
 *   plus the per-row log-sum-exp of the scaled scores, LSE_i = m_i + ln l_i
 *   (the pages do not define it; the reading taken is the natural log of
 *   the sum of exp over the scaled, masked scores of the row, m included).
 *
 *   Head sharing (grouped-query attention, rkmt.cn page section 3.2): query
 *   head h reads key/value head h / (h_q / h_kv) -- contiguous groups.
 *
 * Layouts (all contiguous, row-major):
 *   q   : bf16 bits [batch][s_q][h_q][d]
 *   k,v : bf16 bits [batch][s_k][h_kv][d]
 *   rows: int32 [batch][h_q][n_rows] query indices to evaluate (NULL: every
 *         row 0..s_q-1, and n_rows must equal s_q)
 *   o   : double [batch][h_q][n_rows][d]
 *   lse : double [batch][h_q][n_rows]
 *   p   : optional double [batch][h_q][n_rows][s_k] (the normalised P)
 *
 * BF16 inputs are decoded exactly (a bf16 value is the top half of an IEEE
 * binary32), then widened to double; everything after that is FP64.
 *
 * Returns 0 on success, a negative code on a bad argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Decode a whole bf16 array into doubles (done once so the inner loops read
 * plain doubles). */
static double *decode_bf16(const uint16_t *src, int64_t n)
{
    double *dst = (double *)malloc((size_t)n * sizeof(double));
    if (!dst) return NULL;
    for (int64_t i = 0; i < n; ++i) dst[i] = bf16_bits_to_double(src[i]);
    return dst;
}

/* One (batch, query head) pair over a chunk of its requested rows.
 * S is materialised for the chunk: n_chunk x s_k doubles. */
static void attend_rows(const double *Q, const double *K, const double *V,
                        int b, int h, int h_q, int h_kv, int s_q, int s_k,
                        int d, int causal, int window_left, double scale,
                        const int32_t *rows, int r0, int r1, int n_rows,
                        double *o, double *lse, double *p, double *S)
{
    const int group = h_q / h_kv;
    const int g = h / group;                      /* key/value head */
    const int64_t q_row_stride = (int64_t)h_q * d;  /* step of one token */
    const int64_t kv_row_stride = (int64_t)h_kv * d;
    const double *Qb = Q + (int64_t)b * s_q * q_row_stride + (int64_t)h * d;
    const double *Kb = K + (int64_t)b * s_k * kv_row_stride + (int64_t)g * d;
    const double *Vb = V + (int64_t)b * s_k * kv_row_stride + (int64_t)g * d;
    const int64_t bh = (int64_t)b * h_q + h;
    const int off = s_k - s_q;  /* causal: row i sees keys 0 .. i + off */

    for (int r = r0; r < r1; ++r) {
        const int i = rows ? rows[bh * n_rows + r] : r;
        double *Srow = S + (int64_t)(r - r0) * s_k;

        /* step 1: scores, then the causal mask */
        for (int j = 0; j < s_k; ++j) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c)
                dot += Qb[(int64_t)i * q_row_stride + c] *
                       Kb[(int64_t)j * kv_row_stride + c];
            Srow[j] = scale * dot;
            if (causal && j > i + off) Srow[j] = -INFINITY;
            if (window_left >= 0 && j < i + off - window_left) Srow[j] = -INFINITY;
        }

        /* step 2: stable softmax over the row */
        double m = -INFINITY;
        for (int j = 0; j < s_k; ++j)
            if (Srow[j] > m) m = Srow[j];
        double l = 0.0;
        for (int j = 0; j < s_k; ++j) {
            Srow[j] = exp(Srow[j] - m); /* E[i][j]; exp(-inf) = 0 */
            l += Srow[j];
        }
        for (int j = 0; j < s_k; ++j) Srow[j] = Srow[j] / l; /* P[i][j] */

        if (p) memcpy(p + (bh * n_rows + r) * s_k, Srow, (size_t)s_k * sizeof(double));

        /* step 3: P times V.  orow[c] accumulates P[j] * V[j][c] over
         * j = 0, 1, ..., s_k-1 in that order (the loops are nested j-outer
         * only so V is read row by row). */
        double *orow = o + (bh * n_rows + r) * d;
        for (int c = 0; c < d; ++c) orow[c] = 0.0;
        for (int j = 0; j < s_k; ++j) {
            const double *vrow = Vb + (int64_t)j * kv_row_stride;
            for (int c = 0; c < d; ++c)
                orow[c] += Srow[j] * vrow[c];
        }
        lse[bh * n_rows + r] = m + log(l);
    }
}

/* FP8 E4M3 (the "e4m3fn" variant): 1 sign bit, 4 exponent bits with bias 7,
 * 3 mantissa bits; exponent 0 encodes subnormals m * 2^-9; there are no
 * infinities, and S.1111.111 is NaN.  Decoded exactly into a double. */
static double e4m3_to_double(uint8_t bits)
{
    const int sign = bits >> 7, e = (bits >> 3) & 15, m = bits & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -mag : mag;
}

double oracle_e4m3_to_double(uint8_t bits) { return e4m3_to_double(bits); }

static int forward_on_doubles(double *Q, double *K, double *V, int batch, int h_q, int h_kv,
                              int s_q, int s_k, int d, int causal, int window_left,
                              double scale, const int32_t *rows, int n_rows, double *o,
                              double *lse, double *p);

int oracle_attn_fwd_f64(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        int batch, int h_q, int h_kv, int s_q, int s_k, int d,
                        int causal, int window_left, double scale,
                        const int32_t *rows, int n_rows,
                        double *o, double *lse, double *p)
{
    if (!q || !k || !v || !o || !lse) return -1;
    if (batch <= 0 || h_q <= 0 || h_kv <= 0 || s_q <= 0 || s_k <= 0 || d <= 0) return -2;
    if (h_q % h_kv != 0) return -3;
    if (n_rows <= 0 || (!rows && n_rows != s_q)) return -4;
    if (rows) {
        for (int64_t t = 0; t < (int64_t)batch * h_q * n_rows; ++t)
            if (rows[t] < 0 || rows[t] >= s_q) return -5;
    }
    /* A causal row must see at least one key (row i sees keys 0..i). */
    if (causal && s_q > s_k) return -6;
    /* A window is a causal mask's lower edge. */
    if (window_left < -1 || (window_left >= 0 && !causal)) return -8;

    double *Q = decode_bf16(q, (int64_t)batch * s_q * h_q * d);
    double *K = decode_bf16(k, (int64_t)batch * s_k * h_kv * d);
    double *V = decode_bf16(v, (int64_t)batch * s_k * h_kv * d);
    if (!Q || !K || !V) { free(Q); free(K); free(V); return -7; }
    return forward_on_doubles(Q, K, V, batch, h_q, h_kv, s_q, s_k, d, causal, window_left,
                              scale, rows, n_rows, o, lse, p);
}

/*
 * The forward on FP8 E4M3 inputs with per-tensor scales: the inputs are the
 * values Q = q_scale * e4m3(q), K = k_scale * e4m3(k), V = v_scale * e4m3(v),
 * decoded exactly into doubles; everything after that is the forward above
 * (the pages' low-precision GEMM inputs with higher-precision softmax: the
 * bjdmk.com.cn survey page, section 3; the rkmt.cn page, section 3.1.1).
 * Layouts as oracle_attn_fwd_f64 with one byte per input element.
 */
int oracle_attn_fwd_fp8_f64(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                            double q_scale, double k_scale, double v_scale,
                            int batch, int h_q, int h_kv, int s_q, int s_k, int d,
                            int causal, int window_left, double scale,
                            const int32_t *rows, int n_rows,
                            double *o, double *lse, double *p)
{
    if (!q || !k || !v || !o || !lse) return -1;
    if (batch <= 0 || h_q <= 0 || h_kv <= 0 || s_q <= 0 || s_k <= 0 || d <= 0) return -2;
    if (h_q % h_kv != 0) return -3;
    if (n_rows <= 0 || (!rows && n_rows != s_q)) return -4;
    if (causal && s_q > s_k) return -6;
    if (window_left < -1 || (window_left >= 0 && !causal)) return -8;
    const int64_t nq = (int64_t)batch * s_q * h_q * d, nk = (int64_t)batch * s_k * h_kv * d;
    double *Q = (double *)malloc((size_t)nq * sizeof(double));
    double *K = (double *)malloc((size_t)nk * sizeof(double));
    double *V = (double *)malloc((size_t)nk * sizeof(double));
    if (!Q || !K || !V) { free(Q); free(K); free(V); return -7; }
    for (int64_t t = 0; t < nq; ++t) Q[t] = q_scale * e4m3_to_double(q[t]);
    for (int64_t t = 0; t < nk; ++t) {
        K[t] = k_scale * e4m3_to_double(k[t]);
        V[t] = v_scale * e4m3_to_double(v[t]);
    }
    return forward_on_doubles(Q, K, V, batch, h_q, h_kv, s_q, s_k, d, causal, window_left,
                              scale, rows, n_rows, o, lse, p);
}

/* Shared tail of both forward entries: takes ownership of Q, K, V. */
static int forward_on_doubles(double *Q, double *K, double *V, int batch, int h_q, int h_kv,
                              int s_q, int s_k, int d, int causal, int window_left,
                              double scale, const int32_t *rows, int n_rows, double *o,
                              double *lse, double *p)
{
    if (rows) {
        for (int64_t t = 0; t < (int64_t)batch * h_q * n_rows; ++t)
            if (rows[t] < 0 || rows[t] >= s_q) { free(Q); free(K); free(V); return -5; }
    }
    const int chunk = 32;
    const int n_chunks = (n_rows + chunk - 1) / chunk;
    const int64_t n_tasks = (int64_t)batch * h_q * n_chunks;
    int failed = 0;

#pragma omp parallel
    {
        double *S = (double *)malloc((size_t)chunk * s_k * sizeof(double));
        if (!S) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < n_tasks; ++t) {
            if (!S) continue;
            const int64_t bh = t / n_chunks;
            const int cidx = (int)(t % n_chunks);
            const int b = (int)(bh / h_q), h = (int)(bh % h_q);
            const int r0 = cidx * chunk;
            const int r1 = r0 + chunk < n_rows ? r0 + chunk : n_rows;
            attend_rows(Q, K, V, b, h, h_q, h_kv, s_q, s_k, d, causal, window_left, scale,
                        rows, r0, r1, n_rows, o, lse, p, S);
        }
        free(S);
    }
    free(Q); free(K); free(V);
    return failed ? -7 : 0;
}

/* Number of OpenMP threads the oracle will use (reported beside its timing). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * ---------------------------------------------------------------------------
 * Backward pass (gradients of the forward above).  TEST INFRASTRUCTURE ONLY,
 * like the forward.
 *
 * The pages describe FlashAttention's backward as recomputing the attention
 * weights from saved row statistics instead of storing them (bjdmk.com.cn
 * survey page, section 5.1) and reusing the forward's intermediates
 * (intelliparadigm.com AVO page, section 3.2).  What the backward computes is
 * fixed by the chain rule applied to the forward's definition; this is that
 * definition written out, with P materialised from scratch (no saved
 * statistics are taken from the caller):
 *
 *   P   = softmax_rows(scale * Q K^T + mask)      (as in the forward)
 *   dV  = P^T dO                                   dV[j] = sum_i P[i][j] dO[i]
 *   dP  = dO V^T                                   dP[i][j] = dO[i] . V[j]
 *   D_i = sum_j P[i][j] dP[i][j]
 *   dS  = P * (dP - D)                             (elementwise, D per row)
 *   dQ  = scale * dS K                             dQ[i] = scale sum_j dS[i][j] K[j]
 *   dK  = scale * dS^T Q                           dK[j] = scale sum_i dS[i][j] Q[i]
 *
 * (the softmax Jacobian dS[i][j] = sum_k dP[i][k] P[i][k] (delta_jk - P[i][j])
 * gives the dS line).  Grouped heads: dK and dV of key/value head g sum the
 * contributions of every query head h with h / (h_q / h_kv) = g.
 *
 * Layouts: q, do bf16 bits [batch][s_q][h_q][d]; k, v [batch][s_k][h_kv][d];
 * dq double [batch][s_q][h_q][d]; dk, dv double [batch][s_k][h_kv][d].
 * causal / window_left as the forward.  Returns 0, or a negative code on a
 * bad argument (-7: out of memory).
 */
static void backward_group(const double *Q, const double *K, const double *V, const double *dO,
                           int b, int g, int h_q, int h_kv, int s_q, int s_k, int d,
                           int causal, int window_left, double scale,
                           double *dq, double *dk, double *dv, double *P, double *dP)
{
    const int group = h_q / h_kv;
    const int64_t qs = (int64_t)h_q * d, ks = (int64_t)h_kv * d;
    const int off = s_k - s_q;
    const double *Kb = K + (int64_t)b * s_k * ks + (int64_t)g * d;
    const double *Vb = V + (int64_t)b * s_k * ks + (int64_t)g * d;
    double *dKb = dk + (int64_t)b * s_k * ks + (int64_t)g * d;
    double *dVb = dv + (int64_t)b * s_k * ks + (int64_t)g * d;

    for (int h = g * group; h < (g + 1) * group; ++h) {
        const double *Qb = Q + (int64_t)b * s_q * qs + (int64_t)h * d;
        const double *dOb = dO + (int64_t)b * s_q * qs + (int64_t)h * d;
        double *dQb = dq + (int64_t)b * s_q * qs + (int64_t)h * d;

        /* P, row by row (the forward's steps 1 and 2) */
        for (int i = 0; i < s_q; ++i) {
            double *Prow = P + (int64_t)i * s_k;
            for (int j = 0; j < s_k; ++j) {
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += Qb[(int64_t)i * qs + c] * Kb[(int64_t)j * ks + c];
                Prow[j] = scale * dot;
                if (causal && j > i + off) Prow[j] = -INFINITY;
                if (window_left >= 0 && j < i + off - window_left) Prow[j] = -INFINITY;
            }
            double m = -INFINITY;
            for (int j = 0; j < s_k; ++j)
                if (Prow[j] > m) m = Prow[j];
            double l = 0.0;
            for (int j = 0; j < s_k; ++j) {
                Prow[j] = exp(Prow[j] - m);
                l += Prow[j];
            }
            for (int j = 0; j < s_k; ++j) Prow[j] = Prow[j] / l;
        }
        /* dP = dO V^T, D_i = sum_j P dP, dS = P (dP - D) (stored over dP) */
        for (int i = 0; i < s_q; ++i) {
            const double *Prow = P + (int64_t)i * s_k;
            double *dProw = dP + (int64_t)i * s_k;
            for (int j = 0; j < s_k; ++j) {
                double dot = 0.0;
                for (int c = 0; c < d; ++c) dot += dOb[(int64_t)i * qs + c] * Vb[(int64_t)j * ks + c];
                dProw[j] = dot;
            }
            double Di = 0.0;
            for (int j = 0; j < s_k; ++j) Di += Prow[j] * dProw[j];
            for (int j = 0; j < s_k; ++j) dProw[j] = Prow[j] * (dProw[j] - Di);
        }
        /* dQ = scale dS K */
        for (int i = 0; i < s_q; ++i) {
            const double *dSrow = dP + (int64_t)i * s_k;
            for (int c = 0; c < d; ++c) {
                double acc = 0.0;
                for (int j = 0; j < s_k; ++j) acc += dSrow[j] * Kb[(int64_t)j * ks + c];
                dQb[(int64_t)i * qs + c] = scale * acc;
            }
        }
        /* dK += scale dS^T Q;  dV += P^T dO  (summed over the group's heads) */
        for (int j = 0; j < s_k; ++j) {
            for (int c = 0; c < d; ++c) {
                double acc_k = 0.0, acc_v = 0.0;
                for (int i = 0; i < s_q; ++i) {
                    acc_k += dP[(int64_t)i * s_k + j] * Qb[(int64_t)i * qs + c];
                    acc_v += P[(int64_t)i * s_k + j] * dOb[(int64_t)i * qs + c];
                }
                dKb[(int64_t)j * ks + c] += scale * acc_k;
                dVb[(int64_t)j * ks + c] += acc_v;
            }
        }
    }
}

int oracle_attn_bwd_f64(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const uint16_t *dout, int batch, int h_q, int h_kv, int s_q, int s_k,
                        int d, int causal, int window_left, double scale,
                        double *dq, double *dk, double *dv)
{
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return -1;
    if (batch <= 0 || h_q <= 0 || h_kv <= 0 || s_q <= 0 || s_k <= 0 || d <= 0) return -2;
    if (h_q % h_kv != 0) return -3;
    if (causal && s_q > s_k) return -6;
    if (window_left < -1 || (window_left >= 0 && !causal)) return -8;

    const int64_t nq = (int64_t)batch * s_q * h_q * d, nk = (int64_t)batch * s_k * h_kv * d;
    double *Q = decode_bf16(q, nq), *K = decode_bf16(k, nk), *V = decode_bf16(v, nk);
    double *dO = decode_bf16(dout, nq);
    if (!Q || !K || !V || !dO) { free(Q); free(K); free(V); free(dO); return -7; }
    for (int64_t t = 0; t < nk; ++t) { dk[t] = 0.0; dv[t] = 0.0; }

    const int64_t n_tasks = (int64_t)batch * h_kv;
    int failed = 0;
#pragma omp parallel
    {
        double *P = (double *)malloc((size_t)s_q * s_k * sizeof(double));
        double *dP = (double *)malloc((size_t)s_q * s_k * sizeof(double));
        if (!P || !dP) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < n_tasks; ++t) {
            if (!P || !dP) continue;
            backward_group(Q, K, V, dO, (int)(t / h_kv), (int)(t % h_kv), h_q, h_kv, s_q, s_k, d,
                           causal, window_left, scale, dq, dk, dv, P, dP);
        }
        free(P);
        free(dP);
    }
    free(Q); free(K); free(V); free(dO);
    return failed ? -7 : 0;
}
