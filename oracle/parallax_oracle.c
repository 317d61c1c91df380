/*
 * parallax_oracle.c -- the fp64 CPU oracle for the Parallax attention operator.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is read by the parity tests, by the
 * smoke check and by the CPU-baseline leg of the benchmark.  The product path
 * (the CUDA library) never links, loads or calls it, and it shares no code,
 * header, table or helper with that library.
 *
 * What it computes (plain definition, no blocking, no one-pass rewrite):
 *
 *   For one query row i with key set J (causal: keys 0..i; full: all keys;
 *   decode: the first seqlen rows of the cache):
 *     z_j  = (q_i . k_j) / sqrt(d)                      scaled scores
 *     mu   = max_j z_j,  e_j = exp(z_j - mu),  l = sum_j e_j
 *     s_j  = e_j / l                                    softmax weights
 *     lse  = mu + ln(l)                                 natural log
 *     o    = sum_j s_j v_j                              softmax attention
 *     kbar = sum_j s_j k_j                              weighted key mean
 *     c    = sum_j s_j ((k_j - kbar) . rho_i) (v_j - o) = C_i rho_i
 *     y_i  = o - c
 *   with C_i = sum_j s_j (v_j - o)(k_j - kbar)^T the softmax-weighted
 *   value/key covariance (d_v x d_k) and rho_i the learned probe.
 *
 * Sources:
 *   - zubnet.ai news item "Parallax mantiene softmax, correccion de covarianza
 *     aprendida" (paragraph 2, "El mecanismo es aditivo"): the output equals
 *     softmax attention minus a projected covariance term; the KV covariance
 *     is multiplied by a learned probe rho_i = W_R x_i taken from the layer
 *     input; W_R = 0 recovers standard softmax exactly.
 *   - encorp.ai blog "Integraciones de IA personalizadas tras la atencion
 *     Parallax", section "Por que eliminar el solucionador de gradiente
 *     conjugado...": the per-query solve of Local Linear Attention is replaced
 *     by a learned projector W_R acting on the layer input.
 *   Readings where the pages are silent (which covariance, the sign, the
 *   weights, the layout of W_R) are the plainest ones: the same softmax
 *   weights s_j (summing to one, no n/(n-1) correction), rho probing the key
 *   side (a_ij = k_j . rho_i, no 1/sqrt(d) on it), a minus sign, and
 *   rho[b,h,t,:] = x[b,t,:] @ W_R[:, h*d:(h+1)*d] with W_R stored
 *   [d_model, H*d] row-major, no bias.
 *
 * Floating point: every operation is IEEE fp64 in source order.  Build with
 * -O2 -ffp-contract=off and without -ffast-math so the compiler neither fuses
 * nor reassociates.  OpenMP only distributes independent rows over threads;
 * it changes no arithmetic inside a row.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* One query row against n keys.  K and V point at n rows of d doubles.      */
/* rho_i may be NULL: then the covariance branch is absent (softmax only).    */
/* z is caller scratch of n doubles.  Returns nothing; writes y_i, *lse_i.    */
/* ------------------------------------------------------------------------ */
static void row_parallax(const double *q_i, const double *K, const double *V,
                         const double *rho_i, long n, int d,
                         double *y_i, double *lse_i, double *z)
{
    int e;
    long j;
    if (n <= 0) {
        /* Empty key set: defined as y = 0 and lse = -inf. */
        for (e = 0; e < d; ++e) y_i[e] = 0.0;
        if (lse_i) *lse_i = -INFINITY;
        return;
    }
    const double inv_sqrt_d = 1.0 / sqrt((double)d);

    /* scaled scores and their maximum */
    double mu = -INFINITY;
    for (j = 0; j < n; ++j) {
        const double *k_j = K + (size_t)j * d;
        double dot = 0.0;
        for (e = 0; e < d; ++e) dot += q_i[e] * k_j[e];
        z[j] = dot * inv_sqrt_d;
        if (z[j] > mu) mu = z[j];
    }

    /* softmax weights: e_j = exp(z_j - mu), s_j = e_j / l */
    double l = 0.0;
    for (j = 0; j < n; ++j) {
        z[j] = exp(z[j] - mu);
        l += z[j];
    }
    for (j = 0; j < n; ++j) z[j] = z[j] / l;       /* z now holds s_j */
    if (lse_i) *lse_i = mu + log(l);

    /* pass 1: o = sum s_j v_j, kbar = sum s_j k_j */
    double *o = y_i;                                 /* o is built in y_i */
    double *kbar = (double *)calloc((size_t)d, sizeof(double));
    for (e = 0; e < d; ++e) o[e] = 0.0;
    for (j = 0; j < n; ++j) {
        const double s = z[j];
        const double *k_j = K + (size_t)j * d;
        const double *v_j = V + (size_t)j * d;
        for (e = 0; e < d; ++e) {
            o[e] += s * v_j[e];
            kbar[e] += s * k_j[e];
        }
    }
    if (rho_i == NULL) {                             /* softmax only: y = o */
        free(kbar);
        return;
    }

    /* pass 2, centered: c = sum_j s_j ((k_j - kbar) . rho) (v_j - o) */
    double *c = (double *)calloc((size_t)d, sizeof(double));
    for (j = 0; j < n; ++j) {
        const double *k_j = K + (size_t)j * d;
        const double *v_j = V + (size_t)j * d;
        double proj = 0.0;
        for (e = 0; e < d; ++e) proj += (k_j[e] - kbar[e]) * rho_i[e];
        const double w = z[j] * proj;
        for (e = 0; e < d; ++e) c[e] += w * (v_j[e] - o[e]);
    }
    for (e = 0; e < d; ++e) y_i[e] = o[e] - c[e];
    free(c);
    free(kbar);
}

/* ------------------------------------------------------------------------ */
/* Prefill / forward.  q,k,v,rho,y: [B,H,T,d] row-major; lse: [B,H,T].       */
/* rho may be NULL (softmax only); lse may be NULL.                          */
/* causal != 0: query i sees keys 0..i; else all T keys.                     */
/* ------------------------------------------------------------------------ */
int oracle_fwd(const double *q, const double *k, const double *v, const double *rho,
               double *y, double *lse, int B, int H, int T, int d, int causal)
{
    if (B < 0 || H < 0 || T < 0 || d <= 0) return 1;
    const long rows = (long)B * H * T;
    long r;
#pragma omp parallel for schedule(dynamic, 16)
    for (r = 0; r < rows; ++r) {
        const long bh = r / T;
        const long i = r % T;
        const size_t head = (size_t)bh * T * d;
        const long n = causal ? i + 1 : T;
        double *z = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        row_parallax(q + head + (size_t)i * d, k + head, v + head,
                     rho ? rho + head + (size_t)i * d : NULL, n, d,
                     y + head + (size_t)i * d, lse ? lse + r : NULL, z);
        free(z);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Forward on a subset of rows.  rows[n] are flat row ids (bh*T + i); the    */
/* results go to y_rows[n, d] and lse_rows[n] in the order given.            */
/* ------------------------------------------------------------------------ */
int oracle_fwd_rows(const double *q, const double *k, const double *v, const double *rho,
                    int B, int H, int T, int d, int causal,
                    const long *rows, long nrows, double *y_rows, double *lse_rows)
{
    if (B < 0 || H < 0 || T < 0 || d <= 0) return 1;
    const long total = (long)B * H * T;
    long t;
    for (t = 0; t < nrows; ++t)
        if (rows[t] < 0 || rows[t] >= total) return 2;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < nrows; ++t) {
        const long r = rows[t];
        const long bh = r / T;
        const long i = r % T;
        const size_t head = (size_t)bh * T * d;
        const long n = causal ? i + 1 : T;
        double *z = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        row_parallax(q + head + (size_t)i * d, k + head, v + head,
                     rho ? rho + head + (size_t)i * d : NULL, n, d,
                     y_rows + (size_t)t * d, lse_rows ? lse_rows + t : NULL, z);
        free(z);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Decode: one query per (b,h) against the first seqlens[b] cache rows.      */
/* q,rho,y: [B,H,d]; kc,vc: [B,H,Tcap,d]; seqlens: [B]; lse: [B,H].          */
/* The cache already holds the current token.  Only the (b,h) pairs listed   */
/* in bh_list (flat b*H+h, nbh entries) are computed when bh_list != NULL;   */
/* their results go to y[t*d..], lse[t] in list order.                       */
/* ------------------------------------------------------------------------ */
int oracle_decode(const double *q, const double *rho, const double *kc, const double *vc,
                  const int *seqlens, double *y, double *lse,
                  int B, int H, int Tcap, int d, const long *bh_list, long nbh)
{
    if (B < 0 || H < 0 || Tcap < 0 || d <= 0) return 1;
    long count = bh_list ? nbh : (long)B * H;
    long t;
    for (t = 0; t < (bh_list ? nbh : 0); ++t)
        if (bh_list[t] < 0 || bh_list[t] >= (long)B * H) return 2;
    for (t = 0; t < B; ++t)
        if (seqlens[t] < 0 || seqlens[t] > Tcap) return 3;
#pragma omp parallel for schedule(dynamic, 1)
    for (t = 0; t < count; ++t) {
        const long bh = bh_list ? bh_list[t] : t;
        const long b = bh / H;
        const long n = seqlens[b];
        const size_t cache = (size_t)bh * Tcap * d;
        double *z = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        row_parallax(q + (size_t)bh * d, kc + cache, vc + cache,
                     rho ? rho + (size_t)bh * d : NULL, n, d,
                     y + (size_t)t * d, lse ? lse + t : NULL, z);
        free(z);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* rho projection: rho[b,h,t,e] = sum_c x[b,t,c] * W_R[c, h*d + e].          */
/* x: [B,T,dm]; W_R: [dm, H*d] row-major; rho: [B,H,T,d].                     */
/* When bt_list != NULL only the listed token rows (flat b*T+t) are done and */
/* written to rho[tt, H, d] in list order.                                    */
/* ------------------------------------------------------------------------ */
int oracle_rho_proj(const double *x, const double *W, double *rho,
                    int B, int T, int dm, int H, int d, const long *bt_list, long nbt)
{
    if (B < 0 || T < 0 || dm <= 0 || H <= 0 || d <= 0) return 1;
    const long count = bt_list ? nbt : (long)B * T;
    const long N = (long)H * d;
    long t;
    for (t = 0; t < (bt_list ? nbt : 0); ++t)
        if (bt_list[t] < 0 || bt_list[t] >= (long)B * T) return 2;
#pragma omp parallel for schedule(static)
    for (t = 0; t < count; ++t) {
        const long bt = bt_list ? bt_list[t] : t;
        const long b = bt / T;
        const long tok = bt % T;
        const double *x_row = x + (size_t)bt * dm;
        long h, e, c;
        for (h = 0; h < H; ++h) {
            for (e = 0; e < d; ++e) {
                double acc = 0.0;
                for (c = 0; c < dm; ++c) acc += x_row[c] * W[(size_t)c * N + h * d + e];
                if (bt_list)
                    rho[((size_t)t * H + h) * d + e] = acc;
                else
                    rho[(((size_t)b * H + h) * T + tok) * d + e] = acc;
            }
        }
    }
    return 0;
}

/* Threads the oracle will use (OpenMP), 1 when built without OpenMP. */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
