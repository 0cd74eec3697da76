/*
 * rtr_oracle.c -- plain, slow, double-precision reference for the masked
 * attention of RTR-DiT ("DiT as Real-Time Rerenderer: Streaming Video
 * Stylization with Autoregressive Diffusion Transformer", papernotes.org note,
 * Method > Key Designs 2, the attention/mask equation).
 *
 * TEST INFRASTRUCTURE.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library) shares no code with it and never calls it.
 *
 * What it computes, written out from the definition with no blocking, no
 * online softmax and no reordering:
 *
 *   Attn(Q,K,V) = softmax(Q K^T / sqrt(d) + M) V,
 *   M[i][j] = 0 if floor(j/k) <= floor(i/k), -inf otherwise,
 *
 * where d is the head dimension and k the number of spatial tokens per latent
 * frame (same section).  i and j are LOGICAL positions in the token sequence;
 * tokens of one frame see each other and a frame sees only earlier frames.
 *
 * Layout of every tensor is [tokens][heads][d], row-major, double precision.
 * The caller converts its bf16 / fp32 input bits to double exactly before the
 * call, so the oracle sees the same values the GPU sees.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* The mask M of the attention equation: query at logical position i may see
 * key at logical position j iff floor(j/k) <= floor(i/k).  Positions are
 * non-negative, so C integer division is the floor. */
int rtr_oracle_visible(int64_t i, int64_t j, int64_t k)
{
    return (j / k) <= (i / k);
}

/*
 * Masked softmax attention for a set of query rows.
 *
 *   q      [nq][heads][d]   query rows
 *   q_pos  [nq]             logical position of each query row
 *   key    [nk][heads][d]   keys; key j sits at logical position j
 *   val    [nk][heads][d]   values
 *   k_per_frame             k of the mask equation (tokens per latent frame)
 *   causal                  1: apply M;  0: every key is visible (the
 *                           unmasked attention of cross-attention / the
 *                           bidirectional teacher)
 *   scale                   multiplies q.k (1/sqrt(d) in the equation)
 *   out    [nq][heads][d]
 *
 * Returns 0, or 1 if a row's work buffers could not be allocated (that row's
 * output is then left as NaN and the caller must treat the result as
 * failed).
 * Per (row, head):  s_j = scale * sum_t q_t key_jt over visible j,
 * m = max_j s_j, p_j = exp(s_j - m), out = sum_j p_j val_j / sum_j p_j.
 * Subtracting m is the usual exact rewrite of softmax (it cancels in the
 * ratio) and keeps exp() finite.  A row that sees no key returns zeros.
 */
int rtr_oracle_attention(const double *q, const int64_t *q_pos, int64_t nq,
                          const double *key, const double *val, int64_t nk,
                          int64_t heads, int64_t d, int64_t k_per_frame,
                          int causal, double scale, double *out, int nthreads)
{
#ifdef _OPENMP
    /* the thread count applies to this call only */
    const int nt = nthreads > 0 ? nthreads : omp_get_max_threads();
#else
    (void)nthreads;
#endif
    int64_t npairs = nq * heads;
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (int64_t pr = 0; pr < npairs; ++pr) {
        int64_t r = pr / heads, h = pr % heads;
        const double *qi = q + (r * heads + h) * d;
        double *oi = out + (r * heads + h) * d;
        double *s = (double *)malloc((size_t)(nk > 0 ? nk : 1) * sizeof(double));
        unsigned char *vis = (unsigned char *)malloc((size_t)(nk > 0 ? nk : 1));
        if (!s || !vis) {
            free(s);
            free(vis);
            for (int64_t t = 0; t < d; ++t) oi[t] = NAN;
#pragma omp atomic write
            failed = 1;
            continue;
        }
        double m = -INFINITY;
        for (int64_t j = 0; j < nk; ++j) {
            vis[j] = causal ? (unsigned char)rtr_oracle_visible(q_pos[r], j, k_per_frame) : 1;
            if (!vis[j]) continue;
            const double *kj = key + (j * heads + h) * d;
            double dot = 0.0;
            for (int64_t t = 0; t < d; ++t) dot += qi[t] * kj[t];
            s[j] = scale * dot;
            if (s[j] > m) m = s[j];
        }
        double den = 0.0;
        for (int64_t t = 0; t < d; ++t) oi[t] = 0.0;
        for (int64_t j = 0; j < nk; ++j) {
            if (!vis[j]) continue;
            double p = exp(s[j] - m);
            den += p;
            const double *vj = val + (j * heads + h) * d;
            for (int64_t t = 0; t < d; ++t) oi[t] += p * vj[t];
        }
        if (den > 0.0)
            for (int64_t t = 0; t < d; ++t) oi[t] /= den;
        free(s);
        free(vis);
    }
    return failed;
}

/* Number of threads OpenMP would use (reported next to CPU timings). */
int rtr_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
