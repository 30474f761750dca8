/*
 * swa_oracle.c - plain float64 CPU reference for sliding-window attention (SWA)
 * with grouped-query attention (GQA).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle the CUDA path is checked
 * against.  Only the tests, the smoke check and the benchmark's CPU-baseline leg
 * may load it; the library's product path never calls it, and it shares no
 * code, header or table with the CUDA path.
 *
 * What it computes (Mistral 7B, section 2 "Architectural details"):
 *   - Sliding Window Attention paragraph and Figure 1 caption: the hidden state
 *     at position i attends to the previous layer's states at positions between
 *     i - W and i, at most W of them.  Read as: key position j is visible to
 *     query position i iff  i - W < j <= i.
 *   - Grouped-query attention (section 1): groups of query heads share one
 *     key/value head.  Read as contiguous groups: query head h uses kv head
 *     h / (Hq / Hkv)  (the grouping of the GQA paper the text cites).
 *   - The attention itself is the plain definition
 *         s_j   = scale * <q_i, k_j>                      for visible j
 *         o_i   = sum_j exp(s_j - max_j s_j) v_j / sum_j exp(s_j - max_j s_j)
 *     evaluated in float64 with no tiling, blocking or reordering.
 *
 * Every key carries its absolute position; a key with a negative position is
 * an empty cache slot and is never visible.  The caller (oracle/__init__.py)
 * decides which keys exist - the rolling cache and the chunk - so this file
 * holds only the visibility rule and the softmax-weighted sum.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC swa_oracle.c -o liboracle.so -lm
 * (no -ffast-math: IEEE float64 throughout).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Visibility of key position j to query position i with window W
 * (Mistral 7B, section 2, Sliding Window Attention and Figure 1). */
static int swa_visible(int64_t i, int64_t j, int64_t W)
{
    return j >= 0 && j <= i && j > i - W;
}

/*
 * Attention of n_q query rows against n_k keys.
 *   q     [n_q][Hq][d]    float64      q_pos [n_q]   absolute positions
 *   k, v  [n_k][Hkv][d]   float64      k_pos [n_k]   absolute positions (<0: empty)
 *   out   [n_q][Hq][d]    float64 (written)
 * Returns the number of (row, head) pairs that saw no key (written as zeros).
 */
int64_t swa_oracle_attend(int64_t n_q, const double *q, const int64_t *q_pos,
                          int64_t n_k, const double *k, const double *v,
                          const int64_t *k_pos, int Hq, int Hkv, int d, int64_t W,
                          double scale, double *out, int n_threads)
{
    const int G = Hq / Hkv;
    const int64_t n_tasks = n_q * (int64_t)Hq;
    int64_t empty = 0;
#ifdef _OPENMP
    if (n_threads <= 0)
        n_threads = omp_get_max_threads();
#else
    (void)n_threads;
#endif

#pragma omp parallel num_threads(n_threads) reduction(+ : empty)
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(n_k > 0 ? n_k : 1));
#pragma omp for schedule(dynamic, 4)
        for (int64_t task = 0; task < n_tasks; ++task) {
            const int64_t r = task / Hq;
            const int h = (int)(task % Hq);
            const int g = h / G;
            const int64_t i = q_pos[r];
            const double *qv = q + (r * Hq + h) * (int64_t)d;
            double *o = out + (r * Hq + h) * (int64_t)d;

            /* scores of visible keys and their maximum */
            double m = -INFINITY;
            int64_t n_vis = 0;
            for (int64_t j = 0; j < n_k; ++j) {
                if (!swa_visible(i, k_pos[j], W))
                    continue;
                const double *kv = k + (j * Hkv + g) * (int64_t)d;
                double dot = 0.0;
                for (int c = 0; c < d; ++c)
                    dot += qv[c] * kv[c];
                s[j] = scale * dot;
                if (s[j] > m)
                    m = s[j];
                ++n_vis;
            }
            for (int c = 0; c < d; ++c)
                o[c] = 0.0;
            if (n_vis == 0) {
                ++empty;
                continue;
            }
            /* softmax-weighted sum of the visible values */
            double l = 0.0;
            for (int64_t j = 0; j < n_k; ++j) {
                if (!swa_visible(i, k_pos[j], W))
                    continue;
                const double e = exp(s[j] - m);
                const double *vv = v + (j * Hkv + g) * (int64_t)d;
                l += e;
                for (int c = 0; c < d; ++c)
                    o[c] += e * vv[c];
            }
            for (int c = 0; c < d; ++c)
                o[c] /= l;
        }
        free(s);
    }
    return empty;
}

/* Thread count the OpenMP runtime would use by default (for reporting). */
int swa_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
