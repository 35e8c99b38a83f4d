/*
 * Triple-loop attention in long double, for tiny shapes only.
 *
 * TEST INFRASTRUCTURE ONLY: it pins the fp64 NumPy oracle (oracle/attn.py) with an
 * implementation that shares nothing with it (no BLAS, no NumPy, wider arithmetic).  The
 * CUDA library never links or calls it.
 *
 * Computes, for one (batch, head) slice, the plain definition of non-causal softmax
 * attention over the keys k0 <= j < k1 (the joint image+text attention of a DiT block; the
 * xDiT overview page, section 2.1, describes DiT inference as prefill-like with no KV
 * cache, so every query sees every key):
 *     x_ij  = scale * sum_d q[i][d] * k[j][d]
 *     m_i   = max_j x_ij
 *     out_i = sum_j exp(x_ij - m_i) v[j] / sum_j exp(x_ij - m_i)
 *     lse_i = m_i + log sum_j exp(x_ij - m_i)
 * An empty range gives out = 0 and lse = -inf.
 *
 * Layout: q [sq][d], k and v [skv][d], out [sq][d], lse [sq]; all row-major double.
 */
#include <math.h>

void brute_attention(const double *q, const double *k, const double *v, int sq, int skv,
                     int d, double scale, int k0, int k1, double *out, double *lse) {
    (void)skv;
    for (int i = 0; i < sq; ++i) {
        if (k1 <= k0) {
            for (int c = 0; c < d; ++c) out[(long)i * d + c] = 0.0;
            lse[i] = -INFINITY;
            continue;
        }
        long double m = -INFINITY;
        for (int j = k0; j < k1; ++j) {
            long double dot = 0.0L;
            for (int c = 0; c < d; ++c)
                dot += (long double)q[(long)i * d + c] * (long double)k[(long)j * d + c];
            long double x = (long double)scale * dot;
            if (x > m) m = x;
        }
        long double den = 0.0L;
        for (int c = 0; c < d; ++c) out[(long)i * d + c] = 0.0;
        long double acc[1024];
        for (int c = 0; c < d && c < 1024; ++c) acc[c] = 0.0L;
        for (int j = k0; j < k1; ++j) {
            long double dot = 0.0L;
            for (int c = 0; c < d; ++c)
                dot += (long double)q[(long)i * d + c] * (long double)k[(long)j * d + c];
            long double w = expl((long double)scale * dot - m);
            den += w;
            for (int c = 0; c < d && c < 1024; ++c) acc[c] += w * (long double)v[(long)j * d + c];
        }
        for (int c = 0; c < d && c < 1024; ++c) out[(long)i * d + c] = (double)(acc[c] / den);
        lse[i] = (double)(m + logl(den));
    }
}
