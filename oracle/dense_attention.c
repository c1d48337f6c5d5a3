/*
 * Dense (contiguous, unpaged) fp64 attention in plain C.
 *
 * TEST INFRASTRUCTURE ONLY: this file pins the NumPy oracle on tiny inputs.
 * It knows nothing about blocks or tables; the tests lay a sequence's keys
 * out contiguously, give the NumPy oracle an identity block table over the
 * same memory, and require both to agree.  The result is
 *     out = sum_j w_j v_j,  w_j = exp(s*(q.k_j) - M) / sum_i exp(s*(q.k_i) - M)
 * where M is the largest logit (subtracting it leaves w unchanged).
 *
 * Build: gcc -O2 -shared -fPIC dense_attention.c -o libdense_attention.so -lm
 */
#include <math.h>

/* One query over L contiguous keys/values of width D.  L == 0 gives zeros. */
void dense_attention(const double *q, const double *K, const double *V, int L, int D,
                     double scale, double *out)
{
    int i, d;
    double M = -INFINITY, denom = 0.0;
    for (d = 0; d < D; ++d) out[d] = 0.0;
    if (L <= 0) return;
    for (i = 0; i < L; ++i) {
        double x = 0.0;
        for (d = 0; d < D; ++d) x += q[d] * K[(long)i * D + d];
        x *= scale;
        if (x > M) M = x;
    }
    for (i = 0; i < L; ++i) {
        double x = 0.0, w;
        for (d = 0; d < D; ++d) x += q[d] * K[(long)i * D + d];
        w = exp(x * scale - M);
        denom += w;
        for (d = 0; d < D; ++d) out[d] += w * V[(long)i * D + d];
    }
    for (d = 0; d < D; ++d) out[d] /= denom;
}

/* Causal chunk: n queries at positions L-n .. L-1 of an L-key sequence;
 * query i sees keys 0 .. L-n+i.  q is [n, D], out is [n, D]. */
void dense_causal_chunk(const double *q, const double *K, const double *V, int L, int n, int D,
                        double scale, double *out)
{
    int i;
    for (i = 0; i < n; ++i)
        dense_attention(q + (long)i * D, K, V, L - n + i + 1, D, scale, out + (long)i * D);
}
