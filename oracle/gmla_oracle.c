/*
 * Gated MLA oracle: plain float64 CPU loops.  TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg load
 * this library.  It shares no code, header or constant with the CUDA path and
 * never calls it.  Every function is the plain definition of one step of the
 * method, with no blocking, fusion or reordering beyond the definition:
 *
 *   orc_linear     C = X W_c^T, Q = X W_q^T, K = C W_k^T, V = C W_v^T,
 *                  G = X W_g^T and the final (.) W_o^T -- the "XW^T" products
 *                  of the "Gated MLA" problem page, sections "Start from
 *                  familiar attention" and "The channel-wise output gate".
 *   orc_attention  per head A = softmax(Q K^T / sqrt(D_h) + M) and the head
 *                  context A V -- "Gated MLA", "Start from familiar
 *                  attention"; the mask M (0 for s <= t, -inf for s > t) of
 *                  "Kimi K2 - Construct causal mask"; the softmax over keys of
 *                  "Kimi K3 - Softmax over keys" (weights of visible keys sum
 *                  to one, blocked keys weigh exactly zero).
 *   orc_gate       sigmoid(G) (.) O -- "Gated MLA", "The channel-wise output
 *                  gate".
 *   orc_round_bf16 bfloat16 round-to-nearest-even of a float64, used only to
 *                  mirror the bfloat16 tensors stored at the library boundary.
 *
 * Softmax is evaluated as exp(S - m) / sum exp(S - m) with m the row maximum
 * over visible keys; this equals the page's exp(S) / sum exp(S) exactly in
 * real arithmetic and avoids overflow.
 *
 * Query row t of a call with Tq queries and Tk keys sits at absolute
 * position Tk - Tq + t (positions are numbered from the cached length, as in
 * "Kimi K2 - Construct causal mask", the position-id excerpt); in causal mode
 * it sees keys s <= Tk - Tq + t.
 *
 * orc_mutation (default 0) switches in deliberate mistakes so the tests can
 * show that the pins catch them; it is never set outside those tests.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int orc_mutation = 0;

enum {
    MUT_NONE = 0,
    MUT_MASK_AFTER_SOFTMAX = 1, /* normalise over all keys, then zero blocked ones */
    MUT_NO_SCALE = 2,           /* drop the 1/sqrt(D_h) factor */
    MUT_STRICT_CAUSAL = 3,      /* s < t instead of s <= t */
    MUT_KEY_OFF_BY_ONE = 4,     /* read key s+1 (wrapping) instead of key s */
};

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Y[m, n] = sum_k X[m, k] * W[n, k]   (X: [M, K] rows of stride ldx, W: [N, K]).
 * rows: optional list of nrows row indices m to compute (others untouched). */
void orc_linear(const double *X, long ldx, long M, long K, const double *W, long N,
                double *Y, long ldy, const long *rows, long nrows) {
    long cnt = rows ? nrows : M;
#pragma omp parallel for schedule(dynamic, 1)
    for (long r = 0; r < cnt; ++r) {
        long m = rows ? rows[r] : r;
        const double *x = X + m * ldx;
        double *y = Y + m * ldy;
        for (long n = 0; n < N; ++n) {
            const double *w = W + n * K;
            double acc = 0.0;
            for (long k = 0; k < K; ++k) acc += x[k] * w[k];
            y[n] = acc;
        }
    }
}

/* Attention for rows (b, h, t).  Element i of head h of token t of batch b of
 * tensor Z lives at Z[b*zs[0] + t*zs[1] + h*zs[2] + i].  W (optional) is
 * [B, H, Tq, Tk]; lse (optional) is [B, H, Tq] with lse = log sum_s exp(S_s).
 * rows: optional list of nrows (b, h, t) triples; NULL means every row. */
void orc_attention(const double *Q, const long *qs, const double *K, const long *ks,
                   const double *V, const long *vs, long B, long H, long Tq, long Tk, long D,
                   int causal, double scale, double *O, const long *os, double *W, double *lse,
                   const long *rows, long nrows) {
    long cnt = rows ? nrows : B * H * Tq;
#pragma omp parallel
    {
        double *S = (double *)malloc(sizeof(double) * (size_t)(Tk > 0 ? Tk : 1));
        char *vis = (char *)malloc((size_t)(Tk > 0 ? Tk : 1));
#pragma omp for schedule(dynamic, 4)
        for (long r = 0; r < cnt; ++r) {
            long b, h, t;
            if (rows) {
                b = rows[3 * r];
                h = rows[3 * r + 1];
                t = rows[3 * r + 2];
            } else {
                b = r / (H * Tq);
                h = (r / Tq) % H;
                t = r % Tq;
            }
            long pos = Tk - Tq + t; /* absolute position of this query */
            const double *q = Q + b * qs[0] + t * qs[1] + h * qs[2];
            double sc = (orc_mutation == MUT_NO_SCALE) ? 1.0 : scale;
            double m = -INFINITY;
            for (long s = 0; s < Tk; ++s) {
                int v = 1;
                if (causal) v = (orc_mutation == MUT_STRICT_CAUSAL) ? (s < pos) : (s <= pos);
                vis[s] = (char)v;
                long sk = (orc_mutation == MUT_KEY_OFF_BY_ONE) ? (s + 1) % Tk : s;
                const double *k = K + b * ks[0] + sk * ks[1] + h * ks[2];
                double dot = 0.0;
                for (long i = 0; i < D; ++i) dot += q[i] * k[i];
                S[s] = dot * sc;
                if ((v || orc_mutation == MUT_MASK_AFTER_SOFTMAX) && S[s] > m) m = S[s];
            }
            double sum = 0.0;
            for (long s = 0; s < Tk; ++s) {
                if (vis[s] || orc_mutation == MUT_MASK_AFTER_SOFTMAX) {
                    S[s] = exp(S[s] - m);
                    sum += S[s];
                } else {
                    S[s] = 0.0;
                }
            }
            for (long s = 0; s < Tk; ++s) {
                S[s] = S[s] / sum;
                if (!vis[s]) S[s] = 0.0; /* blocked keys weigh exactly zero */
            }
            double *o = O + b * os[0] + t * os[1] + h * os[2];
            for (long i = 0; i < D; ++i) o[i] = 0.0;
            for (long s = 0; s < Tk; ++s) {
                if (S[s] == 0.0) continue;
                const double *v = V + b * vs[0] + s * vs[1] + h * vs[2];
                for (long i = 0; i < D; ++i) o[i] += S[s] * v[i];
            }
            if (W) memcpy(W + ((b * H + h) * Tq + t) * Tk, S, sizeof(double) * (size_t)Tk);
            if (lse) lse[(b * H + h) * Tq + t] = m + log(sum);
        }
        free(S);
        free(vis);
    }
}

/* out[i] = sigmoid(G[i]) * O[i],  sigmoid(x) = 1 / (1 + exp(-x)). */
void orc_gate(const double *O, const double *G, long n, double *out) {
#pragma omp parallel for schedule(static)
    for (long i = 0; i < n; ++i) out[i] = O[i] * (1.0 / (1.0 + exp(-G[i])));
}

/* bfloat16 round-to-nearest-even of float64 values (finite inputs; values
 * beyond bfloat16's range become +-inf, NaN stays NaN). */
void orc_round_bf16(const double *x, long n, double *out) {
#pragma omp parallel for schedule(static)
    for (long i = 0; i < n; ++i) {
        double v = x[i];
        if (v == 0.0 || isnan(v) || isinf(v)) {
            out[i] = v;
            continue;
        }
        int e;
        double m = frexp(v, &e); /* v = m * 2^e, 0.5 <= |m| < 1 */
        if (e < -125) {          /* bfloat16 subnormal range: fixed quantum 2^-133 */
            out[i] = ldexp(nearbyint(ldexp(v, 133)), -133);
            continue;
        }
        double r = ldexp(nearbyint(ldexp(m, 8)), e - 8); /* 8 significant bits, ties to even */
        if (fabs(r) > 3.3895313892515355e38) r = v > 0 ? INFINITY : -INFINITY;
        out[i] = r;
    }
}
