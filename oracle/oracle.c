/*
 * CPU oracle for block-sparse causal attention forward.  TEST INFRASTRUCTURE
 * ONLY: the tests, the package's smoke check and the bench's CPU-baseline leg
 * may load it; the product path never does.  It shares no code, header or
 * constant with the CUDA path.
 *
 * Everything here is the plain definition, written for a reader to check by
 * eye against the pages:
 *
 *  - oracle_allowed: the mask predicate.  "Sparse Attention" glossary page
 *    (ultralytics.com/de/glossary/sparse-attention), section "Ein Muster in
 *    Einsparungen verwandeln", the local_plus_sinks example: a pair is allowed
 *    when it is causal and either inside the window (q - kv <= window,
 *    inclusive) or its key is one of the first `sinks` tokens.  The strided
 *    and global-token variants follow the same page's section "Gängige
 *    Sparsity-Muster" (every s-th prior token; global tokens attend to and are
 *    attended by every position) and the "Sparse-трансформеры" page
 *    (1gpt.online), section "Основные шаблоны разреженности".  Readings taken
 *    where the pages leave a choice: the stride is relative ((q - kv) mod s ==
 *    0); causality is applied to the global rows and columns too, unless
 *    `global_rows_see_all` selects the other reading.
 *    Without causality (causal = 0) the window is two-sided, |q - kv| <= window
 *    (the sliding window of "Основные шаблоны разреженности": w neighbours on
 *    the left and on the right), and `area` > 0 admits the pairs of one stripe
 *    of `area` consecutive tokens (the Area Attention of the "Sparse Attention"
 *    glossary page, section "Anwendungen": a 40 x 40 feature map cut into four
 *    stripes of 400 tokens, attention only inside each stripe).  With `area`
 *    and `summary` > 0 this is the "fixed" pattern of "Основные шаблоны
 *    разреженности": blocks with local attention inside, linked through
 *    dedicated summary positions, read here as the last `summary` positions
 *    of every block, which every (causally later) query may attend to.
 *
 *  - oracle_block_mask: brute force.  For every (q-tile, kv-tile) pair count
 *    the allowed (q, kv) pairs one by one; zero means empty, all of them means
 *    full, anything else partial ("Ein Muster in Einsparungen verwandeln":
 *    the block mask records which 128 x 128 blocks hold no allowed pair).
 *
 *  - oracle_attention: per query, the explicit allowed key set, then the
 *    softmax of the scaled scores over that set, in fp64.  This is the
 *    masked_attention prototype of the "Sparse-трансформеры" page, section
 *    "Как это выглядит в коде" (scores q.k / sqrt(d), -inf outside the mask,
 *    softmax, times V), evaluated row by row over only the allowed keys, which
 *    gives the same numbers without materialising the masked matrix.
 *    LSE is the natural log of the sum of exp(scaled score) over the set.
 *
 *  - oracle_count_pairs: the number of allowed pairs, one by one.
 *
 *  - oracle_attention_bwd: the gradients of that same function (the
 *    masked_attention prototype of "Как это выглядит в коде") with respect to
 *    Q, K and V for an upstream gradient dO.  The pages print no backward
 *    pass; this is the chain rule through the softmax over each query's
 *    allowed set, written out term by term (see the function's comment).
 *
 * Inputs are bf16 bit patterns, widened exactly to double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int32_t causal;              /* 1: every allowed pair has q >= kv */
    int32_t window;              /* >= 0: pairs with 0 <= q - kv <= window; < 0: no band */
    int32_t sinks;               /* keys kv < sinks */
    int32_t stride;              /* > 0: pairs with (q - kv) mod stride == 0 */
    int32_t n_global;            /* keys kv < n_global and queries q < n_global */
    int32_t global_rows_see_all; /* 1: rows q < n_global ignore causality (alternative reading) */
    int32_t area;                /* > 0: pairs in the same stripe, floor(q / area) == floor(kv / area) */
    int32_t summary;             /* with area > 0: keys in the last `summary` positions of any stripe */
} oracle_pattern;

int oracle_allowed(const oracle_pattern *p, int64_t q, int64_t kv)
{
    int64_t delta = q - kv;
    int64_t dist = delta < 0 ? -delta : delta;
    if (p->global_rows_see_all && q < p->n_global)
        return 1;
    if (p->causal && delta < 0)
        return 0;
    if (!p->causal && p->stride > 0)
        return -1; /* a stride without causality is not defined here */
    if (p->window >= 0 && dist <= p->window)
        return 1;
    if (kv < p->sinks)
        return 1;
    if (p->stride > 0 && delta % p->stride == 0)
        return 1;
    if (kv < p->n_global || q < p->n_global)
        return 1;
    if (p->area > 0 && q / p->area == kv / p->area)
        return 1;
    if (p->area > 0 && p->summary > 0 && kv % p->area >= p->area - p->summary)
        return 1;
    return 0;
}

/* Allowed keys of each listed query row, 0 <= kv < N, counted one by one. */
int oracle_row_counts(const oracle_pattern *p, int64_t N, const int64_t *rows, int64_t n_rows, int64_t *out)
{
    for (int64_t r = 0; r < n_rows; r++)
        if (rows[r] < 0 || rows[r] >= N)
            return -1;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t r = 0; r < n_rows; r++) {
        int64_t c = 0;
        for (int64_t kv = 0; kv < N; kv++)
            c += oracle_allowed(p, rows[r], kv) == 1;
        out[r] = c;
    }
    return 0;
}

/* Number of allowed (q, kv) pairs with 0 <= q, kv < N, counted one by one. */
int64_t oracle_count_pairs(const oracle_pattern *p, int64_t N)
{
    int64_t total = 0;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : total)
    for (int64_t q = 0; q < N; q++) {
        int64_t c = 0;
        for (int64_t kv = 0; kv < N; kv++)
            c += oracle_allowed(p, q, kv) == 1;
        total += c;
    }
    return total;
}

/*
 * Brute-force tile classifier.  T = ceil(N / block) tiles per side; the last
 * tile is ragged when block does not divide N and only its in-range pairs
 * count.  Outputs, each T*T long and row-major by q-tile:
 *   index[i*T + c]  c-th non-empty kv tile of q-tile i, ascending; -1 after the last
 *   full[i*T + c]   1 when every in-range pair of that tile is allowed, else 0; 0 after the last
 *   counts[i]       number of non-empty kv tiles of q-tile i
 * Returns the total number of non-empty tiles, or -1 on a bad argument.
 */
int64_t oracle_block_mask(const oracle_pattern *p, int64_t N, int32_t block,
                          int32_t *counts, int32_t *index, uint8_t *full)
{
    if (N < 0 || block <= 0)
        return -1;
    int64_t T = (N + block - 1) / block;
    int64_t live = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : live)
    for (int64_t i = 0; i < T; i++) {
        int64_t q0 = i * block, q1 = q0 + block < N ? q0 + block : N;
        int32_t c = 0;
        for (int64_t j = 0; j < T; j++) {
            int64_t k0 = j * block, k1 = k0 + block < N ? k0 + block : N;
            int64_t allowed = 0;
            for (int64_t q = q0; q < q1; q++)
                for (int64_t kv = k0; kv < k1; kv++)
                    allowed += oracle_allowed(p, q, kv) == 1;
            if (allowed == 0)
                continue;
            index[i * T + c] = (int32_t)j;
            full[i * T + c] = allowed == (q1 - q0) * (k1 - k0);
            c++;
        }
        counts[i] = c;
        for (int64_t t = c; t < T; t++) {
            index[i * T + t] = -1;
            full[i * T + t] = 0;
        }
        live += c;
    }
    return live;
}

static double bf16_to_double(uint16_t h)
{
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/*
 * Attention forward by definition.  Layouts (contiguous):
 *   Q [B, Hq, N, D], K and V [B, Hkv, N, D]   bf16 bit patterns
 *   rows[n_rows]   the query positions to evaluate (NULL: all N, n_rows = N)
 *   O   [B, Hq, n_rows, D]  double
 *   LSE [B, Hq, n_rows]     double; -inf and O = 0 for a query with no allowed key
 * Query head hq reads key/value head hq / (Hq / Hkv).
 * Returns 0, or -1 on a bad argument.
 */
int oracle_attention(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                     int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t D,
                     const oracle_pattern *p, double scale,
                     const int64_t *rows, int64_t n_rows,
                     double *O, double *LSE, int32_t n_threads)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || N < 0 || D <= 0)
        return -1;
    if (rows == NULL)
        n_rows = N;
    int64_t group = Hq / Hkv;
#ifdef _OPENMP
    if (n_threads > 0)
        omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif

#pragma omp parallel
    {
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)(N > 0 ? N : 1));
        double *s = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        double *qrow = (double *)malloc(sizeof(double) * (size_t)D);
        double *acc = (double *)malloc(sizeof(double) * (size_t)D);

#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < n_rows; r++) {
            int64_t q = rows ? rows[r] : r;
            /* the allowed key set of this query; the pattern does not depend on (b, h) */
            int64_t n_keys = 0;
            for (int64_t kv = 0; kv < N; kv++)
                if (oracle_allowed(p, q, kv) == 1)
                    keys[n_keys++] = kv;

            for (int64_t b = 0; b < B; b++) {
                for (int64_t hq = 0; hq < Hq; hq++) {
                    int64_t hkv = hq / group;
                    const uint16_t *qp = Q + ((b * Hq + hq) * N + q) * D;
                    const uint16_t *kb = K + (b * Hkv + hkv) * N * D;
                    const uint16_t *vb = V + (b * Hkv + hkv) * N * D;
                    double *o = O + ((b * Hq + hq) * n_rows + r) * D;
                    double *lse = LSE + (b * Hq + hq) * n_rows + r;

                    if (n_keys == 0) {
                        for (int64_t c = 0; c < D; c++)
                            o[c] = 0.0;
                        *lse = -INFINITY;
                        continue;
                    }
                    for (int64_t c = 0; c < D; c++)
                        qrow[c] = bf16_to_double(qp[c]);

                    /* scores over the allowed set */
                    double m = -INFINITY;
                    for (int64_t t = 0; t < n_keys; t++) {
                        const uint16_t *kp = kb + keys[t] * D;
                        double dot = 0.0;
                        for (int64_t c = 0; c < D; c++)
                            dot += qrow[c] * bf16_to_double(kp[c]);
                        s[t] = scale * dot;
                        if (s[t] > m)
                            m = s[t];
                    }
                    /* softmax weights and the weighted sum of values */
                    double l = 0.0;
                    for (int64_t c = 0; c < D; c++)
                        acc[c] = 0.0;
                    for (int64_t t = 0; t < n_keys; t++) {
                        double w = exp(s[t] - m);
                        l += w;
                        const uint16_t *vp = vb + keys[t] * D;
                        for (int64_t c = 0; c < D; c++)
                            acc[c] += w * bf16_to_double(vp[c]);
                    }
                    for (int64_t c = 0; c < D; c++)
                        o[c] = acc[c] / l;
                    *lse = m + log(l);
                }
            }
        }
        free(keys);
        free(s);
        free(qrow);
        free(acc);
    }
    return 0;
}

/*
 * Backward of attention by definition.  Inputs are doubles (callers widen bf16
 * exactly), contiguous:
 *   Q, dO [B, Hq, N, D];  K, V [B, Hkv, N, D]
 * Outputs (contiguous, double):
 *   O [B, Hq, N, D], LSE [B, Hq, N]   the forward pass, as oracle_attention
 *   dQ [B, Hq, N, D], dK, dV [B, Hkv, N, D]
 *
 * For query q of head hq, A(q) its allowed key set, s_kv = scale Q_q.K_kv and
 * P_kv = exp(s_kv - LSE_q) the softmax weights over A(q) (zero outside), the
 * output is O_q = sum_kv P_kv V_kv, and for a scalar loss with dL/dO = dO:
 *   dP_kv = dO_q . V_kv                      (gradient of the weights)
 *   Delta_q = sum_kv P_kv dP_kv              (the softmax Jacobian's row term)
 *   dS_kv = P_kv (dP_kv - Delta_q)           (gradient of the scores)
 *   dQ_q  = scale sum_kv dS_kv K_kv
 *   dK_kv = scale sum_(hq in group, q) dS_kv Q_q
 *   dV_kv = sum_(hq in group, q) P_kv dO_q
 * A query with no allowed key has O = 0, LSE = -inf and contributes nothing.
 * Pass 1 walks query rows (O, LSE, Delta, dQ); pass 2 walks key rows and sums
 * over every query that may attend to it (dK, dV).  Returns 0, or -1 on a bad
 * argument.
 */
int oracle_attention_bwd(const double *Q, const double *K, const double *V, const double *dO,
                         int64_t B, int64_t Hq, int64_t Hkv, int64_t N, int64_t D,
                         const oracle_pattern *p, double scale,
                         double *O, double *LSE, double *dQ, double *dK, double *dV, int32_t n_threads)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || N < 0 || D <= 0)
        return -1;
    int64_t group = Hq / Hkv;
    double *delta = (double *)malloc(sizeof(double) * (size_t)(B * Hq * N > 0 ? B * Hq * N : 1));
    if (!delta)
        return -1;
#ifdef _OPENMP
    if (n_threads > 0)
        omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif

    /* pass 1: per query row */
#pragma omp parallel
    {
        int64_t *keys = (int64_t *)malloc(sizeof(int64_t) * (size_t)(N > 0 ? N : 1));
        double *s = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        double *dp = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));

#pragma omp for schedule(dynamic, 4)
        for (int64_t row = 0; row < B * Hq * N; row++) {
            int64_t q = row % N, bh = row / N, b = bh / Hq, hq = bh % Hq, hkv = hq / group;
            const double *qv = Q + row * D, *dov = dO + row * D;
            const double *kb = K + (b * Hkv + hkv) * N * D, *vb = V + (b * Hkv + hkv) * N * D;
            double *o = O + row * D, *dq = dQ + row * D;
            int64_t n_keys = 0;
            for (int64_t kv = 0; kv < N; kv++)
                if (oracle_allowed(p, q, kv) == 1)
                    keys[n_keys++] = kv;
            for (int64_t c = 0; c < D; c++) {
                o[c] = 0.0;
                dq[c] = 0.0;
            }
            if (n_keys == 0) {
                LSE[row] = -INFINITY;
                delta[row] = 0.0;
                continue;
            }
            double m = -INFINITY;
            for (int64_t t = 0; t < n_keys; t++) {
                double dot = 0.0;
                for (int64_t c = 0; c < D; c++)
                    dot += qv[c] * kb[keys[t] * D + c];
                s[t] = scale * dot;
                if (s[t] > m)
                    m = s[t];
            }
            double l = 0.0;
            for (int64_t t = 0; t < n_keys; t++)
                l += exp(s[t] - m);
            double lse = m + log(l);
            LSE[row] = lse;
            double dl = 0.0;
            for (int64_t t = 0; t < n_keys; t++) {
                double pw = exp(s[t] - lse);
                double d = 0.0;
                for (int64_t c = 0; c < D; c++) {
                    o[c] += pw * vb[keys[t] * D + c];
                    d += dov[c] * vb[keys[t] * D + c];
                }
                dp[t] = d;
                dl += pw * d;
            }
            delta[row] = dl;
            for (int64_t t = 0; t < n_keys; t++) {
                double ds = exp(s[t] - lse) * (dp[t] - dl);
                for (int64_t c = 0; c < D; c++)
                    dq[c] += scale * ds * kb[keys[t] * D + c];
            }
        }
        free(keys);
        free(s);
        free(dp);
    }

    /* pass 2: per key row, over every query of the group that may attend to it */
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t row = 0; row < B * Hkv * N; row++) {
        int64_t kv = row % N, bh = row / N, b = bh / Hkv, hkv = bh % Hkv;
        const double *kv_k = K + row * D, *kv_v = V + row * D;
        double *dk = dK + row * D, *dv = dV + row * D;
        for (int64_t c = 0; c < D; c++) {
            dk[c] = 0.0;
            dv[c] = 0.0;
        }
        for (int64_t hq = hkv * group; hq < (hkv + 1) * group; hq++) {
            for (int64_t q = 0; q < N; q++) {
                if (oracle_allowed(p, q, kv) != 1)
                    continue;
                int64_t qrow = (b * Hq + hq) * N + q;
                const double *qv = Q + qrow * D, *dov = dO + qrow * D;
                double dot = 0.0, d = 0.0;
                for (int64_t c = 0; c < D; c++) {
                    dot += qv[c] * kv_k[c];
                    d += dov[c] * kv_v[c];
                }
                double pw = exp(scale * dot - LSE[qrow]);
                double ds = pw * (d - delta[qrow]);
                for (int64_t c = 0; c < D; c++) {
                    dv[c] += pw * dov[c];
                    dk[c] += scale * ds * qv[c];
                }
            }
        }
    }
    free(delta);
    return 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
