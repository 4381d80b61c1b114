/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the TokenGate pruned-prefill hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load
 * this file; only the tests, the package's smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or table with the CUDA library.
 *
 * Source: the MarkTechPost article "Researchers from Stanford and UC Berkeley
 * Introduce TokenGate: token-gated attention speeds up long-context prefill by up
 * to 11.3x" (October 2026), called "the TokenGate article" below.  The article
 * prints no formulas; where it is silent the plainest reading is taken and stated
 * beside the function.
 *
 * Every floating-point computation runs in double precision over the exact
 * values of the bf16 / fp32 inputs.  OpenMP parallelises only across independent
 * output rows; the arithmetic of each row is a plain sequential loop in the
 * order the definition is written.
 *
 * Parity pins (checked by tests/test_oracle_pins.py, independent of this file):
 *   gate       -- torch.nn.functional linear+silu in fp64, the numpy twin,
 *                 permutation / scaling / bias-shift invariants, W1 = 0 case.
 *   select     -- O(n^2) rank counting brute force, hand-worked fixtures,
 *                 |kept| = K + q, question always kept, ascending output.
 *   gather     -- numpy fancy indexing.
 *   attention  -- torch scaled_dot_product_attention in fp64 (GQA expanded,
 *                 additive key bias), row 0 = V[0], bias-shift invariance,
 *                 duplicated-KV-head equivalence, convex-hull bound,
 *                 pruned keys never influence an output.
 *   backward   -- torch autograd in fp64 through an independent softmax
 *                 attention, central finite differences of the forward above,
 *                 a hand-worked two-token fixture, sum_j ds_j = 0 (a constant
 *                 shift of every score leaves the softmax unchanged).
 *   lse        -- torch logsumexp in fp64.
 *   projections -- torch fp64 matmul (positions 0, no norm), a hand-worked
 *                 rotary fixture, relative-position invariance of q.k, norm
 *                 preservation, scale invariance of the per-head norm, and
 *                 pruning commuting with projection at original positions.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 -> double, exactly: a bf16 is the high half of an IEEE fp32. */
static double bf16_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ *
 * Gate MLP scorer.
 * TokenGate article, "How does TokenGate learned token pruning work?" (gate
 * module): an MLP scores every token from its post-attention residual at gate
 * layer L.  The article says only "small MLP"; the scorer taken here is
 * Linear(d -> h), SiLU, Linear(h -> 1):
 *     z_j = b1_j + sum_k W1[j,k] x_ik            (j < h)
 *     a_j = z_j * sigmoid(z_j),  sigmoid(z) = 1 / (1 + exp(-z))
 *     s_i = b2 + sum_j W2_j a_j
 * No normalisation precedes the gate and the score is not squashed.
 * hidden: bf16 [n, d] row-major; W1: bf16 [h, d] (row j = output unit j);
 * b1, W2: bf16 [h]; b2: bf16 [1]; s: double [n].
 * ------------------------------------------------------------------------ */
void orc_gate_score(const uint16_t *hidden, int64_t n, int32_t d,
                    const uint16_t *W1, const uint16_t *b1, const uint16_t *W2,
                    const uint16_t *b2, int32_t h, double *s)
{
    double *w1 = (double *)malloc(sizeof(double) * (size_t)h * (size_t)d);
    for (int64_t t = 0; t < (int64_t)h * d; ++t) w1[t] = bf16_value(W1[t]);
    const double bias2 = bf16_value(b2[0]);

#pragma omp parallel
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(static)
        for (int64_t i = 0; i < n; ++i) {
            const uint16_t *row = hidden + (size_t)i * (size_t)d;
            for (int32_t k = 0; k < d; ++k) x[k] = bf16_value(row[k]);
            double out = 0.0;
            for (int32_t j = 0; j < h; ++j) {
                const double *wj = w1 + (size_t)j * (size_t)d;
                double z = bf16_value(b1[j]);
                for (int32_t k = 0; k < d; ++k) z += wj[k] * x[k];
                const double a = z / (1.0 + exp(-z));
                out += bf16_value(W2[j]) * a;
            }
            s[i] = out + bias2;
        }
        free(x);
    }
    free(w1);
}

/* ------------------------------------------------------------------------ *
 * Top-K selection with the question always kept.
 * TokenGate article, "How does TokenGate learned token pruning work?": a top-K
 * selector keeps the highest-scoring tokens; only the document part of the
 * prompt is prunable and the question is never pruned.
 * Readings where the article is silent:
 *   - ties go to the lower index; -0.0 and +0.0 compare equal (IEEE);
 *   - NaN ranks below every number (below -inf), ties among NaNs by index;
 *   - a budget above the document length keeps every document token.
 * The order is a strict total order on (score, index), so the kept set is
 * unique.  Output: kept indices in ascending order; returns their count.
 * ------------------------------------------------------------------------ */
typedef struct {
    float s;
    int32_t i;
} scored_index;

static int before(const scored_index *a, const scored_index *b)
{
    const int an = isnan(a->s), bn = isnan(b->s);
    if (an != bn) return bn;               /* the non-NaN one comes first */
    if (!an && a->s != b->s) return a->s > b->s;
    return a->i < b->i;
}

static int cmp_rank(const void *pa, const void *pb)
{
    const scored_index *a = (const scored_index *)pa, *b = (const scored_index *)pb;
    if (before(a, b)) return -1;
    if (before(b, a)) return 1;
    return 0;
}

int64_t orc_select_topk(const float *scores, const uint8_t *doc_mask, int64_t n,
                        int64_t k, int32_t *kept)
{
    int64_t n_doc = 0;
    for (int64_t i = 0; i < n; ++i) n_doc += doc_mask[i] != 0;
    scored_index *doc = (scored_index *)malloc(sizeof(scored_index) * (size_t)(n_doc > 0 ? n_doc : 1));
    int64_t t = 0;
    for (int64_t i = 0; i < n; ++i)
        if (doc_mask[i]) { doc[t].s = scores[i]; doc[t].i = (int32_t)i; ++t; }
    qsort(doc, (size_t)n_doc, sizeof(scored_index), cmp_rank);

    const int64_t take = k < 0 ? 0 : (k < n_doc ? k : n_doc);
    uint8_t *keep = (uint8_t *)calloc((size_t)(n > 0 ? n : 1), 1);
    for (int64_t r = 0; r < take; ++r) keep[doc[r].i] = 1;
    for (int64_t i = 0; i < n; ++i)
        if (!doc_mask[i]) keep[i] = 1;

    int64_t m = 0;
    for (int64_t i = 0; i < n; ++i)
        if (keep[i]) kept[m++] = (int32_t)i;
    free(keep);
    free(doc);
    return m;
}

/* ------------------------------------------------------------------------ *
 * Random-K selection (the random-selector ablation of the TokenGate article,
 * "How does TokenGate perform on benchmarks?").  Each document token draws a
 * random key from SplitMix64 (Steele, Lea and Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014) as a counter-based generator:
 * the value for position i is the (i + 1)-th output of the generator seeded with
 * ``seed``.  The k document tokens with the largest key >> 33 are kept (ties to
 * the lower index), every question token is kept, output ascending.
 * ------------------------------------------------------------------------ */
uint64_t orc_splitmix64(uint64_t seed, uint64_t index)
{
    uint64_t x = seed;
    /* advance the state index + 1 times by the golden gamma, then mix */
    x += (index + 1) * 0x9E3779B97F4A7C15ull;
    uint64_t z = x;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

typedef struct {
    uint64_t key;
    int32_t i;
} keyed_index;

static int cmp_key_desc(const void *pa, const void *pb)
{
    const keyed_index *a = (const keyed_index *)pa, *b = (const keyed_index *)pb;
    if (a->key != b->key) return a->key > b->key ? -1 : 1;
    return a->i < b->i ? -1 : (a->i > b->i);
}

int64_t orc_select_random_k(const uint8_t *doc_mask, int64_t n, int64_t k, uint64_t seed, int32_t *kept)
{
    int64_t n_doc = 0;
    for (int64_t i = 0; i < n; ++i) n_doc += doc_mask[i] != 0;
    keyed_index *doc = (keyed_index *)malloc(sizeof(keyed_index) * (size_t)(n_doc > 0 ? n_doc : 1));
    int64_t t = 0;
    for (int64_t i = 0; i < n; ++i)
        if (doc_mask[i]) {
            doc[t].key = orc_splitmix64(seed, (uint64_t)i) >> 33;
            doc[t].i = (int32_t)i;
            ++t;
        }
    qsort(doc, (size_t)n_doc, sizeof(keyed_index), cmp_key_desc);
    const int64_t take = k < 0 ? 0 : (k < n_doc ? k : n_doc);
    uint8_t *keep = (uint8_t *)calloc((size_t)(n > 0 ? n : 1), 1);
    for (int64_t r = 0; r < take; ++r) keep[doc[r].i] = 1;
    for (int64_t i = 0; i < n; ++i)
        if (!doc_mask[i]) keep[i] = 1;
    int64_t m = 0;
    for (int64_t i = 0; i < n; ++i)
        if (keep[i]) kept[m++] = (int32_t)i;
    free(keep);
    free(doc);
    return m;
}

/* ------------------------------------------------------------------------ *
 * Gather / compaction.
 * TokenGate article, "How does TokenGate learned token pruning work?" (pruned
 * forward): layers above L process only the kept tokens.
 *     hidden_k[r, :] = hidden[kept[r], :],   s_k[r] = scores[kept[r]]
 * ------------------------------------------------------------------------ */
void orc_gather(const uint16_t *hidden, int32_t d, const int32_t *kept, int64_t n_kept,
                uint16_t *hidden_k, const float *scores, float *s_k)
{
    for (int64_t r = 0; r < n_kept; ++r) {
        memcpy(hidden_k + (size_t)r * (size_t)d, hidden + (size_t)kept[r] * (size_t)d,
               sizeof(uint16_t) * (size_t)d);
        if (scores && s_k) s_k[r] = scores[kept[r]];
    }
}

/* ------------------------------------------------------------------------ *
 * Token-gated causal GQA attention over the kept tokens.
 * TokenGate article, "What is token-gated attention?": each kept token's score
 * becomes a bias on the attention logits of the layers above the gate, with a
 * learnable per-head gain and a learnable temperature.  The article prints no
 * formula; the one taken here:
 *     g      = h / (Hq / Hkv)                      (grouped KV head of q-head h)
 *     l_ij   = tau * (Q[i,h,:] . K[j,g,:]) / sqrt(D) + gain_h * s_j,   j <= i
 *     O[i,h] = sum_j softmax_j(l_i.) V[j,g,:]
 * Causality is in compacted order, which is the original order because the
 * kept indices are ascending.  Question keys carry their own score as bias.
 * Q: bf16 [S, Hq, D]; K, V: bf16 [S, Hkv, D]; s: fp32 [S]; gain: fp32 [Hq].
 * Only the rows listed in ``rows`` are computed (all rows for a full run);
 * O: double [n_rows, Hq, D].
 *
 * spread (NULL to skip): double [n_rows, Hq, D], the mean absolute deviation of
 * the value rows under the row's softmax weights,
 *     spread[i,h,c] = sum_j softmax_j(l_i.) |V[j,g,c] - O[i,h,c]|.
 * It is not part of the method: it measures how far a perturbation of the weights
 * can move the output (relative weight errors of at most e move O[i,h,c] by at
 * most about 2 e spread[i,h,c]), which the tests use to size their tolerance.
 * ------------------------------------------------------------------------ */
void orc_gated_attention_rows(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                              const float *s, const float *gain, double tau,
                              int64_t S, int32_t Hq, int32_t Hkv, int32_t D,
                              const int64_t *rows, int64_t n_rows, double *O, double *spread)
{
    const int32_t group = Hq / Hkv;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    (void)S;

#pragma omp parallel
    {
        double *q = NULL, *l = NULL;
        int64_t l_cap = 0;
        q = (double *)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < n_rows * Hq; ++t) {
            const int64_t r = t / Hq;
            const int32_t hh = (int32_t)(t % Hq);
            const int64_t i = rows[r];
            const int32_t g = hh / group;
            if (i + 1 > l_cap) {
                free(l);
                l_cap = i + 1;
                l = (double *)malloc(sizeof(double) * (size_t)l_cap);
            }
            for (int32_t c = 0; c < D; ++c) q[c] = bf16_value(Q[((size_t)i * Hq + hh) * D + c]);
            double m = -INFINITY;
            for (int64_t j = 0; j <= i; ++j) {
                const uint16_t *kj = K + ((size_t)j * Hkv + g) * D;
                double dot = 0.0;
                for (int32_t c = 0; c < D; ++c) dot += q[c] * bf16_value(kj[c]);
                l[j] = tau * dot * inv_sqrt_d + (double)gain[hh] * (double)s[j];
                if (l[j] > m) m = l[j];
            }
            double denom = 0.0;
            double *o = O + ((size_t)r * Hq + hh) * D;
            for (int32_t c = 0; c < D; ++c) o[c] = 0.0;
            for (int64_t j = 0; j <= i; ++j) {
                const double p = exp(l[j] - m);
                denom += p;
                const uint16_t *vj = V + ((size_t)j * Hkv + g) * D;
                for (int32_t c = 0; c < D; ++c) o[c] += p * bf16_value(vj[c]);
            }
            for (int32_t c = 0; c < D; ++c) o[c] /= denom;
            if (spread) {
                double *sp = spread + ((size_t)r * Hq + hh) * D;
                for (int32_t c = 0; c < D; ++c) sp[c] = 0.0;
                for (int64_t j = 0; j <= i; ++j) {
                    const double w = exp(l[j] - m) / denom;
                    const uint16_t *vj = V + ((size_t)j * Hkv + g) * D;
                    for (int32_t c = 0; c < D; ++c) sp[c] += w * fabs(bf16_value(vj[c]) - o[c]);
                }
            }
        }
        free(q);
        free(l);
    }
}

/* ------------------------------------------------------------------------ *
 * Log-sum-exp of each attention row (the normaliser of the softmax above):
 *     lse[r, h] = log sum_{j <= i} exp(l_ij),   i = rows[r]
 * with l_ij the token-gated logit defined above.  lse: double [n_rows, Hq].
 * ------------------------------------------------------------------------ */
void orc_gated_attention_lse_rows(const uint16_t *Q, const uint16_t *K, const float *s,
                                  const float *gain, double tau, int32_t Hq, int32_t Hkv,
                                  int32_t D, const int64_t *rows, int64_t n_rows, double *lse)
{
    const int32_t group = Hq / Hkv;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t t = 0; t < n_rows * Hq; ++t) {
        const int64_t r = t / Hq;
        const int32_t hh = (int32_t)(t % Hq);
        const int64_t i = rows[r];
        const int32_t g = hh / group;
        const uint16_t *qi = Q + ((size_t)i * Hq + hh) * D;
        double m = -INFINITY;
        for (int pass = 0; pass < 2; ++pass) {
            double sum = 0.0;
            for (int64_t j = 0; j <= i; ++j) {
                const uint16_t *kj = K + ((size_t)j * Hkv + g) * D;
                double dot = 0.0;
                for (int32_t c = 0; c < D; ++c) dot += bf16_value(qi[c]) * bf16_value(kj[c]);
                const double l = tau * dot * inv_sqrt_d + (double)gain[hh] * (double)s[j];
                if (pass == 0) {
                    if (l > m) m = l;
                } else {
                    sum += exp(l - m);
                }
            }
            if (pass == 1) lse[(size_t)r * Hq + hh] = m + log(sum);
        }
    }
}

/* ------------------------------------------------------------------------ *
 * Backward of token-gated attention with respect to the key scores, the per-head
 * gains and the temperature: the gradient path from the attention layers back to
 * the gate.  TokenGate article, "What is token-gated attention?": the gate score
 * enters every layer above L as a logit bias with a learnable per-head gain and a
 * learnable temperature, and the gate is trained through it.
 * For an upstream gradient dO of the output O defined above (loss L with
 * dL/dO = dO), per head h and query row i, with P_i. = softmax_j(l_i.), j <= i:
 *     dP_ij    = dO[i,h,:] . V[j,g,:]
 *     Delta_i  = sum_j P_ij dP_ij            (= dO_i . O_i)
 *     dl_ij    = P_ij (dP_ij - Delta_i)     (dL/dl_ij through the softmax)
 * and, since l_ij = tau (q_i . k_j)/sqrt(D) + gain_h s_j,
 *     ds_j    += gain_h dl_ij
 *     dgain_h += s_j dl_ij
 *     dtau    += dl_ij (q_i . k_j) / sqrt(D)
 * summed over every head h and row i.  dO: bf16 [S, Hq, D].  Outputs are double:
 * ds [S], dgain [Hq], dtau [1].  Heads run in parallel into per-head buffers that
 * are then added in head order.
 * ------------------------------------------------------------------------ */
void orc_gated_attention_backward(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                                  const float *s, const float *gain, double tau,
                                  const uint16_t *dO, int64_t S, int32_t Hq, int32_t Hkv,
                                  int32_t D, double *ds, double *dgain, double *dtau)
{
    const int32_t group = Hq / Hkv;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    double *ds_h = (double *)calloc((size_t)Hq * (size_t)(S > 0 ? S : 1), sizeof(double));
    double *dtau_h = (double *)calloc((size_t)Hq, sizeof(double));

#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t hh = 0; hh < Hq; ++hh) {
        const int32_t g = hh / group;
        double *dsh = ds_h + (size_t)hh * (size_t)S;
        double *l = (double *)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1));
        double *qk = (double *)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1));
        double *dp = (double *)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1));
        double dg = 0.0, dt = 0.0;
        for (int64_t i = 0; i < S; ++i) {
            const uint16_t *qi = Q + ((size_t)i * Hq + hh) * D;
            const uint16_t *doi = dO + ((size_t)i * Hq + hh) * D;
            double m = -INFINITY;
            for (int64_t j = 0; j <= i; ++j) {
                const uint16_t *kj = K + ((size_t)j * Hkv + g) * D;
                const uint16_t *vj = V + ((size_t)j * Hkv + g) * D;
                double dot = 0.0, dpv = 0.0;
                for (int32_t c = 0; c < D; ++c) {
                    dot += bf16_value(qi[c]) * bf16_value(kj[c]);
                    dpv += bf16_value(doi[c]) * bf16_value(vj[c]);
                }
                qk[j] = dot * inv_sqrt_d;
                dp[j] = dpv;
                l[j] = tau * qk[j] + (double)gain[hh] * (double)s[j];
                if (l[j] > m) m = l[j];
            }
            double denom = 0.0;
            for (int64_t j = 0; j <= i; ++j) {
                l[j] = exp(l[j] - m);  /* unnormalised weight */
                denom += l[j];
            }
            double delta = 0.0;
            for (int64_t j = 0; j <= i; ++j) {
                l[j] /= denom;         /* P_ij */
                delta += l[j] * dp[j];
            }
            for (int64_t j = 0; j <= i; ++j) {
                const double dl = l[j] * (dp[j] - delta);
                dsh[j] += (double)gain[hh] * dl;
                dg += (double)s[j] * dl;
                dt += dl * qk[j];
            }
        }
        dgain[hh] = dg;
        dtau_h[hh] = dt;
        free(l);
        free(qk);
        free(dp);
    }
    double t = 0.0;
    for (int32_t hh = 0; hh < Hq; ++hh) t += dtau_h[hh];
    *dtau = t;
    for (int64_t j = 0; j < S; ++j) {
        double a = 0.0;
        for (int32_t hh = 0; hh < Hq; ++hh) a += ds_h[(size_t)hh * (size_t)S + j];
        ds[j] = a;
    }
    free(ds_h);
    free(dtau_h);
}

/* ------------------------------------------------------------------------ *
 * Projections of a pruned layer (the layers above the gate).
 * TokenGate article, "How does TokenGate learned token pruning work?" (pruned
 * forward): the layers above L run on the kept tokens only, and those tokens
 * stay at their prompt positions.  The article names the Qwen3 backbones but no
 * layer formula; the plainest reading of a Qwen3 attention block is taken:
 *
 *   y      = W_qkv x_i                   W_qkv: bf16 [(Hq + 2 Hkv) D, d], rows =
 *                                        Q heads, then K heads, then V heads
 *   per Q / K head (optional, Qwen3 style, weight w of length D):
 *          u_c = y_c / sqrt(mean_c(y_c^2) + eps) * w_c
 *   rotary embedding of Q / K heads at position p_i, pairs (j, j + D/2):
 *          phi_j = p_i * base^(-2j / D)                 (j < D/2)
 *          out_j       = u_j cos phi_j - u_{j+D/2} sin phi_j
 *          out_{j+D/2} = u_{j+D/2} cos phi_j + u_j sin phi_j
 *   V heads are neither normalised nor rotated.
 *
 * hidden: bf16 [S, d]; positions: int32 [S] (the original token index of every
 * kept row); q_norm / k_norm: bf16 [D] or NULL (no normalisation).  Only the
 * listed rows are computed; Q: double [n_rows, Hq, D], K and V: double
 * [n_rows, Hkv, D].
 * ------------------------------------------------------------------------ */
static void rms_normalise(double *u, int32_t D, const uint16_t *w, double eps)
{
    double ss = 0.0;
    for (int32_t c = 0; c < D; ++c) ss += u[c] * u[c];
    const double r = 1.0 / sqrt(ss / (double)D + eps);
    for (int32_t c = 0; c < D; ++c) u[c] = u[c] * r * bf16_value(w[c]);
}

static void rotate(const double *u, int32_t D, int64_t pos, double base, double *out)
{
    const int32_t half = D / 2;
    for (int32_t j = 0; j < half; ++j) {
        const double phi = (double)pos * pow(base, -2.0 * (double)j / (double)D);
        const double c = cos(phi), s = sin(phi);
        out[j] = u[j] * c - u[j + half] * s;
        out[j + half] = u[j + half] * c + u[j] * s;
    }
}

void orc_qkv_rope_rows(const uint16_t *hidden, int32_t d, const uint16_t *W_qkv,
                       const int32_t *positions, double base, int32_t Hq, int32_t Hkv,
                       int32_t D, const uint16_t *q_norm, const uint16_t *k_norm, double eps,
                       const int64_t *rows, int64_t n_rows, double *Q, double *K, double *V)
{
    const int32_t n_out = (Hq + 2 * Hkv) * D;
#pragma omp parallel
    {
        double *y = (double *)malloc(sizeof(double) * (size_t)n_out);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            const int64_t i = rows[r];
            const uint16_t *x = hidden + (size_t)i * (size_t)d;
            for (int32_t o = 0; o < n_out; ++o) {
                const uint16_t *w = W_qkv + (size_t)o * (size_t)d;
                double acc = 0.0;
                for (int32_t k = 0; k < d; ++k) acc += bf16_value(w[k]) * bf16_value(x[k]);
                y[o] = acc;
            }
            for (int32_t hh = 0; hh < Hq + Hkv; ++hh) {
                double *u = y + (size_t)hh * D;
                const int is_q = hh < Hq;
                const uint16_t *nw = is_q ? q_norm : k_norm;
                if (nw) rms_normalise(u, D, nw, eps);
                double *dst = is_q ? Q + ((size_t)r * Hq + hh) * D
                                   : K + ((size_t)r * Hkv + (hh - Hq)) * D;
                rotate(u, D, positions[i], base, dst);
            }
            for (int32_t g = 0; g < Hkv; ++g)
                memcpy(V + ((size_t)r * Hkv + g) * D, y + (size_t)(Hq + Hkv + g) * D,
                       sizeof(double) * (size_t)D);
        }
        free(y);
    }
}

/* Output projection (o_proj) with an optional residual add:
 *     y_i = W x_i (+ residual_i)
 * x: bf16 [M, K]; W: bf16 [N, K] (nn.Linear layout); residual: bf16 [M, N] or
 * NULL.  Only the listed rows are computed; y: double [n_rows, N]. */
void orc_linear_rows(const uint16_t *x, int32_t K, const uint16_t *W, int32_t N,
                     const uint16_t *residual, const int64_t *rows, int64_t n_rows, double *y)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t i = rows[r];
        const uint16_t *xi = x + (size_t)i * (size_t)K;
        for (int32_t o = 0; o < N; ++o) {
            const uint16_t *w = W + (size_t)o * (size_t)K;
            double acc = 0.0;
            for (int32_t k = 0; k < K; ++k) acc += bf16_value(w[k]) * bf16_value(xi[k]);
            if (residual) acc += bf16_value(residual[(size_t)i * (size_t)N + o]);
            y[(size_t)r * N + o] = acc;
        }
    }
}

/* Thread count of the following parallel regions (timing on one core, for reporting);
 * n <= 0 leaves it unchanged.  Results do not depend on it. */
void orc_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Number of OpenMP threads the oracle runs with (for reporting). */
int orc_num_threads(void)
{
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            extern int omp_get_num_threads(void);
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
