/*
 * Plain CPU fp64 oracle for the YOCO / YOCO++ attention core.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, import or
 * call this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library; every function is written from the definitions on the
 * method's pages and is deliberately slow and direct (two-pass softmax per
 * query row, no tiling, no online rescaling, no fusion).
 *
 * Sources (page title, section):
 *  - "You Only Cache Once: Decoder-Decoder Architectures for Language Models"
 *    (paperlayer summary of arXiv 2405.05254v2), section 2 "You Only Cache
 *    Once": the self-decoder produces one global KV that every cross-decoder
 *    layer reuses; section 3 "Design Choices of Self-Decoder", bullet
 *    "Sliding-Window Attention": each query sees only a fixed window;
 *    section 1 "Introduction", bullet "Architecture": both halves are causal.
 *  - "YOCO: Caching Once for Decoder-Decoder Long-Context Language Models"
 *    (podcast transcript), cue 12: the self-decoder output is normalised once
 *    and projected by one pair of matrices into the shared keys and values;
 *    each cross-decoder layer keeps its own query projection, attends causally
 *    to that pair, with grouped-query heads.  Cue 26: every cross-decoder
 *    layer reads the whole shared KV at each decode step.
 *  - "YOCO++: Enhancing YOCO with KV Residual Connections for Efficient LLM
 *    Inference", Abstract: a weighted residual connection between the KVs of
 *    each bottom-half layer and the bottom layer.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - normalisation is LayerNorm without affine, biased variance, eps given;
 *  - softmax scale is a parameter (1/sqrt(D) by default at the call site);
 *  - a window of W keys includes the query's own position: j in (p-W, p];
 *  - GQA maps query head h to KV head floor(h / (Hq/Hkv));
 *  - the ring slot of position p is p mod W, an empty slot holds -1.
 *
 * All arrays are dense, row-major, fp64 (int64/int32 for indices).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* LayerNorm of each row of x[n, d]: (x - mean) / sqrt(var + eps), biased
 * variance, no scale or shift.  Podcast cue 12: "normalized input". */
void oracle_layernorm(const double *x, int64_t n, int64_t d, double eps, double *out) {
    for (int64_t r = 0; r < n; ++r) {
        const double *row = x + r * d;
        double mean = 0.0;
        for (int64_t c = 0; c < d; ++c) mean += row[c];
        mean /= (double)d;
        double var = 0.0;
        for (int64_t c = 0; c < d; ++c) var += (row[c] - mean) * (row[c] - mean);
        var /= (double)d;
        double inv = 1.0 / sqrt(var + eps);
        for (int64_t c = 0; c < d; ++c) out[r * d + c] = (row[c] - mean) * inv;
    }
}

/* Projection: out[n, m] = N(x)[n, d] . W^T where W is [m, d] (one output
 * feature per row) and N is LayerNorm when apply_ln != 0, identity otherwise.
 * Podcast cue 12: normalised once, projected by a pair of matrices. */
void oracle_project(const double *x, int64_t n, int64_t d, const double *w, int64_t m,
                    int apply_ln, double eps, double *out) {
    double *h = (double *)malloc(sizeof(double) * (size_t)(n * d));
    if (!h) return;
    if (apply_ln) oracle_layernorm(x, n, d, eps, h);
    else memcpy(h, x, sizeof(double) * (size_t)(n * d));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n; ++r) {
        for (int64_t c = 0; c < m; ++c) {
            double acc = 0.0;
            for (int64_t i = 0; i < d; ++i) acc += h[r * d + i] * w[c * d + i];
            out[r * m + c] = acc;
        }
    }
    free(h);
}

/* YOCO++ weighted residual: out = a + w * base, elementwise.  YOCO++
 * Abstract: each bottom-half layer's KV plus a weighted copy of the bottom
 * layer's KV. */
void oracle_blend(const double *a, const double *base, int64_t count, double w, double *out) {
    for (int64_t i = 0; i < count; ++i) out[i] = a[i] + w * base[i];
}

/* Is key position j visible to a query at absolute position p?
 * Causal (section 1, "Both components use causal masking"): j <= p.
 * Sliding window (section 3): additionally j > p - window when window > 0. */
static int visible(int64_t j, int64_t p, int64_t window) {
    if (j > p) return 0;
    if (window > 0 && j <= p - window) return 0;
    return 1;
}

/* The visibility matrix itself: out[i * Tkv + j] = 1 when key j is visible to
 * query row i (absolute position q_pos0 + i), by the rule above.  Used to
 * check the kernels' tile plans, not by the attention functions below. */
void oracle_visibility(int64_t Tq, int64_t Tkv, int64_t q_pos0, int64_t window, unsigned char *out) {
    for (int64_t i = 0; i < Tq; ++i)
        for (int64_t j = 0; j < Tkv; ++j) out[i * Tkv + j] = (unsigned char)visible(j, q_pos0 + i, window);
}

/* Softmax attention of one query vector over n_keys candidate key rows.
 * key(t) / val(t) are rows at (base + t * stride); mask[t] != 0 if visible.
 * Two passes: max of the visible scores, then exp-sum and weighted sum.
 * Writes o[D] and the natural-log sum of exp of the scaled scores. */
static void attend_one(const double *qv, int64_t D, double scale,
                       const double *kbase, const double *vbase, int64_t stride,
                       const unsigned char *mask, int64_t n_keys,
                       double *o, double *lse_out) {
    double mx = -INFINITY;
    for (int64_t t = 0; t < n_keys; ++t) {
        if (!mask[t]) continue;
        const double *kr = kbase + t * stride;
        double s = 0.0;
        for (int64_t c = 0; c < D; ++c) s += qv[c] * kr[c];
        s *= scale;
        if (s > mx) mx = s;
    }
    for (int64_t c = 0; c < D; ++c) o[c] = 0.0;
    double den = 0.0;
    for (int64_t t = 0; t < n_keys; ++t) {
        if (!mask[t]) continue;
        const double *kr = kbase + t * stride;
        const double *vr = vbase + t * stride;
        double s = 0.0;
        for (int64_t c = 0; c < D; ++c) s += qv[c] * kr[c];
        s *= scale;
        double p = exp(s - mx);
        den += p;
        for (int64_t c = 0; c < D; ++c) o[c] += p * vr[c];
    }
    if (den > 0.0) {
        for (int64_t c = 0; c < D; ++c) o[c] /= den;
        if (lse_out) *lse_out = mx + log(den);
    } else {
        if (lse_out) *lse_out = -INFINITY;
    }
}

/* Causal / sliding-window GQA attention for a list of query rows.
 * q [B, Tq, Hq, D]; k, v [B, Tkv, Hkv, D].  Query row i of batch b sits at
 * absolute position q_pos0 + i and sees key j (0 <= j < Tkv) when visible().
 * window <= 0 means plain causal.  Query head h reads KV head h / (Hq/Hkv).
 * rows_b / rows_i select n_rows query rows (NULL => all B*Tq rows in order).
 * o [n_rows, Hq, D]; lse [n_rows, Hq] (may be NULL). */
void oracle_attention_rows(const double *q, const double *k, const double *v,
                           int64_t B, int64_t Tq, int64_t Tkv, int64_t Hq, int64_t Hkv,
                           int64_t D, int64_t q_pos0, int64_t window, double scale,
                           const int64_t *rows_b, const int64_t *rows_i, int64_t n_rows,
                           double *o, double *lse) {
    const int64_t G = Hq / Hkv;
    if (!rows_b) n_rows = B * Tq;
#pragma omp parallel
    {
        unsigned char *mask = (unsigned char *)malloc((size_t)(Tkv > 0 ? Tkv : 1));
#pragma omp for schedule(dynamic, 1) collapse(2)
        for (int64_t r = 0; r < n_rows; ++r) {
            for (int64_t h = 0; h < Hq; ++h) {
                int64_t b = rows_b ? rows_b[r] : r / Tq;
                int64_t i = rows_b ? rows_i[r] : r % Tq;
                int64_t p = q_pos0 + i;
                for (int64_t j = 0; j < Tkv; ++j) mask[j] = (unsigned char)visible(j, p, window);
                int64_t g = h / G;
                const double *qv = q + ((b * Tq + i) * Hq + h) * D;
                const double *kb = k + ((b * Tkv) * Hkv + g) * D;
                const double *vb = v + ((b * Tkv) * Hkv + g) * D;
                attend_one(qv, D, scale, kb, vb, Hkv * D, mask, Tkv,
                           o + (r * Hq + h) * D, lse ? lse + r * Hq + h : NULL);
            }
        }
        free(mask);
    }
}

/* Full-tensor form of oracle_attention_rows: o [B, Tq, Hq, D], lse [B, Tq, Hq]. */
void oracle_attention(const double *q, const double *k, const double *v,
                      int64_t B, int64_t Tq, int64_t Tkv, int64_t Hq, int64_t Hkv, int64_t D,
                      int64_t q_pos0, int64_t window, double scale, double *o, double *lse) {
    oracle_attention_rows(q, k, v, B, Tq, Tkv, Hq, Hkv, D, q_pos0, window, scale,
                          NULL, NULL, 0, o, lse);
}

/* Cross-decoder decode step over a packed shared cache (podcast cue 26:
 * each cross layer reads the whole shared KV).  Sequence b occupies cache
 * rows [seq_start[b], seq_start[b] + seq_len[b]) and its query (one token,
 * the newest position) sees all of them.
 * q [B, Hq, D]; k_cache, v_cache [rows, Hkv, D]; o [B, Hq, D]; lse [B, Hq]. */
void oracle_cross_decode(const double *q, const double *k_cache, const double *v_cache,
                         const int64_t *seq_start, const int64_t *seq_len, int64_t B,
                         int64_t Hq, int64_t Hkv, int64_t D, double scale,
                         double *o, double *lse) {
    const int64_t G = Hq / Hkv;
#pragma omp parallel for schedule(dynamic, 1) collapse(2)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t h = 0; h < Hq; ++h) {
            int64_t n = seq_len[b];
            unsigned char *mask = (unsigned char *)malloc((size_t)(n > 0 ? n : 1));
            memset(mask, 1, (size_t)(n > 0 ? n : 1));
            int64_t g = h / G;
            const double *kb = k_cache + (seq_start[b] * Hkv + g) * D;
            const double *vb = v_cache + (seq_start[b] * Hkv + g) * D;
            attend_one(q + (b * Hq + h) * D, D, scale, kb, vb, Hkv * D, mask, n,
                       o + (b * Hq + h) * D, lse ? lse + b * Hq + h : NULL);
            free(mask);
        }
    }
}

/* Ring-buffer slot positions after a prefill of T tokens with window W:
 * the cache keeps only the last min(T, W) positions (section 2: the
 * self-decoder cache is bounded by the window); position p lives in slot
 * p mod W; slots never written hold -1.  Written as the literal sequence of
 * pushes, one position at a time. slot_pos [W]. */
void oracle_ring_prefill_slots(int64_t T, int64_t W, int32_t *slot_pos) {
    for (int64_t s = 0; s < W; ++s) slot_pos[s] = -1;
    for (int64_t p = 0; p < T; ++p) slot_pos[p % W] = (int32_t)p;
}

/* One decode push into a ring: the new token at absolute position pos
 * overwrites slot pos mod W.  ring_k/ring_v [W, Hkv, D], k_new/v_new
 * [Hkv, D], slot_pos [W]. */
void oracle_ring_push(double *ring_k, double *ring_v, int32_t *slot_pos, int64_t W,
                      int64_t Hkv, int64_t D, int64_t pos,
                      const double *k_new, const double *v_new) {
    int64_t s = pos % W;
    memcpy(ring_k + s * Hkv * D, k_new, sizeof(double) * (size_t)(Hkv * D));
    memcpy(ring_v + s * Hkv * D, v_new, sizeof(double) * (size_t)(Hkv * D));
    slot_pos[s] = (int32_t)pos;
}

/* Sliding-window decode read from a ring: the query at absolute position
 * pos attends to every slot whose stored position is in (pos - W, pos].
 * q [Hq, D]; ring_k/ring_v [W, Hkv, D]; o [Hq, D]. */
void oracle_swa_decode_ring(const double *q, const double *ring_k, const double *ring_v,
                            const int32_t *slot_pos, int64_t W, int64_t Hq, int64_t Hkv,
                            int64_t D, int64_t pos, double scale, double *o, double *lse) {
    const int64_t G = Hq / Hkv;
    unsigned char *mask = (unsigned char *)malloc((size_t)W);
    for (int64_t s = 0; s < W; ++s)
        mask[s] = (unsigned char)(slot_pos[s] >= 0 && visible(slot_pos[s], pos, W));
    for (int64_t h = 0; h < Hq; ++h) {
        int64_t g = h / G;
        attend_one(q + h * D, D, scale, ring_k + g * D, ring_v + g * D, Hkv * D, mask, W,
                   o + h * D, lse ? lse + h : NULL);
    }
    free(mask);
}

/* Cache accounting (section 2): a Transformer keeps N x L keys and values,
 * YOCO keeps one global N-row KV plus a constant-size cache per
 * self-decoder layer (C = window rows each).  Bytes for one sequence. */
double oracle_cache_bytes_yoco(int64_t L_self, int64_t window, int64_t N, int64_t Hkv,
                               int64_t D, int64_t elem_bytes) {
    double per_row = 2.0 * (double)Hkv * (double)D * (double)elem_bytes;
    int64_t c = window < N ? window : N;
    return per_row * ((double)N + (double)L_self * (double)c);
}

double oracle_cache_bytes_transformer(int64_t L, int64_t N, int64_t Hkv, int64_t D,
                                      int64_t elem_bytes) {
    return 2.0 * (double)Hkv * (double)D * (double)elem_bytes * (double)N * (double)L;
}

/* ---------------------------------------------------------------------------
 * Gated retention, the alternative self-decoder ("You Only Cache Once",
 * paperlayer summary, section 3 "Design Choices of Self-Decoder", bullets
 * "Gated Retention", and Appendix B "Chunk-wise Representation of Gated
 * Retention"; podcast transcript cue 16).  The pages state the mechanism in
 * words: retention (no softmax) with a data-dependent, head-wise scalar decay
 * gate, sigmoid of the input raised to one over a temperature; a d x d state
 * per head for decoding; a parallel, a recurrent and a chunkwise form that
 * give the same result.  Written out (the readings are in the design notes):
 *
 *   gamma_t = sigmoid(g_t)^(1/tau)                    (g: gate logits)
 *   S_t     = gamma_t S_{t-1} + scale * k_t^T v_t     (S: D x D, S_{-1} given)
 *   o_t     = q_t S_t
 *
 * Layouts: q, k, v [B, T, H, D]; log_gamma [B, T, H]; state [B, H, D, D]
 * with S[d][e] multiplying q_d into o_e. */

/* log gamma = log(sigmoid(g)) / tau, without overflow for large |g|. */
void oracle_gret_log_decay(const double *g, int64_t n, double tau, double *out) {
    for (int64_t i = 0; i < n; ++i) {
        double x = g[i];
        double ls = x >= 0.0 ? -log1p(exp(-x)) : x - log1p(exp(x));
        out[i] = ls / tau;
    }
}

/* Recurrent form: one token at a time through the state.  state: [B,H,D,D]
 * initial state on entry and final state on return; NULL starts from zero
 * and discards the final state. */
void oracle_gret_recurrent(const double *q, const double *k, const double *v,
                           const double *log_gamma, int64_t B, int64_t T, int64_t H, int64_t D,
                           double scale, double *state, double *o) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            double *S = (double *)calloc((size_t)(D * D), sizeof(double));
            if (state) memcpy(S, state + (b * H + h) * D * D, sizeof(double) * (size_t)(D * D));
            for (int64_t t = 0; t < T; ++t) {
                const int64_t row = (b * T + t) * H + h;
                const double gam = exp(log_gamma[row]);
                const double *kt = k + row * D, *vt = v + row * D, *qt = q + row * D;
                for (int64_t d = 0; d < D; ++d)
                    for (int64_t e = 0; e < D; ++e) S[d * D + e] = gam * S[d * D + e] + scale * kt[d] * vt[e];
                for (int64_t e = 0; e < D; ++e) {
                    double acc = 0.0;
                    for (int64_t d = 0; d < D; ++d) acc += qt[d] * S[d * D + e];
                    o[row * D + e] = acc;
                }
            }
            if (state) memcpy(state + (b * H + h) * D * D, S, sizeof(double) * (size_t)(D * D));
            free(S);
        }
    }
}

/* Parallel form: o_t = sum_{s <= t} (prod_{i=s+1..t} gamma_i) scale (q_t . k_s) v_s
 *                    + (prod_{i=0..t} gamma_i) q_t S_init.
 * The products are exp of differences of the running sum of log gamma.
 * state0: [B,H,D,D] initial state or NULL (zero). */
void oracle_gret_parallel(const double *q, const double *k, const double *v,
                          const double *log_gamma, int64_t B, int64_t T, int64_t H, int64_t D,
                          double scale, const double *state0, double *o) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            double *c = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
            double run = 0.0;
            for (int64_t t = 0; t < T; ++t) {
                run += log_gamma[(b * T + t) * H + h];
                c[t] = run;
            }
            for (int64_t t = 0; t < T; ++t) {
                const int64_t rt = (b * T + t) * H + h;
                const double *qt = q + rt * D;
                double *ot = o + rt * D;
                for (int64_t e = 0; e < D; ++e) ot[e] = 0.0;
                for (int64_t s = 0; s <= t; ++s) {
                    const int64_t rs = (b * T + s) * H + h;
                    double dot = 0.0;
                    for (int64_t d = 0; d < D; ++d) dot += qt[d] * k[rs * D + d];
                    const double w = exp(c[t] - c[s]) * scale * dot;
                    for (int64_t e = 0; e < D; ++e) ot[e] += w * v[rs * D + e];
                }
                if (state0) {
                    const double *S = state0 + (b * H + h) * D * D;
                    const double f = exp(c[t]);
                    for (int64_t e = 0; e < D; ++e) {
                        double acc = 0.0;
                        for (int64_t d = 0; d < D; ++d) acc += qt[d] * S[d * D + e];
                        ot[e] += f * acc;
                    }
                }
            }
            free(c);
        }
    }
}

/* Chunkwise form (Appendix B): chunks of C tokens; inside a chunk the
 * parallel form over the chunk's own tokens (the inner-chunk part) plus the
 * state carried in from the chunks before, decayed to each row (the
 * cross-chunk part); at the chunk's end the state is decayed over the whole
 * chunk and the chunk's keys and values are added with their decay to the
 * chunk's end.  state: as in the recurrent form. */
void oracle_gret_chunkwise(const double *q, const double *k, const double *v,
                           const double *log_gamma, int64_t B, int64_t T, int64_t H, int64_t D,
                           double scale, int64_t C, double *state, double *o) {
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t h = 0; h < H; ++h) {
            double *S = (double *)calloc((size_t)(D * D), sizeof(double));
            double *a = (double *)malloc(sizeof(double) * (size_t)(C > 0 ? C : 1));
            if (state) memcpy(S, state + (b * H + h) * D * D, sizeof(double) * (size_t)(D * D));
            for (int64_t j0 = 0; j0 < T; j0 += C) {
                const int64_t len = (T - j0) < C ? (T - j0) : C;
                double run = 0.0;  /* a[r] = sum of log gamma over the chunk's rows 0..r */
                for (int64_t r = 0; r < len; ++r) {
                    run += log_gamma[(b * T + j0 + r) * H + h];
                    a[r] = run;
                }
                for (int64_t r = 0; r < len; ++r) {
                    const int64_t rt = (b * T + j0 + r) * H + h;
                    const double *qt = q + rt * D;
                    double *ot = o + rt * D;
                    /* cross-chunk part: the carried state, decayed to row r */
                    const double f = exp(a[r]);
                    for (int64_t e = 0; e < D; ++e) {
                        double acc = 0.0;
                        for (int64_t d = 0; d < D; ++d) acc += qt[d] * S[d * D + e];
                        ot[e] = f * acc;
                    }
                    /* inner-chunk part */
                    for (int64_t u = 0; u <= r; ++u) {
                        const int64_t ru = (b * T + j0 + u) * H + h;
                        double dot = 0.0;
                        for (int64_t d = 0; d < D; ++d) dot += qt[d] * k[ru * D + d];
                        const double w = exp(a[r] - a[u]) * scale * dot;
                        for (int64_t e = 0; e < D; ++e) ot[e] += w * v[ru * D + e];
                    }
                }
                /* state to the chunk's end */
                const double fe = exp(a[len - 1]);
                for (int64_t i = 0; i < D * D; ++i) S[i] *= fe;
                for (int64_t u = 0; u < len; ++u) {
                    const int64_t ru = (b * T + j0 + u) * H + h;
                    const double w = exp(a[len - 1] - a[u]) * scale;
                    for (int64_t d = 0; d < D; ++d)
                        for (int64_t e = 0; e < D; ++e) S[d * D + e] += w * k[ru * D + d] * v[ru * D + e];
                }
            }
            if (state) memcpy(state + (b * H + h) * D * D, S, sizeof(double) * (size_t)(D * D));
            free(a);
            free(S);
        }
    }
}
