/*
 * yoco.h -- C ABI of libyoco.so, the B200 (sm_100a) attention core of the
 * YOCO / YOCO++ decoder-decoder architecture.
 *
 * The method (sources by page title and section):
 *  - "You Only Cache Once: Decoder-Decoder Architectures for Language Models"
 *    (paperlayer summary of arXiv 2405.05254v2), section 2 "You Only Cache
 *    Once": a self-decoder produces one global KV cache that every
 *    cross-decoder layer reuses through cross-attention; section 3 "Design
 *    Choices of Self-Decoder", "Sliding-Window Attention": the self-decoder
 *    attends within a fixed window, so its cache is bounded.
 *  - "YOCO: Caching Once for Decoder-Decoder Long-Context Language Models"
 *    (podcast transcript), cue 12: the self-decoder output is normalised once
 *    and projected by one pair of matrices into the shared K and V; each
 *    cross-decoder layer has its own query projection and attends causally,
 *    with grouped-query heads; cue 26: every cross layer streams the whole
 *    shared KV at each decode step.
 *  - "YOCO++: Enhancing YOCO with KV Residual Connections for Efficient LLM
 *    Inference", Abstract: each bottom-half layer's KV gets a weighted
 *    residual connection to the bottom layer's KV.
 *
 * Conventions shared by every call
 *  - Layouts are token-major and dense: Q and O are [B, T, Hq, D], K and V
 *    are [B, T, Hkv, D] (or packed [rows, Hkv, D] for the shared decode
 *    cache).  Query head h reads KV head h / (Hq / Hkv).
 *  - Element type is cfg->dtype (bf16 or fp32) for every Q/K/V/O/x/W buffer;
 *    softmax and accumulation are fp32.  lse outputs are fp32, natural log.
 *  - Every pointer is a DEVICE pointer unless stated; the caller owns every
 *    buffer.  The library allocates no device memory; scratch comes from the
 *    caller's workspace argument.
 *  - Every data pointer must be 16-byte aligned.
 *  - Calls are asynchronous on the caller's stream and never synchronise the
 *    host.  Arguments are validated before anything is launched; on
 *    YOCO_ERR_INVALID / YOCO_ERR_UNSUPPORTED / YOCO_ERR_WORKSPACE nothing was
 *    launched and no buffer was touched.  YOCO_ERR_CUDA reports a launch
 *    error.  Device-side bounded waits that give up set a device status word
 *    that yoco_get_device_status() reports.
 *  - Masks: a query at absolute position p sees key position j when j <= p
 *    (causal, section 1 "Architecture": both halves use causal masking) and,
 *    for sliding-window calls, also j > p - window (the window counts the
 *    query's own position).
 */
#ifndef YOCO_H_
#define YOCO_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    YOCO_OK = 0,
    YOCO_ERR_INVALID = 1,      /* bad argument (null, misaligned, bad shape) */
    YOCO_ERR_UNSUPPORTED = 2,  /* valid but not built (head_dim, group size) */
    YOCO_ERR_CUDA = 3,         /* a CUDA launch or runtime call failed */
    YOCO_ERR_WORKSPACE = 4,    /* workspace missing or too small */
    YOCO_ERR_TIMEOUT = 5       /* a device-side bounded wait gave up */
} yoco_status;

typedef enum { YOCO_BF16 = 0, YOCO_FP32 = 1 } yoco_dtype;

/* Attention shape: Hq query heads, Hkv KV heads (Hq % Hkv == 0, group
 * Hq/Hkv in {1, 2, 4, 8}, Hkv <= 32), head dim D in {64, 128}.
 * scale 0 means 1/sqrt(D). */
typedef struct {
    int32_t Hq;
    int32_t Hkv;
    int32_t D;
    float scale;
    int32_t dtype; /* yoco_dtype */
} yoco_attn_cfg;

/* K/V producer with the YOCO++ weighted residual fused into its epilogue.
 * Podcast cue 12 (normalise once, project by one pair of matrices) and the
 * YOCO++ Abstract (KV of a bottom-half layer plus a weight times the bottom
 * layer's KV).
 *   [K | V] = N(x) . W_kv^T;  K += w_k * k_base;  V += w_v * v_base
 * x       [n_tok, d_model]
 * w_kv    [2*Hkv*D, d_model] row-major (one output feature per row; rows
 *         0 .. Hkv*D-1 produce K, the rest produce V)
 * apply_ln  nonzero: N = LayerNorm without affine (biased variance, ln_eps);
 *           zero: N = identity
 * k_base, v_base  [n_tok, Hkv, D] or NULL (no blend for that tensor)
 * dst_rows  NULL: token t is written to output row t.  Otherwise a device
 *           int64 [n_tok]: token t is written to row dst_rows[t] of k_out /
 *           v_out (appending to the shared cache); rows must be distinct and
 *           inside the caller's buffers.
 * k_out, v_out  [rows, Hkv, D]
 * With w = 0 (or NULL bases) this is the plain global-KV projection. */
yoco_status yoco_kv_project_blend(const void *x, int64_t n_tok, int32_t d_model,
                                  const void *w_kv, int32_t apply_ln, float ln_eps,
                                  const void *k_base, const void *v_base, float w_k, float w_v,
                                  const int64_t *dst_rows, void *k_out, void *v_out,
                                  const yoco_attn_cfg *cfg, cudaStream_t stream);

/* Self-decoder sliding-window attention over a prompt, then the ring fill.
 * Section 3 "Sliding-Window Attention".
 * q [B, T, Hq, D]; k, v [B, T, Hkv, D]; o [B, T, Hq, D]; lse [B, Hq, T] or NULL.
 * Query row i sees keys j with i - window < j <= i.
 * ring_k, ring_v [B, window, Hkv, D] and slot_pos int32 [B, window]: all three
 * NULL (no ring) or all set.  After the call slot s holds the newest position
 * p < T with p mod window == s, and slot_pos = p, or -1 (and zero K/V) when no
 * such position exists. */
yoco_status yoco_swa_prefill(const void *q, const void *k, const void *v, int32_t B, int64_t T,
                             int32_t window, void *o, float *lse, void *ring_k, void *ring_v,
                             int32_t *slot_pos, const yoco_attn_cfg *cfg, cudaStream_t stream);

/* Self-decoder sliding-window decode step over the ring.
 * q [B, Hq, D]; k_new, v_new [B, Hkv, D] (already blended); pos device int64
 * [B]: absolute position of the new token of each sequence.  The query
 * attends to the new token and to every other slot whose stored position lies
 * in (pos - window, pos] -- the window after the new K/V replaces slot
 * pos mod window -- and the new K/V is written there (slot_pos updated).
 * o [B, Hq, D].  workspace: yoco_swa_decode_workspace_size() bytes. */
yoco_status yoco_swa_decode(const void *q, const void *k_new, const void *v_new,
                            const int64_t *pos, int32_t B, int32_t window, void *ring_k,
                            void *ring_v, int32_t *slot_pos, void *o, void *workspace,
                            size_t ws_bytes, const yoco_attn_cfg *cfg, cudaStream_t stream);

/* One self-decoder decode step: yoco_kv_project_blend of the B new tokens
 * (n_tok = B, no dst_rows) followed by yoco_swa_decode with the projected
 * K/V -- the YOCO++ blended K/V producer (YOCO++ Abstract) and the section 3
 * "Sliding-Window Attention" decode -- with the same results.  Two launches;
 * for bf16 with B <= 4 and d_model a multiple of 256 the projection streams
 * its weights through registers and the window decode takes its compact
 * layout.
 * x [B, d_model]; w_kv [2 Hkv D, d_model]; k_base, v_base [B, Hkv, D] or
 * NULL (then w_k / w_v are ignored); q [B, Hq, D]; pos device int64 [B];
 * ring_k, ring_v [B, window, Hkv, D]; slot_pos int32 [B, window]; o [B, Hq, D].
 * k_out, v_out [B, Hkv, D] or NULL: receive the new tokens' blended K / V
 * (what yoco_kv_project_blend would write; a bottom layer's output is the
 * base of the layers above it); with NULL the workspace holds them.  The new
 * K/V is rounded to the cache dtype before it is attended to and stored.
 * workspace: yoco_swa_decode_step_workspace_size() bytes.
 * Errors (before any launch): YOCO_ERR_INVALID for B < 0, window < 1,
 * d_model < 1 or rows of d_model elements not a multiple of 16 bytes,
 * ln_eps <= 0, non-finite w_k / w_v, a null required pointer or any
 * pointer not 16-byte aligned; YOCO_ERR_UNSUPPORTED for a head shape no
 * decode is built for; YOCO_ERR_WORKSPACE for a null, misaligned or short
 * workspace.  B = 0 launches nothing and returns YOCO_OK. */
yoco_status yoco_swa_decode_step(const void *x, int32_t d_model, const void *w_kv, int32_t apply_ln,
                                 float ln_eps, const void *k_base, const void *v_base, float w_k, float w_v,
                                 const void *q, const int64_t *pos, int32_t B, int32_t window, void *ring_k,
                                 void *ring_v, int32_t *slot_pos, void *o, void *k_out, void *v_out,
                                 void *workspace, size_t ws_bytes, const yoco_attn_cfg *cfg,
                                 cudaStream_t stream);

/* Cross-decoder causal prefill over the one shared KV.  Section 2 and
 * podcast cue 12: every cross layer has its own Q and attends causally to the
 * same K_g, V_g.
 * q [B, Tq, Hq, D]; k, v [B, Tkv, Hkv, D]; o [B, Tq, Hq, D]; lse [B, Hq, Tq] or
 * NULL.  Query row i sits at absolute position q_pos0 + i (chunked prefill);
 * requires 0 <= q_pos0 and q_pos0 + Tq <= Tkv. */
yoco_status yoco_cross_prefill(const void *q, const void *k, const void *v, int32_t B,
                               int64_t Tq, int64_t Tkv, int64_t q_pos0, void *o, float *lse,
                               const yoco_attn_cfg *cfg, cudaStream_t stream);

/* Cross-decoder decode step: one new query token per sequence reads the whole
 * shared cache (podcast cue 26), split across the GPU and merged.
 * q [B, Hq, D]; k_cache, v_cache packed [cache_rows, Hkv, D] (both buffers
 * hold at least cache_rows rows, 1 <= cache_rows <= 2^31 - 1); sequence b
 * owns rows [seq_start[b], seq_start[b] + seq_len[b]) (device int64 / int32
 * arrays, seq_len including the new token's row).  max_len (host value) sizes
 * the split plan without a device read.
 * o [B, Hq, D]; lse [B, Hq] or NULL.
 * workspace: device scratch of yoco_cross_decode_workspace_size() bytes.
 * Device-side range check: a sequence with seq_len < 1, seq_len > max_len,
 * seq_start < 0 or seq_start + seq_len > cache_rows reads nothing; its o is 0
 * and its lse -inf, the other sequences are computed, and the next
 * yoco_get_device_status returns YOCO_ERR_INVALID.  No read ever leaves the
 * cache's cache_rows rows. */
yoco_status yoco_cross_decode(const void *q, const void *k_cache, const void *v_cache,
                              int64_t cache_rows, const int64_t *seq_start, const int32_t *seq_len,
                              int32_t B, int64_t max_len, void *o, float *lse, void *workspace,
                              size_t ws_bytes, const yoco_attn_cfg *cfg, cudaStream_t stream);

/* yoco_cross_decode for callers that cannot allocate device memory: a C host
 * or plugin that is handed only its input and output buffers, or a process
 * whose framework already holds nearly all device memory in its own pool.
 * The method's pages have no counterpart to this call; it exists for them.
 * Same arguments and result as yoco_cross_decode, without the workspace: the
 * split-KV scratch is a 32 MiB array inside the library, reserved on every
 * GPU that loads it until the process exits.  A decode whose plan needs more
 * (see yoco_cross_decode_workspace_size) returns YOCO_ERR_WORKSPACE and
 * launches nothing.  The first call on a device looks up the array's address
 * on that device (which must be current); make it before any stream capture.
 * The address is kept for the life of the process and does not survive a
 * cudaDeviceReset (or another teardown of the device's primary context) in
 * the same process: do not call this entry point after one.
 * All calls on a device share the array and leave their partials in it;
 * nothing needs clearing between calls, but calls whose kernels overlap on
 * the GPU race on it, so serialise them. */
yoco_status yoco_cross_decode_static(const void *q, const void *k_cache, const void *v_cache,
                                     int64_t cache_rows, const int64_t *seq_start,
                                     const int32_t *seq_len, int32_t B, int64_t max_len, void *o,
                                     float *lse, const yoco_attn_cfg *cfg, cudaStream_t stream);

/* General attention prefill over a key range that may start before the query
 * rows: query row i sits at position q_pos0 + i of the key buffer and sees
 * keys j <= q_pos0 + i, and j > q_pos0 + i - window when window > 0 (0:
 * causal).  It is the call of a chunk of a longer sequence: the
 * cross-decoder chunk over the gathered global K/V (window 0, q_pos0 = the
 * chunk's start), and the self-decoder chunk over its keys preceded by a halo
 * of the previous window - 1 keys ("You Only Cache Once", paperlayer summary,
 * Appendix A: the self-decoder only exchanges with neighbouring devices).
 * Layouts as yoco_cross_prefill; requires 0 <= q_pos0, q_pos0 + Tq <= Tkv,
 * window >= 0. */
yoco_status yoco_attention_prefill(const void *q, const void *k, const void *v, int32_t B, int64_t Tq,
                                   int64_t Tkv, int64_t q_pos0, int32_t window, void *o, float *lse,
                                   const yoco_attn_cfg *cfg, cudaStream_t stream);

/* Workspace bytes for yoco_cross_decode / yoco_swa_decode (0 on bad args). */
size_t yoco_cross_decode_workspace_size(int32_t B, int64_t max_len, const yoco_attn_cfg *cfg);
size_t yoco_swa_decode_workspace_size(int32_t B, int32_t window, const yoco_attn_cfg *cfg);
/* Workspace bytes for yoco_swa_decode_step (0 on bad args). */
size_t yoco_swa_decode_step_workspace_size(int32_t B, int32_t window, const yoco_attn_cfg *cfg);

/* Auxiliary dense projection used around the attention core (query and
 * output projections of the small end-to-end stack):
 *   out = N(x) . W^T + base_w * base
 * x [n, d_in]; w [d_out, d_in]; base [n, d_out] or NULL; out [n, d_out];
 * dtype is a yoco_dtype. */
yoco_status yoco_linear(const void *x, int64_t n, int32_t d_in, const void *w, int32_t d_out,
                        int32_t apply_ln, float ln_eps, const void *base, float base_w,
                        void *out, int32_t dtype, cudaStream_t stream);

/* 8-bit shared cache (podcast transcript, cue 1: the 65B example's "8-bit
 * cache quantization"; the scheme is not stated).  Reading: symmetric int8,
 * one fp32 scale per (token, KV head): scale = absmax / 127 over the head's D
 * values, code = round-half-even(x / scale) (fp32, IEEE division), value =
 * code * scale.  A cache row of an 8-bit K or V cache holds the token's
 * Hkv x D codes, then its Hkv scales, padded to a multiple of 16 bytes:
 * yoco_kv_i8_row_bytes(cfg) bytes (0 on bad arguments).
 *
 * yoco_kv_quantize_i8: k, v [n_tok, Hkv, D] (cfg->dtype) -> rows dst_rows[i]
 * (a device int64 array, or NULL for rows 0..n_tok-1) of k_i8 / v_i8.
 * Decode-time appends pass the new rows' indices, like yoco_kv_project_blend.
 *
 * yoco_cross_decode_i8: yoco_cross_decode over 8-bit caches (same q, o, lse,
 * cache_rows, sequence and workspace arguments and the same device-side range
 * check; cache_rows counts 8-bit rows; the workspace size is
 * yoco_cross_decode_workspace_size with the bf16 cfg).  Built for D = 128
 * and bf16 q / o; other shapes return YOCO_ERR_UNSUPPORTED.  The scores are
 * integer products of the K codes with q held per query head as 15-bit
 * fixed point (a step of 1/16256 of the head's largest |q|, well below bf16's
 * own rounding of q); everything else is the attention over the dequantised
 * values. */
int64_t yoco_kv_i8_row_bytes(const yoco_attn_cfg *cfg);
yoco_status yoco_kv_quantize_i8(const void *k, const void *v, int64_t n_tok, const int64_t *dst_rows, void *k_i8,
                                void *v_i8, const yoco_attn_cfg *cfg, cudaStream_t stream);
yoco_status yoco_cross_decode_i8(const void *q, const void *k_i8, const void *v_i8, int64_t cache_rows,
                                 const int64_t *seq_start, const int32_t *seq_len, int32_t B, int64_t max_len,
                                 void *o, float *lse, void *workspace, size_t ws_bytes, const yoco_attn_cfg *cfg,
                                 cudaStream_t stream);

/* Gated retention, the alternative self-decoder ("You Only Cache Once",
 * paperlayer summary, section 3 "Gated Retention" and Appendix B; podcast
 * transcript cue 16).  Per head h, with a D x D fp32 state S:
 *   gamma_t = sigmoid(g_t)^(1/tau),  S_t = gamma_t S_{t-1} + scale k_t^T v_t,
 *   o_t = q_t S_t,
 * scale = cfg->scale (0: 1/sqrt(D)).  Query and key/value heads are the same
 * heads: cfg->Hq == cfg->Hkv == H.
 *
 * yoco_gret_prefill: chunkwise over a prompt.  q, k, v, o [B, T, H, D] (bf16;
 * fp32 returns YOCO_ERR_UNSUPPORTED); g [B, T, H] fp32 gate logits; tau > 0.
 * state [B, H, D, D] fp32, S[d][e] multiplying q_d into o_e: the initial state
 * on entry and the final state on return, or NULL to start from zero and
 * drop the final state.  Caller-owned device memory; asynchronous on stream.
 * workspace: NULL, or device scratch of yoco_gret_prefill_workspace_size()
 * bytes (a smaller non-zero ws_bytes is YOCO_ERR_WORKSPACE).  With it, when
 * B x H sequences leave SMs idle (D = 128), each sequence's chunks are cut
 * into up to 8 superchunks on separate CTAs: a first pass forms every
 * superchunk's state contribution from a zero start and its total decay, and
 * each superchunk then starts from the decayed sum of those before it (the
 * same recurrence, regrouped).  The size query returns 0 when no split
 * applies. */
size_t yoco_gret_prefill_workspace_size(int32_t B, int64_t T, const yoco_attn_cfg *cfg);
yoco_status yoco_gret_prefill(const void *q, const void *k, const void *v, const float *g, int32_t B,
                              int64_t T, float tau, float *state, void *o, void *workspace, size_t ws_bytes,
                              const yoco_attn_cfg *cfg, cudaStream_t stream);

/* yoco_gret_decode: one recurrent step.  q, k, v, o [B, H, D] (bf16 or fp32);
 * g [B, H] fp32; state [B, H, D, D] fp32, read and updated in place
 * (required). */
yoco_status yoco_gret_decode(const void *q, const void *k, const void *v, const float *g, int32_t B,
                             float tau, float *state, void *o, const yoco_attn_cfg *cfg, cudaStream_t stream);

/* Test-only, with no counterpart on the pages: the work plan the kernels
 * follow, computed on the host by the kernels' own schedule functions, so
 * that tests can check it against the visibility rule pair by pair.  Reads
 * and writes host memory only; launches nothing.
 *
 * kind YOCO_SCHEDULE_PREFILL -- the bf16 tensor-core prefill of
 * yoco_cross_prefill / yoco_swa_prefill for B, Tq, Tkv, q_pos0 (query row i at
 * absolute position q_pos0 + i; q_pos0 + Tq <= Tkv) and window (0: causal).
 * A work tile is one 128-row query tile of one query head, or of two heads
 * (2hp, 2hp + 1) when Hq / Hkv is even.  One record per (query head, KV tile)
 * visit, CTA by CTA, each CTA's visits in the order it makes them:
 *   {cta, b, query head, query tile (128 rows), KV tile (128 keys), masked}
 * where masked = 1 when the tile runs the per-element mask.
 *
 * kind YOCO_SCHEDULE_DECODE -- the split-KV plan of yoco_cross_decode for
 * B sequences with HOST arrays seq_start [B] and seq_len [B], and max_len.
 * A sequence out of range (seq_len < 1, seq_len > max_len or seq_start < 0;
 * the cache size is not an argument here) has no units, as in the kernels.
 * One record per unit, CTA by CTA, in processing order:
 *   {cta, b, split index, first cache row, tokens, pipeline stages}
 *
 * n_cta: the persistent grid's size, 0 = the current device's SM count.
 * records: int64 [cap, 6] on the host (may be NULL when cap = 0); at most
 * cap records are written and *n_records receives the full count. */
enum { YOCO_SCHEDULE_PREFILL = 0, YOCO_SCHEDULE_DECODE = 1 };
yoco_status yoco_debug_tile_schedule(int32_t kind, const yoco_attn_cfg *cfg, int32_t B, int64_t Tq,
                                     int64_t Tkv, int64_t q_pos0, int32_t window,
                                     const int64_t *seq_start, const int32_t *seq_len, int64_t max_len,
                                     int32_t n_cta, int64_t *records, int64_t cap,
                                     int64_t *n_records);

/* KV-cache bytes of one sequence of N tokens (section 2: O(N + C L) for YOCO
 * versus N x L for a Transformer): one global K/V of N rows plus, per
 * self-decoder layer, a ring of min(window, N) rows.  Host only. */
double yoco_cache_bytes(int32_t L_self, int32_t window, int64_t N, const yoco_attn_cfg *cfg);

/* Synchronises the stream, then returns and clears the device status word:
 * YOCO_ERR_TIMEOUT if a kernel's bounded wait gave up since the last call,
 * else YOCO_ERR_INVALID if a decode call met a sequence out of range (see
 * yoco_cross_decode), else YOCO_ERR_CUDA if the stream reports an error,
 * else YOCO_OK. */
yoco_status yoco_get_device_status(cudaStream_t stream);

/* Test-only, with no counterpart on the pages: launches one kernel that waits,
 * through the same bounded mbarrier wait as the library's kernels, on a phase
 * that nothing completes.  The wait gives up after its limit (about 0.1 s),
 * the status word records it, and the next yoco_get_device_status returns
 * YOCO_ERR_TIMEOUT; nothing faults and the context stays usable.  Until the
 * status is read, the library's kernels exit at once (their first check). */
yoco_status yoco_debug_wait_timeout_probe(cudaStream_t stream);

/* Test-only, with no counterpart on the pages: y[i] = the polynomial 2^x[i]
 * that the bf16 prefill kernels evaluate on the FMA pipe for a quarter of
 * their softmax exponentials (Cody-Waite reduction, degree-3 minimax fit on
 * [-1/2, 1/2], relative error <= 7.5e-5; inputs below -125, -inf included,
 * give 2^-125 in place of 0).  x, y: device fp32 [n].  Asynchronous. */
yoco_status yoco_debug_exp2_poly(const float *x, float *y, int64_t n, cudaStream_t stream);

/* Static description of a status code. */
const char *yoco_status_string(yoco_status s);

/* Number of kernels this library has launched in this process (host-side
 * counter, incremented at every launch on every stream). */
uint64_t yoco_launch_count(void);

/* Library version string. */
const char *yoco_version(void);

#ifdef __cplusplus
}
#endif

#endif /* YOCO_H_ */
