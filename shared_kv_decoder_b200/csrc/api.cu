// C ABI of libyoco.so (declared in include/yoco.h): argument validation and
// dispatch to the sm_100a kernels.  Nothing is launched unless every check
// passes; the library never allocates device memory and never synchronises
// the host on a hot call.
#include <math.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "../../include/yoco.h"
#include "launch.h"
#include "schedule.h"

using namespace yoco;

namespace yoco {
static std::atomic<uint64_t> g_launches{0};
void note_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }
}  // namespace yoco

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void *p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void *p) { return p == nullptr || aligned16(p); }
// The decode kernels address cache rows with 32-bit TMA coordinates.
bool ok_cache_rows(int64_t rows) { return rows >= 1 && rows <= INT32_MAX; }

yoco_status check_cfg(const yoco_attn_cfg *cfg) {
    if (!cfg) return YOCO_ERR_INVALID;
    if (cfg->Hq < 1 || cfg->Hkv < 1 || cfg->Hq % cfg->Hkv != 0) return YOCO_ERR_INVALID;
    if (cfg->dtype != YOCO_BF16 && cfg->dtype != YOCO_FP32) return YOCO_ERR_INVALID;
    if (!(cfg->scale >= 0.f) || isinf(cfg->scale)) return YOCO_ERR_INVALID;
    if (cfg->D != 64 && cfg->D != 128) return YOCO_ERR_UNSUPPORTED;
    const int G = cfg->Hq / cfg->Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return YOCO_ERR_UNSUPPORTED;
    return YOCO_OK;
}

float eff_scale(const yoco_attn_cfg *cfg) {
    return cfg->scale > 0.f ? cfg->scale : 1.0f / sqrtf((float)cfg->D);
}

yoco_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return YOCO_OK;
    if (e == cudaErrorNotSupported) return YOCO_ERR_UNSUPPORTED;
    return YOCO_ERR_CUDA;
}

// Projection dispatch: the tensor-core kernel where it applies, else CUDA cores.
yoco_status run_linear(const LinearArgs &a, cudaStream_t s) {
    const cudaError_t e = launch_linear_tc(a, s);
    if (e != cudaErrorNotSupported) return from_cuda(e);
    cudaGetLastError();
    return from_cuda(launch_linear_simt(a, s));
}

// Attention prefill dispatch: bf16 goes to a tcgen05 kernel -- two query
// heads per CTA when the group size is even, else one; fp32 (and any bf16
// shape those kernels were not built for) to the CUDA-core kernel.
yoco_status run_prefill(const PrefillArgs &a, cudaStream_t s) {
    if (a.dtype == kBF16) {
        cudaError_t e = launch_prefill_pair(a, s);
        if (e != cudaErrorNotSupported) return from_cuda(e);
        cudaGetLastError();
        e = launch_prefill_tc(a, s);
        if (e != cudaErrorNotSupported) return from_cuda(e);
        cudaGetLastError();
    }
    return from_cuda(launch_prefill_simt(a, s));
}

}  // namespace

extern "C" {

const char *yoco_version(void) { return "yoco-b200 0.1 (sm_100a)"; }

uint64_t yoco_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *yoco_status_string(yoco_status s) {
    switch (s) {
        case YOCO_OK: return "ok";
        case YOCO_ERR_INVALID: return "invalid argument";
        case YOCO_ERR_UNSUPPORTED: return "unsupported shape or type";
        case YOCO_ERR_CUDA: return "CUDA error";
        case YOCO_ERR_WORKSPACE: return "workspace missing or too small";
        case YOCO_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

yoco_status yoco_kv_project_blend(const void *x, int64_t n_tok, int32_t d_model, const void *w_kv,
                                  int32_t apply_ln, float ln_eps, const void *k_base,
                                  const void *v_base, float w_k, float w_v,
                                  const int64_t *dst_rows, void *k_out, void *v_out,
                                  const yoco_attn_cfg *cfg, cudaStream_t stream) {
    yoco_status st = check_cfg(cfg);
    if (st != YOCO_OK) return st;
    if (n_tok < 0 || d_model < 1 || !(ln_eps > 0.f) || !isfinite(w_k) || !isfinite(w_v))
        return YOCO_ERR_INVALID;
    if (n_tok == 0) return YOCO_OK;
    if (!ok_ptr(x) || !ok_ptr(w_kv) || !ok_ptr(k_out) || !ok_ptr(v_out) || !ok_opt(k_base) ||
        !ok_opt(v_base) || !ok_opt(dst_rows))
        return YOCO_ERR_INVALID;
    if ((int64_t)d_model * dtype_bytes(cfg->dtype) % 16 != 0) return YOCO_ERR_INVALID;
    LinearArgs a;
    a.x = x; a.w = w_kv; a.n = n_tok; a.d_in = d_model;
    a.d_out = 2 * cfg->Hkv * cfg->D; a.split_col = cfg->Hkv * cfg->D;
    a.apply_ln = apply_ln ? 1 : 0; a.eps = ln_eps;
    a.out0 = k_out; a.out1 = v_out; a.base0 = k_base; a.base1 = v_base;
    a.w0 = w_k; a.w1 = w_v; a.dst_rows = dst_rows; a.dtype = cfg->dtype;
    return run_linear(a, stream);
}

yoco_status yoco_linear(const void *x, int64_t n, int32_t d_in, const void *w, int32_t d_out,
                        int32_t apply_ln, float ln_eps, const void *base, float base_w, void *out,
                        int32_t dtype, cudaStream_t stream) {
    if (dtype != YOCO_BF16 && dtype != YOCO_FP32) return YOCO_ERR_INVALID;
    if (n < 0 || d_in < 1 || d_out < 1 || !(ln_eps > 0.f) || !isfinite(base_w))
        return YOCO_ERR_INVALID;
    if (n == 0) return YOCO_OK;
    if (!ok_ptr(x) || !ok_ptr(w) || !ok_ptr(out) || !ok_opt(base)) return YOCO_ERR_INVALID;
    LinearArgs a;
    a.x = x; a.w = w; a.n = n; a.d_in = d_in; a.d_out = d_out; a.split_col = d_out;
    a.apply_ln = apply_ln ? 1 : 0; a.eps = ln_eps;
    a.out0 = out; a.out1 = nullptr; a.base0 = base; a.base1 = nullptr;
    a.w0 = base_w; a.w1 = 0.f; a.dst_rows = nullptr; a.dtype = dtype;
    return run_linear(a, stream);
}

yoco_status yoco_swa_prefill(const void *q, const void *k, const void *v, int32_t B, int64_t T,
                             int32_t window, void *o, float *lse, void *ring_k, void *ring_v,
                             int32_t *slot_pos, const yoco_attn_cfg *cfg, cudaStream_t stream) {
    yoco_status st = check_cfg(cfg);
    if (st != YOCO_OK) return st;
    if (B < 0 || T < 0 || window < 1) return YOCO_ERR_INVALID;
    const int rings = (ring_k != nullptr) + (ring_v != nullptr) + (slot_pos != nullptr);
    if (rings != 0 && rings != 3) return YOCO_ERR_INVALID;
    if (B == 0) return YOCO_OK;
    if (T > 0 && (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(o) || !ok_opt(lse)))
        return YOCO_ERR_INVALID;
    if (rings == 3 && (!ok_ptr(ring_k) || !ok_ptr(ring_v) || !ok_ptr(slot_pos)))
        return YOCO_ERR_INVALID;
    if (T > 0) {
        PrefillArgs a;
        a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
        a.B = B; a.Tq = T; a.Tkv = T; a.q_pos0 = 0; a.window = window;
        a.Hq = cfg->Hq; a.Hkv = cfg->Hkv; a.D = cfg->D; a.dtype = cfg->dtype;
        a.scale = eff_scale(cfg);
        st = run_prefill(a, stream);
        if (st != YOCO_OK) return st;
    }
    if (rings == 3)
        return from_cuda(launch_ring_fill(k, v, B, T, window, cfg->Hkv, cfg->D, cfg->dtype, ring_k,
                                          ring_v, slot_pos, stream));
    return YOCO_OK;
}

yoco_status yoco_cross_prefill(const void *q, const void *k, const void *v, int32_t B, int64_t Tq,
                               int64_t Tkv, int64_t q_pos0, void *o, float *lse,
                               const yoco_attn_cfg *cfg, cudaStream_t stream) {
    yoco_status st = check_cfg(cfg);
    if (st != YOCO_OK) return st;
    if (B < 0 || Tq < 0 || Tkv < 0 || q_pos0 < 0 || q_pos0 + Tq > Tkv) return YOCO_ERR_INVALID;
    if (B == 0 || Tq == 0) return YOCO_OK;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(o) || !ok_opt(lse)) return YOCO_ERR_INVALID;
    PrefillArgs a;
    a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
    a.B = B; a.Tq = Tq; a.Tkv = Tkv; a.q_pos0 = q_pos0; a.window = 0;
    a.Hq = cfg->Hq; a.Hkv = cfg->Hkv; a.D = cfg->D; a.dtype = cfg->dtype;
    a.scale = eff_scale(cfg);
    return run_prefill(a, stream);
}

yoco_status yoco_attention_prefill(const void *q, const void *k, const void *v, int32_t B, int64_t Tq,
                                   int64_t Tkv, int64_t q_pos0, int32_t window, void *o, float *lse,
                                   const yoco_attn_cfg *cfg, cudaStream_t stream) {
    yoco_status st = check_cfg(cfg);
    if (st != YOCO_OK) return st;
    if (B < 0 || Tq < 0 || Tkv < 0 || q_pos0 < 0 || q_pos0 + Tq > Tkv || window < 0) return YOCO_ERR_INVALID;
    if (B == 0 || Tq == 0) return YOCO_OK;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(o) || !ok_opt(lse)) return YOCO_ERR_INVALID;
    PrefillArgs a;
    a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
    a.B = B; a.Tq = Tq; a.Tkv = Tkv; a.q_pos0 = q_pos0; a.window = window;
    a.Hq = cfg->Hq; a.Hkv = cfg->Hkv; a.D = cfg->D; a.dtype = cfg->dtype;
    a.scale = eff_scale(cfg);
    return run_prefill(a, stream);
}

size_t yoco_cross_decode_workspace_size(int32_t B, int64_t max_len, const yoco_attn_cfg *cfg) {
    if (check_cfg(cfg) != YOCO_OK) return 0;
    DecodePlan pl;
    if (!make_decode_plan(B, max_len, cfg->Hq, cfg->Hkv, cfg->D, cfg->dtype, &pl)) return 0;
    return pl.ws_bytes;
}

size_t yoco_swa_decode_workspace_size(int32_t B, int32_t window, const yoco_attn_cfg *cfg) {
    return yoco_cross_decode_workspace_size(B, window, cfg);
}

yoco_status yoco_cross_decode(const void *q, const void *k_cache, const void *v_cache,
                              int64_t cache_rows, const int64_t *seq_start, const int32_t *seq_len,
                              int32_t B, int64_t max_len, void *o, float *lse, void *workspace,
                              size_t ws_bytes, const yoco_attn_cfg *cfg, cudaStream_t stream) {
    yoco_status st = check_cfg(cfg);
    if (st != YOCO_OK) return st;
    if (B < 0 || max_len < 1 || !ok_cache_rows(cache_rows)) return YOCO_ERR_INVALID;
    if (B == 0) return YOCO_OK;
    if (!ok_ptr(q) || !ok_ptr(k_cache) || !ok_ptr(v_cache) || !ok_ptr(seq_start) ||
        !seq_len || !ok_ptr(o) || !ok_opt(lse))
        return YOCO_ERR_INVALID;
    DecodePlan pl;
    if (!make_decode_plan(B, max_len, cfg->Hq, cfg->Hkv, cfg->D, cfg->dtype, &pl))
        return YOCO_ERR_UNSUPPORTED;
    if (!workspace || !aligned16(workspace) || ws_bytes < pl.ws_bytes) return YOCO_ERR_WORKSPACE;
    DecodeArgs a;
    a.q = q; a.k = k_cache; a.v = v_cache; a.seq_start = seq_start; a.seq_len = seq_len;
    a.slot_pos = nullptr; a.pos = nullptr; a.window = 0; a.k_new = a.v_new = nullptr;
    a.cache_rows = cache_rows; a.max_len = max_len;
    a.B = B; a.Hq = cfg->Hq; a.Hkv = cfg->Hkv; a.D = cfg->D; a.dtype = cfg->dtype;
    a.scale = eff_scale(cfg); a.o = o; a.lse = lse; a.ws = workspace;
    return from_cuda(launch_decode(a, pl, stream));
}

yoco_status yoco_swa_decode(const void *q, const void *k_new, const void *v_new,
                            const int64_t *pos, int32_t B, int32_t window, void *ring_k,
                            void *ring_v, int32_t *slot_pos, void *o, void *workspace,
                            size_t ws_bytes, const yoco_attn_cfg *cfg, cudaStream_t stream) {
    yoco_status st = check_cfg(cfg);
    if (st != YOCO_OK) return st;
    if (B < 0 || window < 1) return YOCO_ERR_INVALID;
    if (B == 0) return YOCO_OK;
    if (!ok_ptr(q) || !ok_ptr(k_new) || !ok_ptr(v_new) || !ok_ptr(pos) || !ok_ptr(ring_k) ||
        !ok_ptr(ring_v) || !ok_ptr(slot_pos) || !ok_ptr(o))
        return YOCO_ERR_INVALID;
    DecodePlan pl;
    if (!make_decode_plan(B, window, cfg->Hq, cfg->Hkv, cfg->D, cfg->dtype, &pl))
        return YOCO_ERR_UNSUPPORTED;
    if (!workspace || !aligned16(workspace) || ws_bytes < pl.ws_bytes) return YOCO_ERR_WORKSPACE;
    // the window read skips the new token's slot; the merge adds the new
    // token and writes it into the ring (no separate ring-write kernel)
    DecodeArgs a;
    a.q = q; a.k = ring_k; a.v = ring_v; a.seq_start = nullptr; a.seq_len = nullptr;
    a.slot_pos = slot_pos; a.pos = pos; a.window = window;
    a.k_new = k_new; a.v_new = v_new;
    a.cache_rows = (int64_t)B * window; a.max_len = window;
    a.B = B; a.Hq = cfg->Hq; a.Hkv = cfg->Hkv; a.D = cfg->D; a.dtype = cfg->dtype;
    a.scale = eff_scale(cfg); a.o = o; a.lse = nullptr; a.ws = workspace;
    // bf16: one clustered launch (window read, merge, new token, ring write);
    // other shapes: the split kernel and the merge
    const cudaError_t e = launch_ring_decode(a, stream);
    if (e != cudaErrorNotSupported) return from_cuda(e);
    return from_cuda(launch_decode(a, pl, stream));
}

size_t yoco_swa_decode_step_workspace_size(int32_t B, int32_t window, const yoco_attn_cfg *cfg) {
    if (check_cfg(cfg) != YOCO_OK || B < 0 || window < 1) return 0;
    const size_t dws = yoco_swa_decode_workspace_size(B, window, cfg);
    if (dws == 0) return 0;
    const size_t kv = ((size_t)B * cfg->Hkv * cfg->D * dtype_bytes(cfg->dtype) + 15) / 16 * 16;
    return 2 * kv + dws;
}

yoco_status yoco_swa_decode_step(const void *x, int32_t d_model, const void *w_kv, int32_t apply_ln,
                                 float ln_eps, const void *k_base, const void *v_base, float w_k, float w_v,
                                 const void *q, const int64_t *pos, int32_t B, int32_t window, void *ring_k,
                                 void *ring_v, int32_t *slot_pos, void *o, void *k_out, void *v_out,
                                 void *workspace, size_t ws_bytes, const yoco_attn_cfg *cfg,
                                 cudaStream_t stream) {
    yoco_status st = check_cfg(cfg);
    if (st != YOCO_OK) return st;
    if (B < 0 || window < 1 || d_model < 1 || !(ln_eps > 0.f) || !isfinite(w_k) || !isfinite(w_v))
        return YOCO_ERR_INVALID;
    if (B == 0) return YOCO_OK;
    if (!ok_ptr(x) || !ok_ptr(w_kv) || !ok_ptr(q) || !ok_ptr(pos) || !ok_ptr(ring_k) || !ok_ptr(ring_v) ||
        !ok_ptr(slot_pos) || !ok_ptr(o) || !ok_opt(k_base) || !ok_opt(v_base) || !ok_opt(k_out) ||
        !ok_opt(v_out))
        return YOCO_ERR_INVALID;
    if ((int64_t)d_model * dtype_bytes(cfg->dtype) % 16 != 0) return YOCO_ERR_INVALID;
    DecodePlan pl;
    if (!make_decode_plan(B, window, cfg->Hq, cfg->Hkv, cfg->D, cfg->dtype, &pl)) return YOCO_ERR_UNSUPPORTED;
    const size_t need = yoco_swa_decode_step_workspace_size(B, window, cfg);
    if (!workspace || !aligned16(workspace) || need == 0 || ws_bytes < need) return YOCO_ERR_WORKSPACE;
    // the projection into k_out / v_out (or the workspace), then the window
    // decode.  bf16 few-token projections stream their weights through
    // registers; after that kernel the window decode runs in its compact
    // layout (four CTAs a head), the faster one there.
    const size_t kvb = ((size_t)B * cfg->Hkv * cfg->D * dtype_bytes(cfg->dtype) + 15) / 16 * 16;
    unsigned char *ws = static_cast<unsigned char *>(workspace);
    void *kn = k_out ? k_out : ws;
    void *vn = v_out ? v_out : ws + kvb;
    LinearArgs la;
    la.x = x; la.w = w_kv; la.n = B; la.d_in = d_model;
    la.d_out = 2 * cfg->Hkv * cfg->D; la.split_col = cfg->Hkv * cfg->D;
    la.apply_ln = apply_ln ? 1 : 0; la.eps = ln_eps;
    la.out0 = kn; la.out1 = vn; la.base0 = k_base; la.base1 = v_base;
    la.w0 = w_k; la.w1 = w_v; la.dst_rows = nullptr; la.dtype = cfg->dtype;
    cudaError_t e = launch_linear_few_reg(la, stream);
    const bool compact = e == cudaSuccess;
    if (e == cudaErrorNotSupported) {
        cudaGetLastError();
        st = run_linear(la, stream);
        if (st != YOCO_OK) return st;
    } else if (e != cudaSuccess) {
        return from_cuda(e);
    }
    DecodeArgs a;
    a.q = q; a.k = ring_k; a.v = ring_v; a.seq_start = nullptr; a.seq_len = nullptr;
    a.slot_pos = slot_pos; a.pos = pos; a.window = window;
    a.k_new = kn; a.v_new = vn;
    a.cache_rows = (int64_t)B * window; a.max_len = window;
    a.B = B; a.Hq = cfg->Hq; a.Hkv = cfg->Hkv; a.D = cfg->D; a.dtype = cfg->dtype;
    a.scale = eff_scale(cfg); a.o = o; a.lse = nullptr; a.ws = ws + 2 * kvb;
    const cudaError_t e2 = launch_ring_decode(a, stream, compact);
    if (e2 != cudaErrorNotSupported) return from_cuda(e2);
    cudaGetLastError();
    return from_cuda(launch_decode(a, pl, stream));
}

int64_t yoco_kv_i8_row_bytes(const yoco_attn_cfg *cfg) {
    if (!cfg || cfg->Hkv < 1 || (cfg->D != 64 && cfg->D != 128)) return 0;
    return i8_row_bytes(cfg->Hkv, cfg->D);
}

yoco_status yoco_kv_quantize_i8(const void *k, const void *v, int64_t n_tok, const int64_t *dst_rows, void *k_i8,
                                void *v_i8, const yoco_attn_cfg *cfg, cudaStream_t stream) {
    yoco_status st = check_cfg(cfg);
    if (st != YOCO_OK) return st;
    if (n_tok < 0) return YOCO_ERR_INVALID;
    if (n_tok == 0) return YOCO_OK;
    if (!ok_ptr(k) || !ok_ptr(v) || !ok_opt(dst_rows) || !ok_ptr(k_i8) || !ok_ptr(v_i8)) return YOCO_ERR_INVALID;
    return from_cuda(launch_kv_quantize_i8(k, v, n_tok, cfg->Hkv, cfg->D, cfg->dtype, dst_rows, k_i8, v_i8, stream));
}

yoco_status yoco_cross_decode_i8(const void *q, const void *k_i8, const void *v_i8, int64_t cache_rows,
                                 const int64_t *seq_start, const int32_t *seq_len, int32_t B, int64_t max_len,
                                 void *o, float *lse, void *workspace, size_t ws_bytes, const yoco_attn_cfg *cfg,
                                 cudaStream_t stream) {
    yoco_status st = check_cfg(cfg);
    if (st != YOCO_OK) return st;
    if (B < 0 || max_len < 1 || !ok_cache_rows(cache_rows)) return YOCO_ERR_INVALID;
    if (B == 0) return YOCO_OK;
    if (!ok_ptr(q) || !ok_ptr(k_i8) || !ok_ptr(v_i8) || !ok_ptr(seq_start) || !seq_len || !ok_ptr(o) || !ok_opt(lse))
        return YOCO_ERR_INVALID;
    if (cfg->D != 128 || cfg->dtype != YOCO_BF16) return YOCO_ERR_UNSUPPORTED;
    DecodePlan pl;
    if (!make_decode_plan(B, max_len, cfg->Hq, cfg->Hkv, cfg->D, cfg->dtype, &pl)) return YOCO_ERR_UNSUPPORTED;
    if (!workspace || !aligned16(workspace) || ws_bytes < pl.ws_bytes) return YOCO_ERR_WORKSPACE;
    DecodeArgs a;
    a.q = q; a.k = k_i8; a.v = v_i8; a.seq_start = seq_start; a.seq_len = seq_len;
    a.slot_pos = nullptr; a.pos = nullptr; a.window = 0; a.k_new = a.v_new = nullptr;
    a.cache_rows = cache_rows; a.max_len = max_len;
    a.B = B; a.Hq = cfg->Hq; a.Hkv = cfg->Hkv; a.D = cfg->D; a.dtype = cfg->dtype;
    a.scale = eff_scale(cfg); a.o = o; a.lse = lse; a.ws = workspace;
    return from_cuda(launch_decode_i8(a, pl, stream));
}

size_t yoco_gret_prefill_workspace_size(int32_t B, int64_t T, const yoco_attn_cfg *cfg) {
    if (check_cfg(cfg) != YOCO_OK || cfg->Hq != cfg->Hkv || cfg->dtype != YOCO_BF16) return 0;
    return gret_workspace_bytes(B, cfg->Hq, T, cfg->D);
}

yoco_status yoco_gret_prefill(const void *q, const void *k, const void *v, const float *g, int32_t B,
                              int64_t T, float tau, float *state, void *o, void *workspace, size_t ws_bytes,
                              const yoco_attn_cfg *cfg, cudaStream_t stream) {
    yoco_status st = check_cfg(cfg);
    if (st != YOCO_OK) return st;
    if (cfg->Hq != cfg->Hkv || B < 0 || T < 0 || !(tau > 0.f) || isinf(tau)) return YOCO_ERR_INVALID;
    if (B == 0 || T == 0) return YOCO_OK;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(g) || !ok_opt(state) || !ok_ptr(o) ||
        !ok_opt(workspace))
        return YOCO_ERR_INVALID;
    if (cfg->dtype != YOCO_BF16) return YOCO_ERR_UNSUPPORTED;
    // a workspace enables the split over superchunks; one smaller than the
    // size query's answer is an error, a NULL one (or a size of 0) means no split
    const size_t need = gret_workspace_bytes(B, cfg->Hq, T, cfg->D);
    if (workspace && ws_bytes < need) return YOCO_ERR_WORKSPACE;
    GretArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.state = state; a.o = o;
    a.B = B; a.H = cfg->Hq; a.D = cfg->D; a.dtype = cfg->dtype; a.T = T;
    a.tau = tau; a.scale = eff_scale(cfg);
    a.ws = (workspace && need > 0) ? workspace : nullptr;
    return from_cuda(launch_gret_prefill(a, stream));
}

yoco_status yoco_gret_decode(const void *q, const void *k, const void *v, const float *g, int32_t B,
                             float tau, float *state, void *o, const yoco_attn_cfg *cfg, cudaStream_t stream) {
    yoco_status st = check_cfg(cfg);
    if (st != YOCO_OK) return st;
    if (cfg->Hq != cfg->Hkv || B < 0 || !(tau > 0.f) || isinf(tau)) return YOCO_ERR_INVALID;
    if (B == 0) return YOCO_OK;
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(g) || !ok_ptr(state) || !ok_ptr(o))
        return YOCO_ERR_INVALID;
    GretArgs a;
    a.q = q; a.k = k; a.v = v; a.g = g; a.state = state; a.o = o;
    a.B = B; a.H = cfg->Hq; a.D = cfg->D; a.dtype = cfg->dtype; a.T = 1;
    a.tau = tau; a.scale = eff_scale(cfg); a.ws = nullptr;
    return from_cuda(launch_gret_decode(a, stream));
}

yoco_status yoco_debug_tile_schedule(int32_t kind, const yoco_attn_cfg *cfg, int32_t B, int64_t Tq,
                                     int64_t Tkv, int64_t q_pos0, int32_t window,
                                     const int64_t *seq_start, const int32_t *seq_len, int64_t max_len,
                                     int32_t n_cta, int64_t *records, int64_t cap,
                                     int64_t *n_records) {
    yoco_status st = check_cfg(cfg);
    if (st != YOCO_OK) return st;
    if (!n_records || cap < 0 || (cap > 0 && !records) || B < 0 || n_cta < 0) return YOCO_ERR_INVALID;
    const int sms = n_cta > 0 ? n_cta : device_sm_count();
    int64_t n = 0;
    auto put = [&](int64_t a, int64_t b, int64_t c, int64_t d, int64_t e, int64_t f) {
        if (n < cap) {
            int64_t *r = records + 6 * n;
            r[0] = a; r[1] = b; r[2] = c; r[3] = d; r[4] = e; r[5] = f;
        }
        ++n;
    };
    if (kind == YOCO_SCHEDULE_PREFILL) {
        if (Tq < 0 || Tkv < 0 || q_pos0 < 0 || q_pos0 + Tq > Tkv || window < 0) return YOCO_ERR_INVALID;
        sched::PrefillShape s;
        s.B = B; s.Hq = cfg->Hq; s.Hkv = cfg->Hkv;
        s.Tq = Tq; s.Tkv = Tkv; s.q_pos0 = q_pos0; s.window = window;
        // the kernel run_prefill picks for bf16: two heads per work tile when
        // the group size is even, else one
        const bool pairs = cfg->dtype == YOCO_BF16 && sched::prefill_pairs_heads(cfg->Hq, cfg->Hkv);
        const int heads = pairs ? 2 : 1;
        const int64_t n_qtiles = (Tq + sched::kPrefillBM - 1) / sched::kPrefillBM;
        const int64_t n_work = n_qtiles * (cfg->Hq / heads) * B;
        if (n_work > INT32_MAX / 2) return YOCO_ERR_UNSUPPORTED;
        s.n_qtiles = (int32_t)n_qtiles;
        const int grid = (int)(n_work < sms ? n_work : sms);
        s.band = sched::prefill_band(grid, (cfg->Hq / cfg->Hkv) / heads,
                                     (int64_t)B * Tkv * cfg->Hkv * cfg->D * dtype_bytes(cfg->dtype) * 2, window);
        for (int c = 0; c < grid; ++c)
            for (int r = 0;; ++r) {
                const int w = sched::prefill_work_index(r, c, grid);
                if (w >= n_work) break;
                const sched::PrefillWork x = pairs ? sched::prefill_pair_work(s, w) : sched::prefill_work(s, w);
                for (int t = 0; t < x.n_kv; ++t)
                    for (int hh = 0; hh < heads; ++hh)
                        put(c, x.b, x.h + hh, x.qt, x.jt_lo + t, sched::prefill_tile_masked(s, x, t) ? 1 : 0);
            }
    } else if (kind == YOCO_SCHEDULE_DECODE) {
        if (max_len < 1 || (B > 0 && (!seq_start || !seq_len))) return YOCO_ERR_INVALID;
        DecodePlan pl;
        if (!make_decode_plan(B, max_len, cfg->Hq, cfg->Hkv, cfg->D, cfg->dtype, &pl))
            return YOCO_ERR_UNSUPPORTED;
        // the compact unit list, sequence by sequence, as the kernel enumerates it
        // (the cache's row count is not an argument here: a sequence is in
        // range when 1 <= seq_len <= max_len and seq_start >= 0)
        auto units = [&](int b) {
            return sched::decode_seq_ok(seq_start[b], seq_len[b], max_len, INT64_MAX)
                       ? sched::decode_units(seq_len[b], pl.split, pl.n_split)
                       : 0;
        };
        int64_t total = 0;
        for (int b = 0; b < B; ++b) total += units(b);
        const int64_t slots = (int64_t)B * pl.n_split;
        const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(slots, sms));
        for (int c = 0; c < grid; ++c) {
            int b = 0;
            int64_t before = 0;  // units of sequences < b
            for (int64_t u = c; u < total; u += grid) {
                while (before + units(b) <= u) before += units(b++);
                const int64_t sidx = u - before;
                const int64_t t0 = sidx * pl.split;
                const int64_t n_tok = std::min<int64_t>(pl.split, seq_len[b] - t0);
                put(c, b, sidx, seq_start[b] + t0, n_tok, (n_tok + pl.stage_tokens - 1) / pl.stage_tokens);
            }
        }
    } else {
        return YOCO_ERR_INVALID;
    }
    *n_records = n;
    return YOCO_OK;
}

double yoco_cache_bytes(int32_t L_self, int32_t window, int64_t N, const yoco_attn_cfg *cfg) {
    if (!cfg || L_self < 0 || window < 0 || N < 0 || cfg->Hkv < 1 || cfg->D < 1) return -1.0;
    const double row = 2.0 * cfg->Hkv * cfg->D * (cfg->dtype == YOCO_BF16 ? 2.0 : 4.0);
    const int64_t c = window < N ? window : N;
    return row * ((double)N + (double)L_self * (double)c);
}

yoco_status yoco_debug_wait_timeout_probe(cudaStream_t stream) {
    return from_cuda(launch_wait_timeout_probe(stream));
}

yoco_status yoco_get_device_status(cudaStream_t stream) {
    const cudaError_t e = cudaStreamSynchronize(stream);
    const unsigned int s = read_and_clear_status_decode() | read_and_clear_status_prefill_tc() |
                           read_and_clear_status_prefill_pair() | read_and_clear_status_project_tc() |
                           read_and_clear_status_gret_tc() | read_and_clear_status_linear() |
                           read_and_clear_status_ring() | read_and_clear_status_step_proj();
    if (s & 1u) return YOCO_ERR_TIMEOUT;
    if (s & 2u) return YOCO_ERR_INVALID;
    return e == cudaSuccess ? YOCO_OK : YOCO_ERR_CUDA;
}

}  // extern "C"
