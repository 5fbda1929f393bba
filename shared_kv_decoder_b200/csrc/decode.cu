// Split-KV decode attention for the cross-decoder's shared cache and the
// self-decoder's sliding-window ring (sm_100a).
//
// "YOCO: Caching Once for Decoder-Decoder Long-Context Language Models"
// (podcast transcript), cue 26: at every decode step each cross-decoder layer
// streams the whole shared KV, so decode is bound by HBM bandwidth (cue 4).
// The baseline Transformer of "You Only Cache Once" (paperlayer summary,
// section 2) used Flash-Decoding; the same split-then-merge idea is used
// here, laid out for B200:
//
//  * A CTA owns one unit = a contiguous token range of one sequence for ALL
//    KV heads, so each pipeline stage is ONE contiguous block of HBM
//    (128 rows of [Hkv, D] K plus the same of V) moved by a single
//    cp.async.bulk per tensor into a 2-4 deep shared-memory ring (mbarrier
//    complete_tx).  A dedicated producer warp issues the copies; eight
//    consumer warps compute.  Persistent grid: one CTA per SM strides over
//    the units.
//  * Consumer warp w serves KV head w % Hkv and a 16-token subset of each
//    stage; its eight-lane groups each own one token and split the head dim
//    in 16-byte chunks (conflict-free shared loads), with every query head
//    of the GQA group held in registers, so K/V bytes are read once for all
//    Hq/Hkv query heads.
//  * Softmax is online in the exp2 domain, rescaled once per stage; every
//    token group keeps its own running max, merged with the other groups at
//    the end of the unit; the partial (m, l, o) goes to the workspace and a
//    second kernel merges the splits (log-sum-exp weighting, one warp per
//    (sequence, query head)).
//  * Ring mode (self-decoder): the cache is the ring [B, window, Hkv, D] and
//    a slot is visible when its stored position lies in (pos - window, pos].
#include "common.cuh"
#include "launch.h"

#include <algorithm>

namespace yoco {

static __device__ unsigned int g_status_decode;

constexpr int kConsumerWarps = 8;
constexpr int kDecodeThreads = 32 * (kConsumerWarps + 1);
constexpr int kRowsPerStage = 128;  // stage_tokens * Hkv
constexpr int kTokPerWarp = 16;     // stage tokens handled by one consumer warp
constexpr int kLanesPerTok = 8;
constexpr int kTokPerPass = 32 / kLanesPerTok;
constexpr int kPasses = kTokPerWarp / kTokPerPass;
constexpr int64_t kTargetUnits = 148 * 8;

struct DecodeKParams {
    const void *q, *k, *v;
    const int64_t *seq_start;
    const int32_t *seq_len;
    const int32_t *slot_pos;
    const int64_t *pos;
    int32_t window;
    int32_t B, Hkv, Hq;
    int64_t stage_tokens, split, n_split;
    int32_t sub, stages;
    float scale_log2;
    float *ws_o, *ws_ml;
};

// Before the producer leaves, wait (bounded) until the copies of the last
// `stages` iterations have landed, so no bulk copy is still writing into this
// CTA's shared memory after it exits.  On the normal path every one of them
// completed long ago and this returns at once.
static __device__ void producer_drain(uint64_t *full, uint32_t issued, int stages) {
    const uint32_t first = issued > (uint32_t)stages ? issued - (uint32_t)stages : 0u;
    for (uint32_t itg = first; itg < issued; ++itg)
        if (!mbar_wait(&full[itg % stages], (itg / stages) & 1u, &g_status_decode)) return;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kDecodeThreads, 1) decode_split_kernel(const DecodeKParams p) {
    using C = Chunk<T>;
    constexpr int EPC = C::N;                 // elements per 16-byte chunk
    constexpr int CPR = D / EPC;              // chunks per head row
    constexpr int CPL = CPR / kLanesPerTok;   // chunks per lane
    constexpr int DPL = CPL * EPC;            // dims per lane
    static_assert(CPL >= 1 && CPR % kLanesPerTok == 0, "head dim too small for the lane layout");

    if (*(volatile unsigned int *)&g_status_decode) return;  // an earlier CTA timed out
    extern __shared__ __align__(128) unsigned char smem[];
    const int64_t row_elems = (int64_t)p.Hkv * D;
    const size_t half_bytes = (size_t)kRowsPerStage * D * sizeof(T);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)p.stages * 2 * half_bytes);
    uint64_t *empty = full + p.stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    const T *kg = static_cast<const T *>(p.k);
    const T *vg = static_cast<const T *>(p.v);
    const int64_t total_units = (int64_t)p.B * p.n_split;
    uint32_t it = 0;  // pipeline iteration counter shared by producer and consumers

    for (int64_t u = blockIdx.x; u < total_units; u += gridDim.x) {
        const int b = (int)(u / p.n_split);
        const int64_t s = u % p.n_split;
        const int64_t len = p.seq_len ? (int64_t)p.seq_len[b] : (int64_t)p.window;
        const int64_t t0 = s * p.split;
        if (t0 >= len) continue;
        const int64_t n_tok = min(p.split, len - t0);
        const int64_t row0 = (p.seq_start ? p.seq_start[b] : (int64_t)b * p.window) + t0;
        const int n_st = (int)((n_tok + p.stage_tokens - 1) / p.stage_tokens);

        if (warp == kConsumerWarps) {
            // ---------------------------------------------------- producer
            if (lane == 0) {
                for (int i = 0; i < n_st; ++i) {
                    const uint32_t itg = it + i;
                    const int st = (int)(itg % p.stages);
                    const uint32_t ph = (itg / p.stages) & 1u;
                    if (!mbar_wait(&empty[st], ph ^ 1u, &g_status_decode)) {
                        producer_drain(full, it + i, p.stages);
                        return;
                    }
                    const int64_t cnt = min(p.stage_tokens, n_tok - (int64_t)i * p.stage_tokens);
                    const uint32_t bytes = (uint32_t)(cnt * row_elems * sizeof(T));
                    const int64_t off = (row0 + (int64_t)i * p.stage_tokens) * row_elems;
                    unsigned char *sk = smem + (size_t)st * 2 * half_bytes;
                    mbar_arrive_expect_tx(&full[st], 2 * bytes);
                    bulk_g2s(sk, kg + off, bytes, &full[st]);
                    bulk_g2s(sk + half_bytes, vg + off, bytes, &full[st]);
                }
            }
        } else {
            // --------------------------------------------------- consumers
            const int g = warp % p.Hkv;     // KV head
            const int j = warp / p.Hkv;     // token subset of each stage
            const int tg = lane / kLanesPerTok;
            const int r = lane % kLanesPerTok;
            const int64_t pos_b = p.pos ? p.pos[b] : 0;
            const int32_t *sp = p.slot_pos ? p.slot_pos + (int64_t)b * p.window + t0 : nullptr;

            float qf[G][DPL];
            {
                const T *qb = static_cast<const T *>(p.q) + ((int64_t)b * p.Hq + (int64_t)g * G) * D;
#pragma unroll
                for (int hh = 0; hh < G; ++hh) {
#pragma unroll
                    for (int c = 0; c < CPL; ++c) {
                        const uint4 raw = reinterpret_cast<const uint4 *>(qb + hh * D)[r + kLanesPerTok * c];
                        C::unpack(raw, &qf[hh][c * EPC]);
                    }
#pragma unroll
                    for (int e = 0; e < DPL; ++e) qf[hh][e] *= p.scale_log2;
                }
            }
            float m[G], l[G], o[G][DPL];
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                m[hh] = -INFINITY;
                l[hh] = 0.f;
#pragma unroll
                for (int e = 0; e < DPL; ++e) o[hh][e] = 0.f;
            }

            for (int i = 0; i < n_st; ++i) {
                const uint32_t itg = it + i;
                const int st = (int)(itg % p.stages);
                const uint32_t ph = (itg / p.stages) & 1u;
                if (!__all_sync(0xffffffffu, mbar_wait(&full[st], ph, &g_status_decode))) return;
                const T *sk = reinterpret_cast<const T *>(smem + (size_t)st * 2 * half_bytes);
                const T *sv = reinterpret_cast<const T *>(smem + (size_t)st * 2 * half_bytes + half_bytes);

                float sc[kPasses][G];
                bool valid[kPasses];
#pragma unroll
                for (int ps = 0; ps < kPasses; ++ps) {
                    const int lt = j * kTokPerWarp + ps * kTokPerPass + tg;  // token in stage
                    const int64_t tok = (int64_t)i * p.stage_tokens + lt;    // token in unit
                    bool vld = tok < n_tok;
                    if (vld && sp) {
                        const int32_t sp_t = sp[tok];
                        vld = sp_t >= 0 && sp_t <= pos_b && (int64_t)sp_t > pos_b - p.window;
                    }
                    valid[ps] = vld;
                    const uint4 *kr = reinterpret_cast<const uint4 *>(sk + ((int64_t)lt * p.Hkv + g) * D);
                    float kf[DPL];
#pragma unroll
                    for (int c = 0; c < CPL; ++c) C::unpack(kr[r + kLanesPerTok * c], &kf[c * EPC]);
#pragma unroll
                    for (int hh = 0; hh < G; ++hh) {
                        float a0 = 0.f, a1 = 0.f;
#pragma unroll
                        for (int e = 0; e < DPL; e += 2) {
                            a0 = fmaf(qf[hh][e], kf[e], a0);
                            a1 = fmaf(qf[hh][e + 1], kf[e + 1], a1);
                        }
                        float acc = a0 + a1;
                        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                        acc += __shfl_xor_sync(0xffffffffu, acc, 4);
                        sc[ps][hh] = acc;
                    }
                }
                // one rescale per stage
#pragma unroll
                for (int hh = 0; hh < G; ++hh) {
                    float mx = m[hh];
#pragma unroll
                    for (int ps = 0; ps < kPasses; ++ps)
                        if (valid[ps]) mx = fmaxf(mx, sc[ps][hh]);
                    const float alpha = (mx == -INFINITY) ? 1.f : exp2f(m[hh] - mx);
                    m[hh] = mx;
                    l[hh] *= alpha;
#pragma unroll
                    for (int e = 0; e < DPL; ++e) o[hh][e] *= alpha;
                }
#pragma unroll
                for (int ps = 0; ps < kPasses; ++ps) {
                    if (!valid[ps]) continue;
                    const int lt = j * kTokPerWarp + ps * kTokPerPass + tg;
                    const uint4 *vr = reinterpret_cast<const uint4 *>(sv + ((int64_t)lt * p.Hkv + g) * D);
                    float vf[DPL];
#pragma unroll
                    for (int c = 0; c < CPL; ++c) C::unpack(vr[r + kLanesPerTok * c], &vf[c * EPC]);
#pragma unroll
                    for (int hh = 0; hh < G; ++hh) {
                        const float pp = exp2f(sc[ps][hh] - m[hh]);
                        l[hh] += pp;
#pragma unroll
                        for (int e = 0; e < DPL; ++e) o[hh][e] = fmaf(pp, vf[e], o[hh][e]);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            }

            // merge the four token groups of the warp, write the partial
            const int64_t entry = ((int64_t)b * p.n_split + s) * p.sub + j;
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                float M = m[hh];
                M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 8));
                M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 16));
                const float a = (m[hh] == -INFINITY) ? 0.f : exp2f(m[hh] - M);
                float L = l[hh] * a;
                L += __shfl_xor_sync(0xffffffffu, L, 8);
                L += __shfl_xor_sync(0xffffffffu, L, 16);
                float ov[DPL];
#pragma unroll
                for (int e = 0; e < DPL; ++e) {
                    float t = o[hh][e] * a;
                    t += __shfl_xor_sync(0xffffffffu, t, 8);
                    t += __shfl_xor_sync(0xffffffffu, t, 16);
                    ov[e] = t;
                }
                const int64_t hq = (int64_t)g * G + hh;
                if (tg == 0) {
                    float *dst = p.ws_o + (entry * p.Hq + hq) * D;
#pragma unroll
                    for (int c = 0; c < CPL; ++c) {
                        const int d0 = (r + kLanesPerTok * c) * EPC;
#pragma unroll
                        for (int e = 0; e < EPC; e += 4)
                            *reinterpret_cast<float4 *>(dst + d0 + e) =
                                make_float4(ov[c * EPC + e], ov[c * EPC + e + 1], ov[c * EPC + e + 2],
                                            ov[c * EPC + e + 3]);
                    }
                }
                if (lane == 0) {
                    p.ws_ml[(entry * p.Hq + hq) * 2 + 0] = M;
                    p.ws_ml[(entry * p.Hq + hq) * 2 + 1] = L;
                }
            }
        }
        it += (uint32_t)n_st;
    }
    if (warp == kConsumerWarps && lane == 0) producer_drain(full, it, p.stages);
}

template <typename T, int D>
__global__ void __launch_bounds__(128) decode_merge_kernel(const float *ws_o, const float *ws_ml,
                                                           const int32_t *seq_len, int32_t window,
                                                           int32_t B, int32_t Hq, int64_t split,
                                                           int64_t n_split, int32_t sub, T *o,
                                                           float *lse) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t idx = (int64_t)blockIdx.x * 4 + warp;
    if (idx >= (int64_t)B * Hq) return;
    const int b = (int)(idx / Hq), h = (int)(idx % Hq);
    const int64_t len = seq_len ? (int64_t)seq_len[b] : (int64_t)window;
    const int64_t n_s = min(n_split, max((int64_t)0, (len + split - 1) / split));
    const int64_t n_e = n_s * sub;
    const int64_t e0 = (int64_t)b * n_split * sub;

    float M = -INFINITY;
    for (int64_t e = lane; e < n_e; e += 32) M = fmaxf(M, ws_ml[((e0 + e) * Hq + h) * 2]);
    M = warp_max(M);
    float L = 0.f;
    constexpr int DPL = D / 32;
    float acc[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
    for (int64_t e = 0; e < n_e; ++e) {
        const float me = ws_ml[((e0 + e) * Hq + h) * 2];
        const float le = ws_ml[((e0 + e) * Hq + h) * 2 + 1];
        const float w = (me == -INFINITY) ? 0.f : exp2f(me - M);
        L += le * w;
        const float *src = ws_o + ((e0 + e) * Hq + h) * D;
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[i] = fmaf(w, src[lane + 32 * i], acc[i]);
    }
    const float inv = L > 0.f ? 1.f / L : 0.f;
    T *dst = o + ((int64_t)b * Hq + h) * D;
#pragma unroll
    for (int i = 0; i < DPL; ++i) dst[lane + 32 * i] = from_f32<T>(acc[i] * inv);
    if (lse && lane == 0) lse[(int64_t)b * Hq + h] = L > 0.f ? (M + log2f(L)) * kLn2 : -INFINITY;
}

bool make_decode_plan(int32_t B, int64_t max_len, int Hq, int Hkv, int D, int dtype,
                      DecodePlan *plan) {
    if (B < 0 || max_len < 1 || Hkv < 1 || kRowsPerStage % Hkv != 0 || Hkv > kConsumerWarps ||
        Hq % Hkv != 0)
        return false;
    DecodePlan pl;
    pl.stage_tokens = kRowsPerStage / Hkv;
    pl.sub = kConsumerWarps / Hkv;
    const int64_t min_split = 4 * pl.stage_tokens;
    int64_t per = ((int64_t)std::max(B, 1) * max_len + kTargetUnits - 1) / kTargetUnits;
    per = ((per + pl.stage_tokens - 1) / pl.stage_tokens) * pl.stage_tokens;
    pl.split = std::max(per, min_split);
    pl.n_split = (max_len + pl.split - 1) / pl.split;
    const size_t stage_bytes = 2 * (size_t)kRowsPerStage * D * dtype_bytes(dtype);
    pl.stages = (int)std::max<size_t>(1, std::min<size_t>(4, (200 * 1024) / stage_bytes));
    pl.smem_bytes = pl.stages * stage_bytes + 2 * pl.stages * sizeof(uint64_t);
    const size_t entries = (size_t)B * pl.n_split * pl.sub * Hq;
    pl.ws_bytes = entries * D * sizeof(float) + entries * 2 * sizeof(float);
    *plan = pl;
    return true;
}

int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

template <typename T, int D, int G>
static cudaError_t launch_decode_t(const DecodeArgs &a, const DecodePlan &pl, cudaStream_t st) {
    auto kern = decode_split_kernel<T, D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)pl.smem_bytes);
    if (e != cudaSuccess) return e;
    DecodeKParams p;
    p.q = a.q; p.k = a.k; p.v = a.v;
    p.seq_start = a.seq_start; p.seq_len = a.seq_len;
    p.slot_pos = a.slot_pos; p.pos = a.pos; p.window = a.window;
    p.B = a.B; p.Hkv = a.Hkv; p.Hq = a.Hq;
    p.stage_tokens = pl.stage_tokens; p.split = pl.split; p.n_split = pl.n_split;
    p.sub = pl.sub; p.stages = pl.stages;
    p.scale_log2 = a.scale * kLog2e;
    const size_t entries = (size_t)a.B * pl.n_split * pl.sub * a.Hq;
    p.ws_o = static_cast<float *>(a.ws);
    p.ws_ml = p.ws_o + entries * D;
    const int64_t units = (int64_t)a.B * pl.n_split;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(units, device_sm_count()));
    kern<<<grid, kDecodeThreads, pl.smem_bytes, st>>>(p);
    note_launches(2);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int mgrid = (int)(((int64_t)a.B * a.Hq + 3) / 4);
    decode_merge_kernel<T, D><<<mgrid, 128, 0, st>>>(p.ws_o, p.ws_ml, a.seq_len, a.window, a.B,
                                                     a.Hq, pl.split, pl.n_split, pl.sub,
                                                     static_cast<T *>(a.o), a.lse);
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t launch_decode_g(const DecodeArgs &a, const DecodePlan &pl, cudaStream_t st) {
    switch (a.Hq / a.Hkv) {
        case 1: return launch_decode_t<T, D, 1>(a, pl, st);
        case 2: return launch_decode_t<T, D, 2>(a, pl, st);
        case 4: return launch_decode_t<T, D, 4>(a, pl, st);
        case 8: return launch_decode_t<T, D, 8>(a, pl, st);
    }
    return cudaErrorNotSupported;
}

cudaError_t launch_decode(const DecodeArgs &a, const DecodePlan &pl, cudaStream_t st) {
    if (a.B == 0) return cudaSuccess;
    if (a.dtype == kBF16) {
        if (a.D == 128) return launch_decode_g<__nv_bfloat16, 128>(a, pl, st);
        if (a.D == 64) return launch_decode_g<__nv_bfloat16, 64>(a, pl, st);
    } else {
        if (a.D == 128) return launch_decode_g<float, 128>(a, pl, st);
        if (a.D == 64) return launch_decode_g<float, 64>(a, pl, st);
    }
    return cudaErrorNotSupported;
}

// ------------------------------------------------------------------ ring
template <typename T>
__global__ void ring_write_kernel(const T *k_new, const T *v_new, const int64_t *pos, int32_t window,
                                  int64_t row_elems, T *ring_k, T *ring_v, int32_t *slot_pos) {
    const int b = blockIdx.x;
    const int64_t p = pos[b];
    const int64_t slot = ((p % window) + window) % window;
    T *dk = ring_k + ((int64_t)b * window + slot) * row_elems;
    T *dv = ring_v + ((int64_t)b * window + slot) * row_elems;
    for (int64_t i = threadIdx.x; i < row_elems; i += blockDim.x) {
        dk[i] = k_new[(int64_t)b * row_elems + i];
        dv[i] = v_new[(int64_t)b * row_elems + i];
    }
    if (threadIdx.x == 0) slot_pos[(int64_t)b * window + slot] = (int32_t)p;
}

cudaError_t launch_ring_write(const void *k_new, const void *v_new, const int64_t *pos, int32_t B,
                              int32_t window, int Hkv, int D, int dtype, void *ring_k,
                              void *ring_v, int32_t *slot_pos, cudaStream_t st) {
    if (B == 0) return cudaSuccess;
    const int64_t re = (int64_t)Hkv * D;
    note_launches(1);
    if (dtype == kBF16)
        ring_write_kernel<__nv_bfloat16><<<B, 256, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(k_new), static_cast<const __nv_bfloat16 *>(v_new), pos,
            window, re, static_cast<__nv_bfloat16 *>(ring_k), static_cast<__nv_bfloat16 *>(ring_v),
            slot_pos);
    else
        ring_write_kernel<float><<<B, 256, 0, st>>>(static_cast<const float *>(k_new),
                                                    static_cast<const float *>(v_new), pos, window, re,
                                                    static_cast<float *>(ring_k),
                                                    static_cast<float *>(ring_v), slot_pos);
    return cudaGetLastError();
}

// Ring contents after a prefill of T tokens: slot s keeps the newest position
// p < T with p mod window == s (slot_pos = p), or -1 and zeros.
template <typename T>
__global__ void ring_fill_kernel(const T *k, const T *v, int64_t T_len, int32_t window,
                                 int64_t row_elems, T *ring_k, T *ring_v, int32_t *slot_pos) {
    const int64_t s = blockIdx.x;
    const int b = blockIdx.y;
    T *dk = ring_k + ((int64_t)b * window + s) * row_elems;
    T *dv = ring_v + ((int64_t)b * window + s) * row_elems;
    if (s < T_len) {
        const int64_t p = s + (int64_t)window * ((T_len - 1 - s) / window);
        const T *sk = k + ((int64_t)b * T_len + p) * row_elems;
        const T *sv = v + ((int64_t)b * T_len + p) * row_elems;
        for (int64_t i = threadIdx.x; i < row_elems; i += blockDim.x) {
            dk[i] = sk[i];
            dv[i] = sv[i];
        }
        if (threadIdx.x == 0) slot_pos[(int64_t)b * window + s] = (int32_t)p;
    } else {
        for (int64_t i = threadIdx.x; i < row_elems; i += blockDim.x) {
            dk[i] = from_f32<T>(0.f);
            dv[i] = from_f32<T>(0.f);
        }
        if (threadIdx.x == 0) slot_pos[(int64_t)b * window + s] = -1;
    }
}

cudaError_t launch_ring_fill(const void *k, const void *v, int32_t B, int64_t T, int32_t window,
                             int Hkv, int D, int dtype, void *ring_k, void *ring_v,
                             int32_t *slot_pos, cudaStream_t st) {
    if (B == 0) return cudaSuccess;
    const int64_t re = (int64_t)Hkv * D;
    dim3 grid(window, B);
    note_launches(1);
    if (dtype == kBF16)
        ring_fill_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(
            static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v), T, window,
            re, static_cast<__nv_bfloat16 *>(ring_k), static_cast<__nv_bfloat16 *>(ring_v), slot_pos);
    else
        ring_fill_kernel<float><<<grid, 128, 0, st>>>(static_cast<const float *>(k),
                                                      static_cast<const float *>(v), T, window, re,
                                                      static_cast<float *>(ring_k),
                                                      static_cast<float *>(ring_v), slot_pos);
    return cudaGetLastError();
}

unsigned int read_and_clear_status_decode() {
    unsigned int h = 0, z = 0;
    if (cudaMemcpyFromSymbol(&h, g_status_decode, sizeof(h)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_status_decode, &z, sizeof(z));
    return h;
}

}  // namespace yoco
