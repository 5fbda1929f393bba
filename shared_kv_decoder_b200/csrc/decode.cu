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
//    KV heads, so K/V bytes are read once for every query head of the GQA
//    group.  Persistent grid: one CTA per SM strides over a compact list of
//    the non-empty units.  One producer warp fills a shared-memory ring of
//    stages (128 token-head rows of K and of V each); eight consumer warps
//    compute, warp w serving KV head w % Hkv and a 16-token subset of every
//    stage.
//  * bf16 (decode_tma_kernel): each stage arrives as a few 16 KB TMA tensor
//    boxes with the 128-byte swizzle; S = q K^T and O += P V are warp-wide
//    mma.sync tiles with the group's query heads as the A rows.  fp32
//    (decode_split_kernel) runs on the CUDA cores from one bulk copy per stage
//    and tensor.
//  * Softmax is online in the exp2 domain; the reference max only moves when
//    it grows by more than 2^8.  The partial (m, l, o) of each unit goes to
//    the workspace and a second kernel merges the splits (log-sum-exp
//    weighting, one warp per (sequence, query head)).
//  * Ring mode (self-decoder): the cache is the ring [B, window, Hkv, D] and
//    a slot is visible when its stored position lies in (pos - window, pos].
#include "common.cuh"
#include "launch.h"
#include "schedule.h"
#include "tc.cuh"

#include <algorithm>
#include <type_traits>

namespace yoco {

// Status word of this translation unit: bit 0 (kStatusTimeout) records a
// bounded wait that gave up, bit 1 (kStatusBadSequence) a decode sequence
// whose seq_start / seq_len were out of range.  Only a timeout makes later
// kernels exit at once; a bad sequence affects only itself.
static __device__ unsigned int g_status_decode;
constexpr unsigned int kStatusTimeout = 1u;
constexpr unsigned int kStatusBadSequence = 2u;

constexpr int kConsumerWarps = 8;
constexpr int kDecodeThreads = 32 * (kConsumerWarps + 1);
constexpr int kRowsPerStage = 128;  // stage_tokens * Hkv
constexpr int kTokPerWarp = 16;     // stage tokens handled by one consumer warp
constexpr int kLanesPerTok = 8;
constexpr int kTokPerPass = 32 / kLanesPerTok;
constexpr int kPasses = kTokPerWarp / kTokPerPass;
constexpr int64_t kMinUnits = 148, kMaxUnits = 148 * 12;   // decode units per call (see make_decode_plan)
constexpr int64_t kMaxUnitsPerSeq = 148 * 2;                 // units of one sequence at most
constexpr int64_t kUnitBytes = (int64_t)2 << 20;

struct DecodeKParams {
    const void *q, *k, *v;
    const int64_t *seq_start;
    const int32_t *seq_len;
    const int32_t *slot_pos;
    const int64_t *pos;
    int32_t window;
    int32_t B, Hkv, Hq;
    int64_t cache_rows, max_len;   // rows of the cache buffers; longest allowed sequence
    int64_t stage_tokens, split, n_split;
    int32_t sub, stages;
    float scale_log2;
    float *ws_o, *ws_ml;
};

// The u-th non-empty unit, counting sequence by sequence (a sequence of len
// tokens has ceil(len / split) units).  Computed by each warp with a
// 32-sequence-wide prefix scan, so every CTA strides over the same compact
// list and the ragged lengths spread evenly over the grid.  False when u is
// past the last unit.
static __device__ bool find_unit(const DecodeKParams &p, int64_t u, int *b_out, int64_t *s_out) {
    const int lane = threadIdx.x & 31;
    int64_t base = 0;
    for (int b0 = 0; b0 < p.B; b0 += 32) {
        const int b = b0 + lane;
        int64_t cnt = 0;
        if (b < p.B) {
            // a sequence whose length or rows are out of range has no units
            // (the merge kernel reports it); ring slots are always in range
            const int64_t len = p.seq_len ? (int64_t)p.seq_len[b] : (int64_t)p.window;
            if (!p.seq_len || sched::decode_seq_ok(p.seq_start[b], len, p.max_len, p.cache_rows))
                cnt = sched::decode_units(len, p.split, p.n_split);
        }
        int64_t incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int64_t total = __shfl_sync(0xffffffffu, incl, 31);
        if (u < base + total) {
            const unsigned hit = __ballot_sync(0xffffffffu, base + incl > u);
            const int src = __ffs(hit) - 1;
            const int64_t excl = __shfl_sync(0xffffffffu, incl - cnt, src);
            *b_out = b0 + src;
            *s_out = u - base - excl;
            return true;
        }
        base += total;
    }
    return false;
}

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

    pdl_trigger();
    pdl_wait();
    if (*(volatile unsigned int *)&g_status_decode & kStatusTimeout) return;  // an earlier CTA timed out
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
    uint32_t it = 0;  // pipeline iteration counter shared by producer and consumers

    for (int64_t u = blockIdx.x;; u += gridDim.x) {
        int b;
        int64_t s;
        if (!find_unit(p, u, &b, &s)) break;
        const int64_t len = p.seq_len ? (int64_t)p.seq_len[b] : (int64_t)p.window;
        const int64_t t0 = s * p.split;
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
            // ring mode: the slot the new token goes to is left out here (whatever it
            // holds is replaced); the merge adds the new token from k_new / v_new
            const int64_t new_slot = p.window > 0 ? ((pos_b % p.window) + p.window) % p.window : -1;

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
                        vld = sp_t >= 0 && sp_t <= pos_b && (int64_t)sp_t > pos_b - p.window &&
                              t0 + tok != new_slot;
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

// ---------------------------------------------------------------------------
// bf16 decode on the tensor cores (mma.sync m16n8k16, fp32 accumulate).
//
// The CUDA-core kernel above spends ~150 instructions per KB of K/V (unpack,
// per-head FMAs, eight-lane butterflies) and is issue-bound well below HBM
// bandwidth.  Here the GQA group's query heads form the M rows of a
// 16 x 16 A fragment (G <= 8 real rows), so S = q K^T and O += P V are a few
// warp-wide MMAs per 16 tokens.  P goes from the S accumulators straight into
// the A fragment of P.V (tokens 0-7 and 8-15 of the warp's 16 are the two S
// column tiles).
YOCO_DEV void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
YOCO_DEV void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// c += A * B for one m16n8k16 tile; the A rows 8-15 are always zero here.
YOCO_DEV void mma_16816(float *c, uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
YOCO_DEV uint32_t pack2_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
YOCO_DEV float ex2f(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// decode_tma_kernel: stages reach shared memory as TMA tensor copies.  The
// cache is viewed as the tensor {D, token, KV head} (token stride Hkv*D, head
// stride D), and one box {64, stage_tokens, Hkv} -- 16 KB, every head of the
// stage's tokens for one 64-column block -- lands as 128-byte rows ordered
// [head][token] under the 128-byte swizzle.  A stage is 2*D/64 such copies;
// an earlier feed with one 2 KB bulk copy per token row and tensor (rows
// padded by 16 bytes against bank conflicts) kept fewer bytes in flight and
// streamed 9% slower.  For a head, the eight token rows one ldmatrix gathers
// are consecutive swizzled rows, so they fall in eight different bank groups.
// A stage that ends a sequence short of stage_tokens is not copied (its box
// would read the next sequence's rows, or rows past the cache's end that the
// map fills with zeros); each consumer warp loads its own head's valid rows
// with plain loads and zeroes the rest.  This kernel reads the packed shared
// cache only: the bf16 sliding-window decode has a kernel of its own
// (ring_decode.cu).
template <int D, int G>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    decode_tma_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const DecodeKParams p) {
    pdl_trigger();
    pdl_wait();
    if (*(volatile unsigned int *)&g_status_decode & kStatusTimeout) return;  // an earlier CTA timed out
    static_assert(G >= 1 && G <= 8, "query heads per KV head");
    constexpr int KB = D / 64;                       // 64-column blocks per head row
    constexpr uint32_t kBox = kRowsPerStage * 128;   // one box: 128 rows of 128 bytes
    constexpr uint32_t kStage = 2 * KB * kBox;       // K boxes then V boxes
    constexpr int kChunks = D / 8;                   // 16-byte chunks per head row
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;   // the swizzle repeats every 1024 bytes
    unsigned char *smem = smem_raw + (sbase - raw);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)p.stages * kStage);
    uint64_t *empty = full + p.stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ST = (int)p.stage_tokens;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    const __nv_bfloat16 *kg = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *vg = static_cast<const __nv_bfloat16 *>(p.v);
    uint32_t it = 0;

    for (int64_t u = blockIdx.x;; u += gridDim.x) {
        int b;
        int64_t s;
        if (!find_unit(p, u, &b, &s)) break;
        const int64_t len = (int64_t)p.seq_len[b];
        const int64_t t0 = s * p.split;
        const int64_t n_tok = min(p.split, len - t0);
        const int64_t row0 = p.seq_start[b] + t0;
        const int n_st = (int)((n_tok + ST - 1) / ST);

        if (warp == kConsumerWarps) {
            // ---------------------------------------------------- producer
            for (int i = 0; i < n_st; ++i) {
                const uint32_t itg = it + i;
                const int st = (int)(itg % p.stages);
                const uint32_t ph = (itg / p.stages) & 1u;
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1u, &g_status_decode))) {
                    if (lane == 0) producer_drain(full, it + i, p.stages);
                    return;
                }
                const int64_t r = row0 + (int64_t)i * ST;
                if (lane == 0) {
                    if (n_tok - (int64_t)i * ST >= ST) {
                        const uint32_t dst = sbase + (uint32_t)st * kStage;
                        mbar_arrive_expect_tx(&full[st], kStage);
#pragma unroll
                        for (int kb = 0; kb < KB; ++kb) {
                            tc::tma_load_4d(dst + kb * kBox, &tm_k, kb * 64, (int)r, 0, 0, &full[st]);
                            tc::tma_load_4d(dst + (KB + kb) * kBox, &tm_v, kb * 64, (int)r, 0, 0, &full[st]);
                        }
                    } else {
                        mbar_arrive(&full[st]);  // short stage: the consumers load it
                    }
                }
                __syncwarp();
            }
        } else {
            // --------------------------------------------------- consumers
            const int g = warp % p.Hkv;      // KV head
            const int j = warp / p.Hkv;      // 16-token subset of every stage
            const int gq = lane >> 2;        // fragment row: query head of the group
            const int t = lane & 3;

            uint32_t qa[D / 16][2];
            if (gq < G) {
                const __nv_bfloat16 *qr = static_cast<const __nv_bfloat16 *>(p.q) +
                                          ((int64_t)b * p.Hq + (int64_t)g * G + gq) * D;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    qa[kk][0] = *reinterpret_cast<const uint32_t *>(qr + 16 * kk + 2 * t);
                    qa[kk][1] = *reinterpret_cast<const uint32_t *>(qr + 16 * kk + 8 + 2 * t);
                }
            } else {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) qa[kk][0] = qa[kk][1] = 0u;
            }
            float o[D / 8][4];
#pragma unroll
            for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
            float m = -INFINITY, l = 0.f;
            const int tok0 = j * kTokPerWarp;
            // ldmatrix row addresses (byte offsets inside a box) and the swizzle
            // term of each lane: S reads K rows tok0 + 8*(mat>>1) + rr, P.V reads
            // V rows tok0 + 8*(mat&1) + rr; row R keeps chunk c at c ^ (R & 7)
            const int mat = lane >> 3, rr = lane & 7;
            const uint32_t rowS = (uint32_t)(g * ST + tok0 + 8 * (mat >> 1) + rr) * 128u;
            const uint32_t xs = (uint32_t)((mat & 1) ^ rr);
            const uint32_t rowP = (uint32_t)(g * ST + tok0 + 8 * (mat & 1) + rr) * 128u;
            const uint32_t xp = (uint32_t)((mat >> 1) ^ rr);

            for (int i = 0; i < n_st; ++i) {
                const uint32_t itg = it + i;
                const int st = (int)(itg % p.stages);
                const uint32_t ph = (itg / p.stages) & 1u;
                if (!__all_sync(0xffffffffu, mbar_wait(&full[st], ph, &g_status_decode))) return;
                const uint32_t kst = sbase + (uint32_t)st * kStage;
                const uint32_t vst = kst + KB * kBox;
                const int64_t base_tok = (int64_t)i * ST + tok0;
                const int cnt = (int)min((int64_t)ST, n_tok - (int64_t)i * ST);
                if (cnt < ST) {
                    // short stage: this warp's 16 rows of head g, valid ones from
                    // global memory, the rest zero (0-weight rows then add exact zeros)
                    const int64_t r = row0 + (int64_t)i * ST;
                    for (int idx = lane; idx < kTokPerWarp * kChunks; idx += 32) {
                        const int lt = tok0 + idx / kChunks, ch = idx % kChunks;
                        const uint32_t R = (uint32_t)(g * ST + lt);
                        const uint32_t off = (uint32_t)(ch >> 3) * kBox + R * 128u +
                                             ((((uint32_t)ch & 7u) ^ (R & 7u)) << 4);
                        uint4 kv = make_uint4(0u, 0u, 0u, 0u), vv = kv;
                        if (lt < cnt) {
                            const int64_t e = ((r + lt) * p.Hkv + g) * D + ch * 8;
                            kv = *reinterpret_cast<const uint4 *>(kg + e);
                            vv = *reinterpret_cast<const uint4 *>(vg + e);
                        }
                        *reinterpret_cast<uint4 *>(smem + (kst - sbase) + off) = kv;
                        *reinterpret_cast<uint4 *>(smem + (vst - sbase) + off) = vv;
                    }
                    // these generic-proxy writes precede the copy engine's next
                    // writes into this stage
                    fence_proxy_async_smem();
                    __syncwarp();
                }

                float sc[2][4];
#pragma unroll
                for (int n = 0; n < 2; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kst + (uint32_t)(kk >> 2) * kBox + rowS + (((uint32_t)((kk & 3) << 1) ^ xs) << 4),
                            b0, b1, b2, b3);
                    mma_16816(sc[0], qa[kk][0], qa[kk][1], b0, b1);
                    mma_16816(sc[1], qa[kk][0], qa[kk][1], b2, b3);
                }
                float pv[2][2];
                float mx = -INFINITY;
#pragma unroll
                for (int n = 0; n < 2; ++n) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int lt = 8 * n + 2 * t + e;
                        const int64_t tok = base_tok + lt;
                        const float v = tok < n_tok ? sc[n][e] * p.scale_log2 : -INFINITY;
                        pv[n][e] = v;
                        mx = fmaxf(mx, v);
                    }
                }
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                if (mx > m + 8.f) {
                    // move the reference max only when it grows by more than 2^8
                    const float alpha = (m == -INFINITY) ? 0.f : ex2f(m - mx);
                    m = mx;
                    l *= alpha;
#pragma unroll
                    for (int n = 0; n < D / 8; ++n) {
                        o[n][0] *= alpha;
                        o[n][1] *= alpha;
                    }
                }
                const float neg_m = (m == -INFINITY) ? 0.f : -m;
                const float p00 = ex2f(pv[0][0] + neg_m), p01 = ex2f(pv[0][1] + neg_m);
                const float p10 = ex2f(pv[1][0] + neg_m), p11 = ex2f(pv[1][1] + neg_m);
                l += (p00 + p01) + (p10 + p11);
                const uint32_t a0 = pack2_bf16(p00, p01);
                const uint32_t a2 = pack2_bf16(p10, p11);
#pragma unroll
                for (int n = 0; n < D / 8; n += 2) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vst + (uint32_t)(n >> 3) * kBox + rowP + ((((uint32_t)n & 7u) ^ xp) << 4),
                              b0, b1, b2, b3);
                    mma_16816(o[n], a0, a2, b0, b1);
                    mma_16816(o[n + 1], a0, a2, b2, b3);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            }

            // l over the quad of lanes that share a row; o columns are disjoint
            l += __shfl_xor_sync(0xffffffffu, l, 1);
            l += __shfl_xor_sync(0xffffffffu, l, 2);
            const int64_t entry = ((int64_t)b * p.n_split + s) * p.sub + j;
            if (gq < G) {
                const int64_t hq = (int64_t)g * G + gq;
                float *dst = p.ws_o + (entry * p.Hq + hq) * D;
#pragma unroll
                for (int n = 0; n < D / 8; ++n)
                    *reinterpret_cast<float2 *>(dst + 8 * n + 2 * t) = make_float2(o[n][0], o[n][1]);
                if (t == 0) {
                    p.ws_ml[(entry * p.Hq + hq) * 2 + 0] = m;
                    p.ws_ml[(entry * p.Hq + hq) * 2 + 1] = l;
                }
            }
        }
        it += (uint32_t)n_st;
    }
    if (warp == kConsumerWarps && lane == 0) producer_drain(full, it, p.stages);
}

// ---------------------------------------------------------------------------
// Decode over an 8-bit cache (D = 128).  A cache row holds the Hkv x 128 int8
// codes of one token, then its Hkv fp32 scales (padded to 16 bytes); a value
// is code * scale.  A stage arrives as two 16 KB TMA boxes of codes ([head]
// [token] rows of 128 bytes, 128-byte swizzle) and two small boxes of the
// stage's scales -- half the bytes of the bf16 cache.
//
// The tensor-core tiles read the codes where the TMA put them, with the
// stage's 16 tokens of a head as the 16 MMA rows and the group's query heads
// as the 8 columns (transposed against the bf16 kernel, so no row of an MMA
// is padding when G < 16):
//  * S^T = K q^T is an integer MMA (m16n8k32, s8 x s8 -> s32) straight on the
//    K codes.  q is held as 15-bit fixed point per head (q ~ s_q * x, |x| <=
//    16256) split into two int8 parts x = 128 hi + lo, so S^T = 128 K hi^T +
//    K lo^T exactly in int32; the fixed-point step of q is 2^-14 of its
//    largest element, far below bf16's own rounding of q.  The K scale, s_q
//    and the softmax scale multiply the int32 result.
//  * O^T += V^T P^T is an fp16 MMA: V's codes are turned into fp16 in
//    registers (exact: the byte goes under the exponent of 1024 and 1152 is
//    subtracted), P^T comes from the S^T accumulators by one register
//    transpose (movmatrix) and carries each token's V scale.
// A stage that a sequence's end cuts short is copied by each warp from
// global memory into its own rows of the stage, zero-filled past the end.
constexpr int kI8Stages = 6;

struct DecodeI8Params {
    DecodeKParams k;
    int64_t row_bytes;   // bytes per cache row
    int32_t scale_off;   // byte offset of the scales within a row
    int32_t scale_bytes; // padded bytes of the scales per row
};

YOCO_DEV void mma_16816_f16_t(float *c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                              uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
YOCO_DEV void mma_16832_s8(int *c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
YOCO_DEV uint32_t movmatrix_t(uint32_t x) {
    uint32_t r;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
    return r;
}
YOCO_DEV uint32_t pack2_f16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
// Four int8 codes of a transposed ldmatrix word (bytes: token 2t at dims 2g,
// 2g+1, then token 2t+1 at dims 2g, 2g+1) -> fp16x2 (token 2t, token 2t+1) of
// dim 2g (even) and of dim 2g+1 (odd), exactly.
YOCO_DEV void i8t_to_f16(uint32_t w, uint32_t &even, uint32_t &odd) {
    const uint32_t u = w ^ 0x80808080u;  // code + 128, as unsigned bytes
    const uint32_t bias = 0x64806480u;   // fp16 1152 = 1024 + 128, twice
    const uint32_t a = __byte_perm(u, 0x64646464u, 0x4240);
    const uint32_t b = __byte_perm(u, 0x64646464u, 0x4341);
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(even) : "r"(a), "r"(bias));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(odd) : "r"(b), "r"(bias));
}
// four int8 values -> one word (byte i = v[i])
YOCO_DEV uint32_t pack_s8x4(float v0, float v1, float v2, float v3) {
    return ((uint32_t)(int)v0 & 0xffu) | (((uint32_t)(int)v1 & 0xffu) << 8) | (((uint32_t)(int)v2 & 0xffu) << 16) |
           (((uint32_t)(int)v3 & 0xffu) << 24);
}

template <int G>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    decode_i8_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vs,
                     const DecodeI8Params pi) {
    static_assert(G >= 1 && G <= 8, "the query heads of a group are the 8 columns of an MMA");
    pdl_trigger();
    pdl_wait();
    if (*(volatile unsigned int *)&g_status_decode & kStatusTimeout) return;  // an earlier CTA timed out
    constexpr int D = 128;
    constexpr uint32_t kBox = kRowsPerStage * 128;  // one code box: 128 rows of 128 bytes
    const DecodeKParams &p = pi.k;
    const int ST = (int)p.stage_tokens;
    const uint32_t sbox = (uint32_t)(ST * pi.scale_bytes);             // one scale box
    const uint32_t stage_bytes = 2 * kBox + ((2 * sbox + 1023u) & ~1023u);
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char *smem = smem_raw + (sbase - raw);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)kI8Stages * stage_bytes);
    uint64_t *empty = full + kI8Stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kI8Stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();

    const unsigned char *kg = static_cast<const unsigned char *>(p.k);
    const unsigned char *vg = static_cast<const unsigned char *>(p.v);
    uint32_t it = 0;

    for (int64_t u = blockIdx.x;; u += gridDim.x) {
        int b;
        int64_t s;
        if (!find_unit(p, u, &b, &s)) break;
        const int64_t len = (int64_t)p.seq_len[b];
        const int64_t t0 = s * p.split;
        const int64_t n_tok = min(p.split, len - t0);
        const int64_t row0 = p.seq_start[b] + t0;
        const int n_st = (int)((n_tok + ST - 1) / ST);

        if (warp == kConsumerWarps) {
            // ---------------------------------------------------- producer
            for (int i = 0; i < n_st; ++i) {
                const uint32_t itg = it + i;
                const int st = (int)(itg % kI8Stages);
                const uint32_t ph = (itg / kI8Stages) & 1u;
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ph ^ 1u, &g_status_decode))) {
                    if (lane == 0) producer_drain(full, it + i, kI8Stages);
                    return;
                }
                const int64_t r = row0 + (int64_t)i * ST;
                if (lane == 0) {
                    if (n_tok - (int64_t)i * ST >= ST) {
                        const uint32_t dst = sbase + (uint32_t)st * stage_bytes;
                        mbar_arrive_expect_tx(&full[st], 2 * kBox + 2 * sbox);
                        tc::tma_load_4d(dst, &tm_k, 0, (int)r, 0, 0, &full[st]);
                        tc::tma_load_4d(dst + kBox, &tm_v, 0, (int)r, 0, 0, &full[st]);
                        tc::tma_load_4d(dst + 2 * kBox, &tm_ks, 0, (int)r, 0, 0, &full[st]);
                        tc::tma_load_4d(dst + 2 * kBox + sbox, &tm_vs, 0, (int)r, 0, 0, &full[st]);
                    } else {
                        mbar_arrive(&full[st]);  // short stage: the consumers load it
                    }
                }
                __syncwarp();
            }
        } else {
            // --------------------------------------------------- consumers
            const int kvh = warp % p.Hkv;    // KV head
            const int j = warp / p.Hkv;      // 16-token subset of every stage
            const int gq = lane >> 2;        // S^T row (token) / P^T column (query head)
            const int t = lane & 3;
            const int tok0 = j * kTokPerWarp;

            // q of head gq as two int8 parts (B operand: dims 32kb + 4t.. and
            // 32kb + 16 + 4t..), and per head column 2t + e the factor s_q *
            // softmax scale * log2(e)
            uint32_t qh[4][2], ql[4][2];
            float qs[2];
            {
                float x[4][2][4];
                float amax = 0.f;
#pragma unroll
                for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        if (gq < G) {
                            const __nv_bfloat16 *qr = static_cast<const __nv_bfloat16 *>(p.q) +
                                                      ((int64_t)b * p.Hq + (int64_t)kvh * G + gq) * D +
                                                      32 * kb + 16 * hf + 4 * t;
                            const uint2 w = *reinterpret_cast<const uint2 *>(qr);
                            x[kb][hf][0] = __uint_as_float(w.x << 16);
                            x[kb][hf][1] = __uint_as_float(w.x & 0xffff0000u);
                            x[kb][hf][2] = __uint_as_float(w.y << 16);
                            x[kb][hf][3] = __uint_as_float(w.y & 0xffff0000u);
                        } else {
                            x[kb][hf][0] = x[kb][hf][1] = x[kb][hf][2] = x[kb][hf][3] = 0.f;
                        }
#pragma unroll
                        for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fabsf(x[kb][hf][i]));
                    }
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
                // the split below (x = rint(q * 16256 / amax), hi = rint(x / 128),
                // lo = x - 128 hi) is restated in float32 by tests/test_i8_q_split.py,
                // which checks the int8 ranges, the exact reconstruction and the
                // half-step bound; keep the two in step
                const float inv = amax > 0.f ? 16256.f / amax : 0.f;
#pragma unroll
                for (int kb = 0; kb < 4; ++kb)
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        float hi[4], lo[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float xi = fminf(fmaxf(rintf(x[kb][hf][i] * inv), -16256.f), 16256.f);
                            hi[i] = rintf(xi * (1.f / 128.f));
                            lo[i] = xi - 128.f * hi[i];
                        }
                        qh[kb][hf] = pack_s8x4(hi[0], hi[1], hi[2], hi[3]);
                        ql[kb][hf] = pack_s8x4(lo[0], lo[1], lo[2], lo[3]);
                    }
                const float sq = amax * (1.f / 16256.f);
                qs[0] = __shfl_sync(0xffffffffu, sq, 8 * t) * p.scale_log2;
                qs[1] = __shfl_sync(0xffffffffu, sq, 8 * t + 4) * p.scale_log2;
            }
            float oe[4][4], oo[4][4];  // O^T of dims 32c + 2g (+16) and 32c + 2g + 1 (+16)
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int i = 0; i < 4; ++i) oe[c][i] = oo[c][i] = 0.f;
            float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
            // ldmatrix rows of this lane: K (matrix mi: tokens 8(mi&1).., 16-byte
            // chunk mi>>1 of a 32-dim block), V (tokens 8(mi>>1).., chunk mi&1)
            const int mi = lane >> 3, rr = lane & 7;
            const uint32_t Rk = (uint32_t)(kvh * ST + tok0 + 8 * (mi & 1) + rr);
            const uint32_t Rv = (uint32_t)(kvh * ST + tok0 + 8 * (mi >> 1) + rr);

            for (int i = 0; i < n_st; ++i) {
                const uint32_t itg = it + i;
                const int st = (int)(itg % kI8Stages);
                const uint32_t ph = (itg / kI8Stages) & 1u;
                if (!__all_sync(0xffffffffu, mbar_wait(&full[st], ph, &g_status_decode))) return;
                unsigned char *stg = smem + (size_t)st * stage_bytes;
                const uint32_t stg_s = sbase + (uint32_t)st * stage_bytes;
                const int64_t base_tok = (int64_t)i * ST + tok0;
                const int cnt = (int)min((int64_t)ST, n_tok - (int64_t)i * ST);
                const int64_t r = row0 + (int64_t)i * ST;
                float ks[2], vs[2];  // scales of tokens gq and gq + 8
                if (cnt == ST) {
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {
                        const int lt = tok0 + gq + 8 * h8;
                        ks[h8] = *reinterpret_cast<const float *>(stg + 2 * kBox + lt * pi.scale_bytes + kvh * 4);
                        vs[h8] = *reinterpret_cast<const float *>(stg + 2 * kBox + sbox + lt * pi.scale_bytes + kvh * 4);
                    }
                } else {
                    // short stage: this warp's 16 rows of K and V codes into
                    // their swizzled places, zeros past the end
#pragma unroll
                    for (int c8 = 0; c8 < 8; ++c8) {
                        const int idx = c8 * 32 + lane;  // 0..255
                        const int tsr = idx >> 7, lt = (idx >> 3) & 15, ch = idx & 7;
                        uint4 w = make_uint4(0u, 0u, 0u, 0u);
                        if (tok0 + lt < cnt)
                            w = *reinterpret_cast<const uint4 *>((tsr ? vg : kg) + (r + tok0 + lt) * pi.row_bytes +
                                                                 kvh * D + ch * 16);
                        const uint32_t R = (uint32_t)(kvh * ST + tok0 + lt);
                        *reinterpret_cast<uint4 *>(stg + tsr * kBox + R * 128u + ((ch ^ (R & 7u)) << 4)) = w;
                    }
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {
                        const int lt = tok0 + gq + 8 * h8;
                        ks[h8] = vs[h8] = 0.f;
                        if (lt < cnt) {
                            const int64_t row = r + lt;
                            ks[h8] = *reinterpret_cast<const float *>(kg + row * pi.row_bytes + pi.scale_off + kvh * 4);
                            vs[h8] = *reinterpret_cast<const float *>(vg + row * pi.row_bytes + pi.scale_off + kvh * 4);
                        }
                    }
                    fence_proxy_async_smem();  // before the next TMA write into this stage
                    __syncwarp();
                }
                uint32_t kr[4][4], vr[4][4];
#pragma unroll
                for (int kb = 0; kb < 4; ++kb)
                    ldsm_x4(stg_s + Rk * 128u + ((((uint32_t)(2 * kb + (mi >> 1))) ^ (Rk & 7u)) << 4), kr[kb][0],
                            kr[kb][1], kr[kb][2], kr[kb][3]);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    ldsm_x4_t(stg_s + kBox + Rv * 128u + ((((uint32_t)(2 * c + (mi & 1))) ^ (Rv & 7u)) << 4), vr[c][0],
                              vr[c][1], vr[c][2], vr[c][3]);
                // S^T (16 tokens x 8 heads) in int32: hi and lo parts of q
                int ah[4] = {0, 0, 0, 0}, al[4] = {0, 0, 0, 0};
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    mma_16832_s8(ah, kr[kb][0], kr[kb][1], kr[kb][2], kr[kb][3], qh[kb][0], qh[kb][1]);
                    mma_16832_s8(al, kr[kb][0], kr[kb][1], kr[kb][2], kr[kb][3], ql[kb][0], ql[kb][1]);
                }
                // scores (log2 domain): element 2 h8 + e = token gq + 8 h8, head 2t + e
                float sv[4];
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8) {
                    const int64_t tok = base_tok + gq + 8 * h8;
                    const bool vld = tok < n_tok;
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float acc = (float)(128 * ah[2 * h8 + e] + al[2 * h8 + e]);
                        sv[2 * h8 + e] = vld ? acc * ks[h8] * qs[e] : -INFINITY;
                    }
                }
                float pr[4];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float mx = fmaxf(sv[e], sv[2 + e]);
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                    if (mx > m[e] + 8.f) {
                        const float alpha = (m[e] == -INFINITY) ? 0.f : ex2f(m[e] - mx);
                        m[e] = mx;
                        l[e] *= alpha;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            oe[c][e] *= alpha;
                            oe[c][2 + e] *= alpha;
                            oo[c][e] *= alpha;
                            oo[c][2 + e] *= alpha;
                        }
                    }
                    const float neg_m = (m[e] == -INFINITY) ? 0.f : -m[e];
                    pr[e] = ex2f(sv[e] + neg_m);
                    pr[2 + e] = ex2f(sv[2 + e] + neg_m);
                    l[e] += pr[e] + pr[2 + e];
                }
                // P^T with each token's V scale: transpose the [token][head]
                // fp16 pairs into the B fragments (head gq; tokens 2t, 2t+1 and
                // 2t+8, 2t+9)
                const uint32_t b0 = movmatrix_t(pack2_f16(pr[0] * vs[0], pr[1] * vs[0]));
                const uint32_t b1 = movmatrix_t(pack2_f16(pr[2] * vs[1], pr[3] * vs[1]));
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t e0, o0, e1, o1, e2, o2, e3, o3;
                    i8t_to_f16(vr[c][0], e0, o0);
                    i8t_to_f16(vr[c][1], e1, o1);
                    i8t_to_f16(vr[c][2], e2, o2);
                    i8t_to_f16(vr[c][3], e3, o3);
                    mma_16816_f16_t(oe[c], e0, e1, e2, e3, b0, b1);
                    mma_16816_f16_t(oo[c], o0, o1, o2, o3, b0, b1);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            }

#pragma unroll
            for (int e = 0; e < 2; ++e) {
                l[e] += __shfl_xor_sync(0xffffffffu, l[e], 4);
                l[e] += __shfl_xor_sync(0xffffffffu, l[e], 8);
                l[e] += __shfl_xor_sync(0xffffffffu, l[e], 16);
            }
            const int64_t entry = ((int64_t)b * p.n_split + s) * p.sub + j;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int hh = 2 * t + e;
                if (hh < G) {
                    const int64_t hq = (int64_t)kvh * G + hh;
                    float *dst = p.ws_o + (entry * p.Hq + hq) * D;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        *reinterpret_cast<float2 *>(dst + 32 * c + 2 * gq) = make_float2(oe[c][e], oo[c][e]);
                        *reinterpret_cast<float2 *>(dst + 32 * c + 16 + 2 * gq) = make_float2(oe[c][2 + e], oo[c][2 + e]);
                    }
                    if (gq == 0) {
                        p.ws_ml[(entry * p.Hq + hq) * 2 + 0] = m[e];
                        p.ws_ml[(entry * p.Hq + hq) * 2 + 1] = l[e];
                    }
                }
            }
        }
        it += (uint32_t)n_st;
    }
    if (warp == kConsumerWarps && lane == 0) producer_drain(full, it, kI8Stages);
}

// 8-bit quantisation of K and V rows: one warp per (token, head, tensor);
// absmax over the head's D values, scale = absmax / 127, code = nearest
// integer (half to even) of x / scale, all in fp32 with IEEE division.
template <typename T, int D>
__global__ void kv_quantize_i8_kernel(const T *k, const T *v, int64_t n, int Hkv, const int64_t *dst_rows,
                                      unsigned char *kq, unsigned char *vq, int64_t row_bytes) {
    constexpr int PER = D / 32;
    const int64_t wid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (wid >= n * Hkv * 2) return;
    const int tensor = (int)(wid & 1);
    const int64_t th = wid >> 1, tok = th / Hkv;
    const int h = (int)(th % Hkv);
    const T *src = (tensor ? v : k) + (tok * Hkv + h) * D + lane * PER;
    float x[PER];
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        x[e] = to_f32(src[e]);
        amax = fmaxf(amax, fabsf(x[e]));
    }
    amax = warp_max(amax);
    const float scale = __fdiv_rn(amax, 127.f);
    const int64_t row = dst_rows ? dst_rows[tok] : tok;
    unsigned char *dst = (tensor ? vq : kq) + row * row_bytes;
    uint32_t packed = 0;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        int c = scale > 0.f ? __float2int_rn(__fdiv_rn(x[e], scale)) : 0;
        c = max(-127, min(127, c));
        packed |= (uint32_t)(c & 0xff) << (8 * e);
    }
    if (PER == 4)
        *reinterpret_cast<uint32_t *>(dst + h * D + lane * 4) = packed;
    else
        *reinterpret_cast<uint16_t *>(dst + h * D + lane * 2) = (uint16_t)packed;
    if (lane == 0) {
        reinterpret_cast<float *>(dst + (int64_t)Hkv * D)[h] = scale;
        if (h == 0)  // zero the padding after the scales
            for (int64_t z = (int64_t)Hkv * (D + 4); z < row_bytes; ++z) dst[z] = 0;
    }
}

// Split merge: one CTA of kMergeWarps warps per (sequence, query head).  Warp
// w takes the partial entries w, w + kMergeWarps, ... (each a 512-byte row
// read by the whole warp), four at a time in flight, and keeps its own
// running max, sum and weighted row (online rescaling); the warps' (max, sum,
// row) are then combined through shared memory.  An earlier split of the
// entries in runs of 32 per warp left all but one warp idle at the barrier
// when a sequence had 32 partials (a 4 x 1024 sliding-window ring: 21 us per
// merge under the profiler); with one warp per (sequence, head), a single
// long sequence left the merge with a few dozen warps to read hundreds of
// partial rows each.
constexpr int kMergeWarps = 8;

// The sliding-window decode's new token: its K/V (already blended) and query,
// merged as one more partial, then written into the ring (NULL k_new: cross
// decode, nothing to add).
template <typename T>
struct MergeNewToken {
    const T *q, *k_new, *v_new;
    const int64_t *pos;
    T *ring_k, *ring_v;
    int32_t *slot_pos;
    int32_t Hkv;
    float scale_log2;
};

template <typename T, int D>
__global__ void __launch_bounds__(32 * kMergeWarps) decode_merge_kernel(
    const float *ws_o, const float *ws_ml, const int64_t *seq_start, const int32_t *seq_len, int32_t window,
    int32_t B, int32_t Hq, int64_t max_len, int64_t cache_rows, int64_t split, int64_t n_split, int32_t sub,
    T *o, float *lse, const MergeNewToken<T> nt) {
    constexpr int DPL = D / 32;
    __shared__ float s_m[kMergeWarps], s_l[kMergeWarps];
    __shared__ float s_acc[kMergeWarps][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = (int)(blockIdx.x / Hq), h = (int)(blockIdx.x % Hq);
    pdl_trigger();
    pdl_wait();
    const int64_t len = seq_len ? (int64_t)seq_len[b] : (int64_t)window;
    // the split kernel gave an out-of-range sequence no units; its output
    // becomes 0 (lse -inf) and the status word records it once
    const bool ok = !seq_len || sched::decode_seq_ok(seq_start[b], len, max_len, cache_rows);
    if (!ok && h == 0 && threadIdx.x == 0) atomicOr(&g_status_decode, kStatusBadSequence);
    const int64_t n_s = ok ? sched::decode_units(len, split, n_split) : 0;
    const int64_t n_e = n_s * sub;
    const int64_t e0 = (int64_t)b * n_split * sub;

    // warp w merges partials w, w + 8, ... with an online max (lane l holds
    // dims l, l + 32, ...), four partials' loads in flight at a time
    float M = -INFINITY, Lp = 0.f;
    float acc[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
    for (int64_t c = warp; c < n_e; c += 4 * kMergeWarps) {
        float me[4], le[4], ov[4][DPL];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int64_t e = c + (int64_t)u * kMergeWarps;
            me[u] = -INFINITY;
            le[u] = 0.f;
            if (e < n_e) {
                const float *ml = ws_ml + ((e0 + e) * Hq + h) * 2;
                me[u] = ml[0];
                le[u] = ml[1];
                const float *src = ws_o + ((e0 + e) * Hq + h) * D + lane;
#pragma unroll
                for (int i = 0; i < DPL; ++i) ov[u][i] = src[32 * i];
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (me[u] == -INFINITY) continue;   // an empty partial (or none)
            const float mn = fmaxf(M, me[u]);
            const float fo = (M == -INFINITY) ? 0.f : exp2f(M - mn), fe = exp2f(me[u] - mn);
            Lp = fmaf(Lp, fo, le[u] * fe);
#pragma unroll
            for (int i = 0; i < DPL; ++i) acc[i] = fmaf(acc[i], fo, ov[u][i] * fe);
            M = mn;
        }
    }
    const float L = Lp;   // the same in every lane of the warp
    if (lane == 0) {
        s_m[warp] = M;
        s_l[warp] = L;
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) s_acc[warp][lane + 32 * i] = acc[i];
    __syncthreads();
    if (nt.k_new && h == 0 && warp >= 1) {
        // the new token into the ring (the split kernel has read the ring;
        // nothing else in this launch reads it): slot pos mod window
        const int64_t p = nt.pos[b];
        const int64_t slot = ((p % window) + window) % window;
        const int64_t re = (int64_t)nt.Hkv * D;
        T *dk = nt.ring_k + ((int64_t)b * window + slot) * re;
        T *dv = nt.ring_v + ((int64_t)b * window + slot) * re;
        for (int64_t e = threadIdx.x - 32; e < re; e += 32 * (kMergeWarps - 1)) {
            dk[e] = nt.k_new[(int64_t)b * re + e];
            dv[e] = nt.v_new[(int64_t)b * re + e];
        }
        if (threadIdx.x == 32) nt.slot_pos[(int64_t)b * window + slot] = (int32_t)p;
    }
    if (warp != 0) return;
    float Mg = -INFINITY;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) Mg = fmaxf(Mg, s_m[w]);
    // the new token's score (log2 domain) and value row, as one more partial
    float m_new = -INFINITY, v_row[DPL];
    if (nt.k_new) {
        const int g = h / (Hq / nt.Hkv);
        const T *qh = nt.q + ((int64_t)b * Hq + h) * D;
        const T *kn = nt.k_new + ((int64_t)b * nt.Hkv + g) * D;
        const T *vn = nt.v_new + ((int64_t)b * nt.Hkv + g) * D;
        float dot = 0.f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) {
            dot = fmaf(to_f32(qh[lane + 32 * i]), to_f32(kn[lane + 32 * i]), dot);
            v_row[i] = to_f32(vn[lane + 32 * i]);
        }
        m_new = warp_sum(dot) * nt.scale_log2;
        Mg = fmaxf(Mg, m_new);
    }
    float Lg = 0.f, out[DPL];
#pragma unroll
    for (int i = 0; i < DPL; ++i) out[i] = 0.f;
#pragma unroll
    for (int w = 0; w < kMergeWarps; ++w) {
        const float f = (s_m[w] == -INFINITY) ? 0.f : exp2f(s_m[w] - Mg);
        Lg = fmaf(s_l[w], f, Lg);
#pragma unroll
        for (int i = 0; i < DPL; ++i) out[i] = fmaf(s_acc[w][lane + 32 * i], f, out[i]);
    }
    if (nt.k_new) {
        const float f = exp2f(m_new - Mg);
        Lg += f;
#pragma unroll
        for (int i = 0; i < DPL; ++i) out[i] = fmaf(v_row[i], f, out[i]);
    }
    const float inv = Lg > 0.f ? 1.f / Lg : 0.f;
    T *dst = o + ((int64_t)b * Hq + h) * D;
#pragma unroll
    for (int i = 0; i < DPL; ++i) dst[lane + 32 * i] = from_f32<T>(out[i] * inv);
    if (lse && lane == 0) lse[(int64_t)b * Hq + h] = Lg > 0.f ? (Mg + log2f(Lg)) * kLn2 : -INFINITY;
}

bool make_decode_plan(int32_t B, int64_t max_len, int Hq, int Hkv, int D, int dtype,
                      DecodePlan *plan) {
    if (B < 0 || max_len < 1 || Hkv < 1 || kRowsPerStage % Hkv != 0 || Hkv > kConsumerWarps ||
        Hq % Hkv != 0)
        return false;
    DecodePlan pl;
    pl.stage_tokens = kRowsPerStage / Hkv;
    pl.sub = kConsumerWarps / Hkv;
    // Units: about kUnitBytes of K and V each, between one per SM and twelve
    // per SM (many units balance ragged batches; few keep a short decode from
    // paying per-unit overhead and a long merge), at least two pipeline
    // stages each, and at most two per SM for one sequence: the merge gives a
    // sequence one CTA per query head, which folds the sequence's partials
    // one after another.  A 16 x 64K-128K batch gets the maximum (~111 units
    // a sequence); a 1M-token sequence 296 units, two per CTA (1776 made its
    // merge ~0.1 ms of a 0.75 ms call); a 4 x 1024 sliding-window ring ~128
    // units of two stages, each CTA with its whole unit in flight; one
    // 32K-token sequence ~150 units.
    const int64_t total = (int64_t)std::max(B, 1) * max_len;
    const int64_t tok_bytes = 2 * (int64_t)Hkv * D * (int64_t)dtype_bytes(dtype);
    const int64_t target = std::min<int64_t>(kMaxUnits, std::max<int64_t>(kMinUnits, total * tok_bytes / kUnitBytes));
    const int64_t min_split = 2 * pl.stage_tokens;
    int64_t per = (total + target - 1) / target;
    per = ((per + pl.stage_tokens - 1) / pl.stage_tokens) * pl.stage_tokens;
    pl.split = std::max(per, min_split);
    const int64_t per_seq = (max_len + kMaxUnitsPerSeq - 1) / kMaxUnitsPerSeq;
    pl.split = std::max(pl.split, ((per_seq + pl.stage_tokens - 1) / pl.stage_tokens) * pl.stage_tokens);
    pl.n_split = (max_len + pl.split - 1) / pl.split;
    // a stage holds 128 token-head rows of K and of V; the bf16 kernel adds
    // 1 KB so that its swizzled stages can start on a 1024-byte boundary
    const size_t stage_bytes = 2 * (size_t)kRowsPerStage * D * dtype_bytes(dtype);
    // no deeper than a unit: a short unit's CTA then takes less shared memory
    // and fits on an SM beside the kernel before it (programmatic launch)
    pl.stages = (int)std::max<size_t>(1, std::min<size_t>(std::min<size_t>(dtype == kBF16 ? 6 : 4,
                                                                           (200 * 1024) / stage_bytes),
                                                          (size_t)(pl.split / pl.stage_tokens)));
    pl.smem_bytes = pl.stages * stage_bytes + 2 * pl.stages * sizeof(uint64_t) +
                    (dtype == kBF16 ? 1024 : 0);
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

// TMA view of a packed cache [rows, Hkv, D]: dimensions {D, token, head, 1},
// box {64, stage_tokens, Hkv, 1}.  The token extent is the caller's cache_rows,
// so a box can never read past the allocation (the kernel only asks for
// boxes inside a sequence whose rows it has checked against cache_rows).
static bool make_cache_map(CUtensorMap *m, const void *cache, int64_t cache_rows, int Hkv, int D,
                           int64_t stage_tokens) {
    const uint64_t row_bytes = (uint64_t)Hkv * D * 2;
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)cache_rows, (uint64_t)Hkv, 1};
    const uint64_t strides[3] = {row_bytes, (uint64_t)D * 2, row_bytes};
    const uint32_t box[4] = {64, (uint32_t)stage_tokens, (uint32_t)Hkv, 1};
    return encode_bf16_map_4d(m, cache, dims, strides, box);
}

template <int D, int G>
static cudaError_t launch_decode_tma(const DecodeArgs &a, const DecodePlan &pl, const DecodeKParams &p,
                                     int grid, cudaStream_t st) {
    CUtensorMap mk, mv;
    if (!make_cache_map(&mk, a.k, a.cache_rows, a.Hkv, D, p.stage_tokens) ||
        !make_cache_map(&mv, a.v, a.cache_rows, a.Hkv, D, p.stage_tokens))
        return cudaErrorNotSupported;
    auto kern = decode_tma_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem_bytes);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(grid), dim3(kDecodeThreads), pl.smem_bytes, st, mk, mv, p);
}

template <typename T, int D, int G>
static cudaError_t launch_decode_t(const DecodeArgs &a, const DecodePlan &pl, cudaStream_t st) {
    DecodeKParams p;
    p.q = a.q; p.k = a.k; p.v = a.v;
    p.seq_start = a.seq_start; p.seq_len = a.seq_len;
    p.slot_pos = a.slot_pos; p.pos = a.pos; p.window = a.window;
    p.B = a.B; p.Hkv = a.Hkv; p.Hq = a.Hq;
    p.cache_rows = a.cache_rows; p.max_len = a.max_len;
    p.stage_tokens = pl.stage_tokens; p.split = pl.split; p.n_split = pl.n_split;
    p.sub = pl.sub; p.stages = pl.stages;
    p.scale_log2 = a.scale * kLog2e;
    const size_t entries = (size_t)a.B * pl.n_split * pl.sub * a.Hq;
    p.ws_o = static_cast<float *>(a.ws);
    p.ws_ml = p.ws_o + entries * D;
    const int64_t units = (int64_t)a.B * pl.n_split;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(units, device_sm_count()));
    cudaError_t e;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        // the bf16 window decode runs in ring_decode.cu; this kernel reads the packed cache
        if (!a.seq_len || !a.seq_start) return cudaErrorNotSupported;
        e = launch_decode_tma<D, G>(a, pl, p, grid, st);
    } else {
        auto kern = decode_split_kernel<T, D, G>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.smem_bytes);
        if (e != cudaSuccess) return e;
        e = launch_pdl(kern, dim3(grid), dim3(kDecodeThreads), pl.smem_bytes, st, p);
    }
    note_launches(2);
    if (e != cudaSuccess) return e;
    const int mgrid = (int)((int64_t)a.B * a.Hq);
    MergeNewToken<T> nt = {};
    if (a.k_new) {
        nt.q = static_cast<const T *>(a.q);
        nt.k_new = static_cast<const T *>(a.k_new);
        nt.v_new = static_cast<const T *>(a.v_new);
        nt.pos = a.pos;
        nt.ring_k = static_cast<T *>(const_cast<void *>(a.k));
        nt.ring_v = static_cast<T *>(const_cast<void *>(a.v));
        nt.slot_pos = const_cast<int32_t *>(a.slot_pos);
        nt.Hkv = a.Hkv;
        nt.scale_log2 = a.scale * kLog2e;
    }
    return launch_pdl(decode_merge_kernel<T, D>, dim3(mgrid), dim3(32 * kMergeWarps), 0, st, p.ws_o, p.ws_ml,
                      a.seq_start, a.seq_len, a.window, a.B, a.Hq, a.max_len, a.cache_rows, pl.split, pl.n_split,
                      pl.sub, static_cast<T *>(a.o), a.lse, nt);
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

// ------------------------------------------------------------- 8-bit cache
// TMA views of an 8-bit cache: the codes as {128, token, head, 1} bytes (token
// stride row_bytes, head stride 128), box {128, stage_tokens, Hkv, 1} with the
// 128-byte swizzle; the scales as {scale_bytes, token, 1, 1} starting at the
// row's scale offset, box {scale_bytes, stage_tokens, 1, 1}.
static bool make_i8_maps(CUtensorMap *codes, CUtensorMap *scales, const void *cache, int64_t cache_rows, int Hkv,
                         int64_t ST) {
    const uint64_t rb = (uint64_t)i8_row_bytes(Hkv, 128);
    const uint64_t rows = (uint64_t)cache_rows;
    const uint64_t dims[4] = {128, rows, (uint64_t)Hkv, 1};
    const uint64_t strides[3] = {rb, 128, rb};
    const uint32_t box[4] = {128, (uint32_t)ST, (uint32_t)Hkv, 1};
    const uint64_t sdims[4] = {(uint64_t)i8_scale_bytes(Hkv), rows, 1, 1};
    const uint64_t sstrides[3] = {rb, rb, rb};
    const uint32_t sbox[4] = {(uint32_t)i8_scale_bytes(Hkv), (uint32_t)ST, 1, 1};
    const unsigned char *sp = static_cast<const unsigned char *>(cache) + (int64_t)Hkv * 128;
    return encode_map_4d(codes, cache, true, true, dims, strides, box) &&
           encode_map_4d(scales, sp, true, false, sdims, sstrides, sbox);
}

template <int G>
static cudaError_t launch_decode_i8_g(const DecodeArgs &a, const DecodePlan &pl, cudaStream_t st) {
    CUtensorMap mk, mks, mv, mvs;
    if (!make_i8_maps(&mk, &mks, a.k, a.cache_rows, a.Hkv, pl.stage_tokens) ||
        !make_i8_maps(&mv, &mvs, a.v, a.cache_rows, a.Hkv, pl.stage_tokens))
        return cudaErrorNotSupported;
    DecodeI8Params pi;
    DecodeKParams &p = pi.k;
    p.q = a.q; p.k = a.k; p.v = a.v;
    p.seq_start = a.seq_start; p.seq_len = a.seq_len;
    p.slot_pos = a.slot_pos; p.pos = a.pos; p.window = a.window;
    p.B = a.B; p.Hkv = a.Hkv; p.Hq = a.Hq;
    p.cache_rows = a.cache_rows; p.max_len = a.max_len;
    p.stage_tokens = pl.stage_tokens; p.split = pl.split; p.n_split = pl.n_split;
    p.sub = pl.sub; p.stages = kI8Stages;
    p.scale_log2 = a.scale * kLog2e;
    const size_t entries = (size_t)a.B * pl.n_split * pl.sub * a.Hq;
    p.ws_o = static_cast<float *>(a.ws);
    p.ws_ml = p.ws_o + entries * 128;
    pi.row_bytes = i8_row_bytes(a.Hkv, 128);
    pi.scale_off = a.Hkv * 128;
    pi.scale_bytes = (int32_t)i8_scale_bytes(a.Hkv);
    const uint32_t sbox = (uint32_t)(pl.stage_tokens * pi.scale_bytes);
    const size_t stage_bytes = 2 * (size_t)kRowsPerStage * 128 + ((2 * sbox + 1023u) & ~1023u);
    const size_t smem = 1024 + kI8Stages * stage_bytes + 2 * kI8Stages * sizeof(uint64_t);
    auto kern = decode_i8_kernel<G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t units = (int64_t)a.B * pl.n_split;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(units, device_sm_count()));
    note_launches(2);
    e = launch_pdl(kern, dim3(grid), dim3(kDecodeThreads), smem, st, mk, mv, mks, mvs, pi);
    if (e != cudaSuccess) return e;
    return launch_pdl(decode_merge_kernel<__nv_bfloat16, 128>, dim3((unsigned)((int64_t)a.B * a.Hq)),
                      dim3(32 * kMergeWarps), 0, st, p.ws_o, p.ws_ml, a.seq_start, a.seq_len, a.window, a.B,
                      a.Hq, a.max_len, a.cache_rows, pl.split, pl.n_split, pl.sub,
                      static_cast<__nv_bfloat16 *>(a.o), a.lse, MergeNewToken<__nv_bfloat16>{});
}

cudaError_t launch_decode_i8(const DecodeArgs &a, const DecodePlan &pl, cudaStream_t st) {
    if (a.B == 0) return cudaSuccess;
    if (a.D != 128 || a.dtype != kBF16) return cudaErrorNotSupported;
    switch (a.Hq / a.Hkv) {
        case 1: return launch_decode_i8_g<1>(a, pl, st);
        case 2: return launch_decode_i8_g<2>(a, pl, st);
        case 4: return launch_decode_i8_g<4>(a, pl, st);
        case 8: return launch_decode_i8_g<8>(a, pl, st);
    }
    return cudaErrorNotSupported;
}

cudaError_t launch_kv_quantize_i8(const void *k, const void *v, int64_t n, int Hkv, int D, int dtype,
                                  const int64_t *dst_rows, void *kq, void *vq, cudaStream_t st) {
    if (n == 0) return cudaSuccess;
    const int64_t warps = n * Hkv * 2;
    const int grid = (int)((warps + 7) / 8);
    const int64_t rb = i8_row_bytes(Hkv, D);
    unsigned char *kb = static_cast<unsigned char *>(kq), *vb = static_cast<unsigned char *>(vq);
    note_launches(1);
    if (dtype == kBF16) {
        if (D == 128)
            kv_quantize_i8_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(
                static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v), n, Hkv, dst_rows, kb, vb, rb);
        else
            kv_quantize_i8_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(
                static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(v), n, Hkv, dst_rows, kb, vb, rb);
    } else {
        if (D == 128)
            kv_quantize_i8_kernel<float, 128><<<grid, 256, 0, st>>>(static_cast<const float *>(k),
                                                                   static_cast<const float *>(v), n, Hkv, dst_rows, kb, vb, rb);
        else
            kv_quantize_i8_kernel<float, 64><<<grid, 256, 0, st>>>(static_cast<const float *>(k),
                                                                  static_cast<const float *>(v), n, Hkv, dst_rows, kb, vb, rb);
    }
    return cudaGetLastError();
}

// ------------------------------------------------------------- test probe
// Test-only: one thread waits, through the kernels' own bounded wait, on an
// mbarrier phase that nothing completes.  The wait gives up after its limit,
// records the timeout in the status word and returns: nothing faults, nothing
// hangs, and the context stays usable.
__global__ void wait_timeout_probe_kernel() {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &g_status_decode);  // phase 0 never completes
}

cudaError_t launch_wait_timeout_probe(cudaStream_t st) {
    note_launches(1);
    wait_timeout_probe_kernel<<<1, 32, 0, st>>>();
    return cudaGetLastError();
}

// ------------------------------------------------------------------ ring
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
