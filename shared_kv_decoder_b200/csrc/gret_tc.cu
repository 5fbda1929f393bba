// Gated retention chunkwise prefill on the sm_100a tensor cores (bf16 in,
// fp32 state and accumulation), D = 128.  The same computation as
// gret_prefill_kernel in gret.cu ("You Only Cache Once", paperlayer summary,
// section 3 "Gated Retention" and Appendix B; podcast transcript cue 16):
// per head, S_t = gamma_t S_{t-1} + scale k_t^T v_t and o_t = q_t S_t, taken
// in chunks of 128 tokens.  With c_r the running sum of log gamma over the
// chunk's rows 0..r (base-2 units here):
//   o_r   = sum_{u<=r} 2^{c_r - c_u} scale (q_r . k_u) v_u   +  2^{c_r} q_r S_prev
//   S_new = 2^{c_last} S_prev + sum_u K_w[u]^T v_u,  K_w[u] = 2^{c_last - c_u} scale k_u
// Every exponent is <= 0.
//
// The decayed scores reuse K_w: Q K_w^T = scale 2^{c_last - c_u} (q_r . k_u),
// so 2^{c_r - c_last} (Q K_w^T)[r][u] is the decayed score, one multiply per
// element instead of an exponential.  That needs 2^{c_last - c_u} and
// 2^{c_r - c_last} to stay normal fp32 / bf16 numbers: it is used when the
// chunk's total decay 2^{c_last} is at least 2^-60; a chunk that decays more
// takes the scores from Q K^T with one exponential per element.
//
// One CTA per (batch, head) walks the chunks in order.  TMEM (512 columns):
//   A/P [0,128)   the scores of the chunk, then the decayed, masked P (bf16, first 64)
//   O   [128,256) P V
//   X   [256,384) Q S_prev
//   S   [384,512) the fp32 state (row d = lane d)
// Shared memory (224 KB): Q, K, V (two buffers), K_w, S_prev rounded to bf16
// and laid out like a V tile for the cross term, and the bf16 output tile
// that the TMA stores.  The cross term's rounding is of the same order as the
// bf16 rounding of P in P V and of K_w in the update: an fp64 emulation of
// the chunk loop with every bf16 rounding of this kernel, scores from K_w
// included, gives rel-L2 2.9e-3 against the exact recurrence (2.3e-3 with a
// two-part bf16 split of S and exponentials for the scores); the state
// itself stays fp32 in TMEM.  The running log-decay sums live in registers and are exchanged
// by warp shuffles.
// Warp roles (352 threads):
//   warps 0-3  output: P, then o = O + 2^{c_r} X into the output tile (warp 0
//              lane 0 issues its TMA store)
//   warps 4-7  state: K_w; one pass over S that writes S_prev in bf16 for this
//              chunk's cross term and leaves 2^{c_last} S_prev in TMEM for the
//              update
//   warp 8     TMA: lane 0 Q tiles, lane 1 K tiles, lane 2 V tiles; each also
//              asks L2 for its next tile
//   warp 9     output MMAs: scores = Q K_w^T (or Q K^T); X = Q S_prev; O = P V
//   warp 10    state MMA: S += K_w^T V (A operand MN-major from the K_w tile)
// The recurrence S -> S' runs on warps 4-7 and 10 alone, so it never queues
// behind the output side's MMAs; the two sides meet at K_w (read by both
// MMAs), at the bf16 copy of S_prev (the cross term of a chunk must have read
// it before the next chunk's copy overwrites it) and at the K and V tiles.
// Every warp reads the gate logits of the next chunk while it works on this
// one.  Every mbarrier wait is bounded; a wait that gives up sets the status
// word, and all roles fall through to the common exit, which waits for
// issued copies and MMAs before freeing TMEM.
#include <cuda.h>

#include <algorithm>
#include <cstdint>

#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace yoco {

static __device__ unsigned int g_status_gret_tc;

namespace {

constexpr int kC = 128;            // chunk length
constexpr int kD = 128;            // head dim
constexpr int kThreads = 352;
constexpr uint32_t kBlk = 128 * 128;      // one [128 rows x 128 bytes] swizzled block
constexpr uint32_t kTile = 2 * kBlk;      // a [128, 128] bf16 tile (two 64-column blocks)
constexpr float kFoldMinLog2 = -60.f;     // smallest chunk decay (log2) that folds into K_w
constexpr int kMaxSuperchunks = 8;        // CTAs per sequence at most (see gret_superchunks)

enum Smem : uint32_t {
    kQ = 0,
    kK = kQ + kTile,
    kV0 = kK + kTile,
    kV1 = kV0 + kTile,
    kKw = kV1 + kTile,
    kSb = kKw + kTile,                    // S_prev in bf16
    kOt = kSb + kTile,                    // output tile
    kBars = kOt + kTile,
    kBytes = kBars + 256,
    kAlloc = kBytes + 1024,
};
static_assert(kAlloc <= 227 * 1024, "shared memory per block");

enum Bar {
    kQFull = 0,
    kKFull,
    kVFull,       // two: V buffers
    kQEmpty = kVFull + 2,  // the scores and the cross term done (Q and the bf16 S_prev free)
    kKEmpty,      // the scores done (commit) and K_w written (arrive): 2 arrivals
    kVEmpty,      // two: P V and the state update done (2 commits each)
    kAFull = kVEmpty + 2,  // the scores done (K_w free for the next chunk's)
    kPFull,       // P written (128 arrivals)
    kOFull,       // the cross term and P V done
    kOFree,       // O and X read out of TMEM (128 arrivals)
    kOStaged,     // the output tile written (128 arrivals)
    kOtFree,      // the previous output tile's store has read it
    kSReady,      // K_w, the bf16 S_prev and the decayed S in place (128 arrivals)
    kSUpdated,    // S += K_w^T V done
    kDrainO, kDrainS,
    kNumBars
};
// after the barriers: TMEM address, abort flag, fold flag of the chunk (two)
constexpr uint32_t kMisc = kBars + kNumBars * 8;
static_assert(kNumBars * 8 + 16 <= 256, "barrier area");

struct GretTcParams {
    const float *g;
    float *state;
    int32_t B, H;
    int64_t T;
    float lg_scale;   // log2(e) / tau
    float scale;
    int32_t n_chunks;     // chunks of the whole sequence
    // Superchunks (see launch_gret_prefill_tc): each sequence's chunks split
    // into n_sc contiguous runs of sc_chunks, one CTA each.  n_sc = 1: one CTA
    // walks the whole sequence.
    int32_t n_sc, sc_chunks;
    int32_t state_only;   // this launch forms superchunks 0 .. n_sc - 2's state contributions
    // scratch of a split launch, per sequence: n_sc [D, D] fp32 slots --
    // slot s < n_sc - 1: superchunk s's final state from a zero start; slot
    // n_sc - 1: a copy of the initial state (zeros without one), so that no
    // CTA of the output pass reads `state`, which the last superchunk
    // overwrites -- then n_sc floats, log2 of each superchunk's total decay
    float *sc_state;
    float *sc_log2decay;
};

YOCO_DEV bool wait1(uint64_t *bar, uint32_t parity) { return mbar_wait(bar, parity, &g_status_gret_tc); }
YOCO_DEV bool waitw(uint64_t *bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, &g_status_gret_tc));
}

// base-2 log decay of one token: log2(sigmoid(g)) / tau
YOCO_DEV float log2_decay(float g, float lg_scale) {
    return (fminf(g, 0.f) - log1pf(expf(-fabsf(g)))) * lg_scale;
}

// byte offset of element (row, col) of a [128, 128] bf16 tile in the 128-byte
// swizzled layout of a TMA tile (two blocks of 64 columns)
YOCO_DEV uint32_t sw_off(int row, int col) {
    return (uint32_t)(col >> 6) * kBlk + (uint32_t)row * 128u +
           ((((uint32_t)(col & 63) >> 3) ^ ((uint32_t)row & 7u)) << 4) + (uint32_t)(col & 7) * 2u;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    gret_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const GretTcParams p) {
    if (*(volatile unsigned int *)&g_status_gret_tc) return;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sb = smem_raw + (base - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sb + kBars);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sb + kMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sb + kMisc + 4);
    volatile int *fold_flag = reinterpret_cast<volatile int *>(sb + kMisc + 8);  // [2]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // CTA -> (sequence, superchunk); the state-only launch covers superchunks
    // 0 .. n_sc - 2 (the last one's contribution feeds nothing)
    const bool so = p.state_only != 0;
    const int per_seq = so ? p.n_sc - 1 : p.n_sc;
    const int bh = blockIdx.x / per_seq, sc = blockIdx.x % per_seq;
    const int b = bh / p.H, h = bh % p.H;
    const int j0 = sc * p.sc_chunks;                         // first chunk of this CTA
    const int NC = min(p.sc_chunks, p.n_chunks - j0);        // chunks of this CTA

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            int cnt = 1;
            if (i == kPFull || i == kOFree || i == kOStaged || i == kSReady) cnt = 128;
            // K and V buffers are released by the output side and the state
            // side; a state-only launch has no output side
            if (!so && (i == kKEmpty || i == kVEmpty || i == kVEmpty + 1)) cnt = 2;
            mbar_init(&bars[i], cnt);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tA = tmem, tO = tmem + 128, tX = tmem + 256, tS = tmem + 384;

    if (warp == 8) {
        // ------------------------------------------------------ TMA producer
        // lane 0: Q, lane 1: K, lane 2: V (two buffers)
        if (lane < 3 && !(so && lane == 0)) {   // a state-only launch reads no Q
            const CUtensorMap *map = lane == 0 ? &tm_q : lane == 1 ? &tm_k : &tm_v;
            const int nb = lane == 2 ? 2 : 1;
            const uint32_t dst0 = base + (lane == 0 ? kQ : lane == 1 ? kK : kV0);
            uint64_t *full = &bars[lane == 0 ? kQFull : lane == 1 ? kKFull : kVFull];
            uint64_t *empty = &bars[lane == 0 ? kQEmpty : lane == 1 ? kKEmpty : kVEmpty];
            int j = 0;
            for (; j < NC && !*abort_flag; ++j) {
                const int bi = j % nb, use = j / nb;
                if (use > 0 && !wait1(&empty[bi], (use - 1) & 1)) { *abort_flag = 1; break; }
                mbar_arrive_expect_tx(&full[bi], kC * kD * 2);
                for (int kb = 0; kb < 2; ++kb)
                    tc::tma_load_4d(dst0 + bi * kTile + kb * kBlk, map, kb * 64, h, (j0 + j) * kC, b, &full[bi]);
                if (j + nb < NC)
                    for (int kb = 0; kb < 2; ++kb) tc::tma_prefetch_4d(map, kb * 64, h, (j0 + j + nb) * kC, b);
            }
            // the last copy into each buffer has landed before exit
            for (int jj = j - 1; jj >= 0 && jj >= j - nb; --jj) wait1(&full[jj % nb], (jj / nb) & 1);
        }
    } else if (warp == 9) {
        // ------------------------------------------------ output-side MMAs
        if (lane == 0) {
            constexpr uint32_t idQK = tc::idesc_bf16(128, 128, false, false);
            constexpr uint32_t idMNB = tc::idesc_bf16(128, 128, false, true);
            bool ok = true;
            for (int j = 0; ok && !so && j < NC; ++j) {
                const uint32_t ph = j & 1, bi = j & 1, ph2 = (j >> 1) & 1;
                const uint32_t v_s = base + kV0 + bi * kTile;
                // scores: Q K_w^T when the chunk folds, else Q K^T
                if (!wait1(&bars[kSReady], ph) || !wait1(&bars[kQFull], ph) || !wait1(&bars[kKFull], ph) ||
                    *abort_flag) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const uint32_t kb_s = base + (fold_flag[bi] ? kKw : kK);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBlk + (kk & 3) * 32;
                    tc::mma_bf16_ss(tA, tc::smem_desc_sw128(base + kQ + off, 16, 1024),
                                    tc::smem_desc_sw128(kb_s + off, 16, 1024), idQK, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&bars[kAFull]);
                tc::mma_commit(&bars[kKEmpty]);
                // X = Q S_prev; X and O must have been read out
                if (j > 0 && !wait1(&bars[kOFree], (j - 1) & 1)) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBlk + (kk & 3) * 32;
                    tc::mma_bf16_ss(tX, tc::smem_desc_sw128(base + kQ + off, 16, 1024),
                                    tc::smem_desc_sw128(base + kSb + kk * 2048, kBlk, 1024), idMNB, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&bars[kQEmpty]);
                // O = P V
                if (!wait1(&bars[kPFull], ph) || !wait1(&bars[kVFull + bi], ph2)) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    tc::mma_bf16_ts(tO, tA + kk * 8, tc::smem_desc_sw128(v_s + kk * 2048, kBlk, 1024), idMNB,
                                    kk > 0 ? 1u : 0u);
                tc::mma_commit(&bars[kOFull]);
                tc::mma_commit(&bars[kVEmpty + bi]);
            }
            if (!ok) *abort_flag = 1;
            tc::mma_commit(&bars[kDrainO]);
            wait1(&bars[kDrainO], 0);
        }
    } else if (warp == 10) {
        // -------------------------------------------------------- state MMA
        if (lane == 0) {
            constexpr uint32_t idUpd = tc::idesc_bf16(128, 128, true, true);
            bool ok = true;
            for (int j = 0; ok && j < NC; ++j) {
                const uint32_t ph = j & 1, bi = j & 1, ph2 = (j >> 1) & 1;
                if (!wait1(&bars[kSReady], ph) || *abort_flag) { ok = false; break; }
                mbar_arrive(&bars[kKEmpty]);  // the state warps are done reading K
                if (!wait1(&bars[kVFull + bi], ph2)) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    tc::mma_bf16_ss(tS, tc::smem_desc_sw128(base + kKw + kk * 2048, kBlk, 1024),
                                    tc::smem_desc_sw128(base + kV0 + bi * kTile + kk * 2048, kBlk, 1024), idUpd, 1u);
                tc::mma_commit(&bars[kVEmpty + bi]);
                tc::mma_commit(&bars[kSUpdated]);
            }
            if (!ok) *abort_flag = 1;
            tc::mma_commit(&bars[kDrainS]);
            wait1(&bars[kDrainS], 0);
        }
    } else {
        // ------------------------------------------- output and state warps
        const bool state_role = warp >= 4;
        const int r = (warp & 3) * 32 + lane;                 // TMEM lane = chunk row / state row
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const float *gb = p.g + (int64_t)b * p.T * p.H + h;
        const bool store_thread = warp == 0 && lane == 0;   // issues the output tile's TMA store
        bool ok = true;
        float sc_log2 = 0.f;   // running log2 of this CTA's total decay (state-only launch)

        if (state_role) {
            // initial state into TMEM rows: zero for a state-only launch; for
            // superchunk s > 0 of the output launch, the state after the
            // superchunks before it,
            //   S_s = 2^(G_0 + .. + G_{s-1}) S_init + sum_{s' < s} 2^(G_{s'+1} + .. + G_{s-1}) dS_{s'}
            // (G: a superchunk's log2 total decay, dS: its state from zero)
            const float *s0 = p.state ? p.state + ((int64_t)b * p.H + h) * kD * kD + (int64_t)r * kD : nullptr;
            float *dS = nullptr, *s_copy = nullptr;
            const float *G = nullptr;
            if (p.n_sc > 1) {
                dS = p.sc_state + (int64_t)bh * p.n_sc * kD * kD + (int64_t)r * kD;
                s_copy = dS + (int64_t)(p.n_sc - 1) * kD * kD;
                G = p.sc_log2decay + (int64_t)bh * p.n_sc;
                if (!so) s0 = s_copy;   // the state-only pass copied the initial state
            }
#pragma unroll
            for (int c = 0; c < kD; c += 32) {
                float v[32];
                if (so) {
                    if (sc == 0) {   // the initial state's copy for the output pass
#pragma unroll
                        for (int e = 0; e < 32; ++e) s_copy[c + e] = s0 ? s0[c + e] : 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0.f;
                } else if (p.n_sc == 1) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = s0 ? s0[c + e] : 0.f;
                } else {
                    float tail = 0.f;   // G_{s'+1} + .. + G_{sc-1}, built from s' = sc - 1 down
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = 0.f;
                    for (int s2 = sc - 1; s2 >= 0; --s2) {
                        const float wgt = tc::ex2(tail);
                        const float *row = dS + (int64_t)s2 * kD * kD + c;
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = fmaf(wgt, row[e], v[e]);
                        tail += G[s2];
                    }
                    const float wgt = tc::ex2(tail);
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = fmaf(wgt, s0[c + e], v[e]);
                }
                tc::tmem_st32(tS + lane_off + c, v);
            }
            tc::wait_st();
        }

        // gate logits of the chunk after the current one (lane l: rows 4l..4l+3)
        float gn[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t t = (int64_t)j0 * kC + 4 * lane + i;
            gn[i] = t < p.T ? gb[t * p.H] : 0.f;
        }

        for (int j = 0; ok && j < NC; ++j) {
            const uint32_t ph = j & 1;
            const int64_t t0 = (int64_t)(j0 + j) * kC;
            // running base-2 log-decay sums of the chunk in registers: lane l
            // holds c_u for u = 4l..4l+3 (padded rows decay by 1)
            float x[4];
            {
                float run = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    run += t0 + 4 * lane + i < p.T ? log2_decay(gn[i], p.lg_scale) : 0.f;
                    x[i] = run;
                }
                if (j + 1 < NC) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int64_t t = t0 + kC + 4 * lane + i;
                        gn[i] = t < p.T ? gb[t * p.H] : 0.f;
                    }
                }
                float incl = run;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                const float excl = incl - run;
#pragma unroll
                for (int i = 0; i < 4; ++i) x[i] += excl;
            }
            // c_r of this thread's row r (held by lane r / 4) and c_last
            float c_r;
            {
                const int src = r >> 2;
                const float y0 = __shfl_sync(0xffffffffu, x[0], src), y1 = __shfl_sync(0xffffffffu, x[1], src);
                const float y2 = __shfl_sync(0xffffffffu, x[2], src), y3 = __shfl_sync(0xffffffffu, x[3], src);
                const int sel = r & 3;
                c_r = sel == 0 ? y0 : sel == 1 ? y1 : sel == 2 ? y2 : y3;
            }
            const float c_last = __shfl_sync(0xffffffffu, x[3], 31);
            const bool fold = c_last >= kFoldMinLog2;   // the same in every warp
            sc_log2 += c_last;

            if (so && !state_role) break;   // a state-only launch: the output warps have nothing to do
            if (!state_role) {
                // ---- P: 2^{c_r - c_last} (Q K_w^T) or scale 2^{c_r - c_u} (Q K^T),
                // for u <= r, else 0
                if (!waitw(&bars[kAFull], ph)) { ok = false; break; }
                tc::fence_after_sync();
                const float fr = tc::ex2(c_r - c_last);
#pragma unroll
                for (int qt = 0; qt < 4; ++qt) {
                    float a[32];
                    tc::tmem_ld32(tA + lane_off + qt * 32, a);
                    tc::wait_ld();
                    uint32_t pk[16];
                    if (fold) {
#pragma unroll
                        for (int u2 = 0; u2 < 32; u2 += 2) {
                            const int u = qt * 32 + u2;
                            pk[u2 / 2] = tc::pack_bf16x2(u <= r ? a[u2] * fr : 0.f, u + 1 <= r ? a[u2 + 1] * fr : 0.f);
                        }
                    } else {
#pragma unroll
                        for (int u2 = 0; u2 < 32; u2 += 2) {
                            const int u = qt * 32 + u2;
                            const float cu0 = __shfl_sync(0xffffffffu, x[u & 3], u >> 2);
                            const float cu1 = __shfl_sync(0xffffffffu, x[(u + 1) & 3], (u + 1) >> 2);
                            const float w0 = u <= r ? p.scale * tc::ex2(c_r - cu0) : 0.f;
                            const float w1 = u + 1 <= r ? p.scale * tc::ex2(c_r - cu1) : 0.f;
                            pk[u2 / 2] = tc::pack_bf16x2(a[u2] * w0, a[u2 + 1] * w1);
                        }
                    }
                    tc::tmem_st16u(tA + lane_off + qt * 16, pk);
                }
                tc::wait_st();
                tc::fence_before_sync();
                mbar_arrive(&bars[kPFull]);
                // ---- o = O + 2^{c_r} X into the output tile, then its TMA store
                if (!waitw(&bars[kOFull], ph)) { ok = false; break; }
                tc::fence_after_sync();
                // the previous chunk's store has read the tile
                if (j > 0) {
                    if (store_thread) {
                        tc::bulk_wait_read_all();
                        mbar_arrive(&bars[kOtFree]);
                    }
                    if (!waitw(&bars[kOtFree], (j - 1) & 1)) { ok = false; break; }
                }
                const float f = tc::ex2(c_r);
#pragma unroll
                for (int c = 0; c < kD; c += 32) {
                    float ov[32], xv[32];
                    tc::tmem_ld32(tO + lane_off + c, ov);
                    tc::tmem_ld32(tX + lane_off + c, xv);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 w;
                        w.x = tc::pack_bf16x2(fmaf(f, xv[e], ov[e]), fmaf(f, xv[e + 1], ov[e + 1]));
                        w.y = tc::pack_bf16x2(fmaf(f, xv[e + 2], ov[e + 2]), fmaf(f, xv[e + 3], ov[e + 3]));
                        w.z = tc::pack_bf16x2(fmaf(f, xv[e + 4], ov[e + 4]), fmaf(f, xv[e + 5], ov[e + 5]));
                        w.w = tc::pack_bf16x2(fmaf(f, xv[e + 6], ov[e + 6]), fmaf(f, xv[e + 7], ov[e + 7]));
                        *reinterpret_cast<uint4 *>(sb + kOt + sw_off(r, c + e)) = w;
                    }
                }
                tc::fence_before_sync();
                mbar_arrive(&bars[kOFree]);
                fence_proxy_async_smem();
                mbar_arrive(&bars[kOStaged]);
                if (warp == 0) {
                    bool sok = true;
                    if (lane == 0) {
                        sok = wait1(&bars[kOStaged], ph);
                        if (sok) {
                            // rows past the sequence's end are not written
                            tc::tma_store_4d(&tm_o, base + kOt, 0, h, (int)t0, b);
                            tc::tma_store_4d(&tm_o, base + kOt + kBlk, 64, h, (int)t0, b);
                            tc::bulk_commit_group();
                        }
                    }
                    if (!__shfl_sync(0xffffffffu, (int)sok, 0)) { ok = false; break; }
                }
            } else {
                // ---- K_w = K * scale * 2^{c_last - c_u} (row u = r of the K tile);
                // the previous update and the previous scores have read K_w
                if (!waitw(&bars[kKFull], ph)) { ok = false; break; }
                if (!so && j > 0 && !waitw(&bars[kAFull], (j - 1) & 1)) { ok = false; break; }
                {
                    const float w = p.scale * tc::ex2(c_last - c_r);
#pragma unroll
                    for (int c = 0; c < kD; c += 8) {
                        const uint32_t off = sw_off(r, c);
                        const uint4 kv = *reinterpret_cast<const uint4 *>(sb + kK + off);
                        const uint32_t *kp = &kv.x;
                        uint4 out;
                        uint32_t *op = &out.x;
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            op[q] = tc::pack_bf16x2(__uint_as_float(kp[q] << 16) * w,
                                                    __uint_as_float(kp[q] & 0xffff0000u) * w);
                        *reinterpret_cast<uint4 *>(sb + kKw + off) = out;
                    }
                }
                // ---- one pass over S_prev: its bf16 copy for this chunk's cross
                // term (once the previous cross term has read the last copy),
                // and S *= 2^{c_last} in TMEM
                if (!so && j > 0 && !waitw(&bars[kQEmpty], (j - 1) & 1)) { ok = false; break; }
                {
                    const float f = tc::ex2(c_last);
                    tc::fence_after_sync();
#pragma unroll
                    for (int c = 0; c < kD; c += 32) {
                        float v[32];
                        tc::tmem_ld32(tS + lane_off + c, v);
                        tc::wait_ld();
                        if (!so) {   // the cross term's bf16 copy (no cross term without outputs)
#pragma unroll
                            for (int e = 0; e < 32; e += 8) {
                                uint4 hv;
                                hv.x = tc::pack_bf16x2(v[e], v[e + 1]);
                                hv.y = tc::pack_bf16x2(v[e + 2], v[e + 3]);
                                hv.z = tc::pack_bf16x2(v[e + 4], v[e + 5]);
                                hv.w = tc::pack_bf16x2(v[e + 6], v[e + 7]);
                                *reinterpret_cast<uint4 *>(sb + kSb + sw_off(r, c + e)) = hv;
                            }
                        }
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] *= f;
                        tc::tmem_st32(tS + lane_off + c, v);
                    }
                    tc::wait_st();
                }
                if (warp == 4 && lane == 0) fold_flag[j & 1] = fold ? 1 : 0;
                fence_proxy_async_smem();
                tc::fence_before_sync();
                mbar_arrive(&bars[kSReady]);
                if (!waitw(&bars[kSUpdated], ph)) { ok = false; break; }
            }
        }
        // the final state: a state-only CTA's into the scratch (with its log2
        // total decay); in the output launch only the last superchunk's
        float *sfin = nullptr;
        if (so)
            sfin = p.sc_state + ((int64_t)bh * p.n_sc + sc) * kD * kD + (int64_t)r * kD;
        else if (p.state && sc == p.n_sc - 1)
            sfin = p.state + ((int64_t)b * p.H + h) * kD * kD + (int64_t)r * kD;
        if (so && ok && warp == 4 && lane == 0) p.sc_log2decay[(int64_t)bh * p.n_sc + sc] = sc_log2;
        if (ok && state_role && sfin) {
            tc::fence_after_sync();
#pragma unroll
            for (int c = 0; c < kD; c += 32) {
                float v[32];
                tc::tmem_ld32(tS + lane_off + c, v);
                tc::wait_ld();
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(sfin + c + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
            }
        }
        if (store_thread) tc::bulk_wait_all();  // the output tiles are written before exit
        if (!ok) *abort_flag = 1;
        tc::wait_st();
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 9) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------- host
namespace {

// 4-D bf16 map over [B, T, H, D] (innermost D), box {64, 1, 128, 1}, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *ptr, int64_t B, int64_t T, int64_t H) {
    const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)H, (uint64_t)T, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)(kD * 2), (uint64_t)(H * kD * 2), (uint64_t)(T * H * kD * 2)};
    const uint32_t box[4] = {64, 1, 128, 1};
    return encode_bf16_map_4d(m, ptr, dims, strides, box);
}

}  // namespace

cudaError_t launch_gret_prefill_tc(const GretArgs &a, cudaStream_t st) {
    if (a.dtype != kBF16 || a.D != kD) return cudaErrorNotSupported;
    if (a.B == 0 || a.T == 0 || a.H == 0) return cudaSuccess;
    if ((int64_t)a.B * a.H > INT32_MAX || a.T > INT32_MAX) return cudaErrorNotSupported;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, a.q, a.B, a.T, a.H) || !make_map(&mk, a.k, a.B, a.T, a.H) ||
        !make_map(&mv, a.v, a.B, a.T, a.H) || !make_map(&mo, a.o, a.B, a.T, a.H))
        return cudaErrorNotSupported;
    GretTcParams p;
    p.g = a.g;
    p.state = a.state;
    p.B = a.B; p.H = a.H; p.T = a.T;
    p.lg_scale = kLog2e / a.tau;
    p.scale = a.scale;
    p.n_chunks = (int)((a.T + kC - 1) / kC);
    p.n_sc = a.ws ? gret_superchunks(a.B, a.H, a.T, device_sm_count()) : 1;
    p.sc_chunks = (p.n_chunks + p.n_sc - 1) / p.n_sc;
    p.n_sc = (p.n_chunks + p.sc_chunks - 1) / p.sc_chunks;   // no empty superchunk
    p.sc_state = static_cast<float *>(a.ws);
    p.sc_log2decay = p.sc_state ? p.sc_state + (size_t)a.B * a.H * p.n_sc * kD * kD : nullptr;
    cudaError_t e = cudaFuncSetAttribute(gret_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAlloc);
    if (e != cudaSuccess) return e;
    const int bh = a.B * a.H;
    if (p.n_sc > 1) {
        // pass 1: every superchunk but the last forms its state from zero
        p.state_only = 1;
        note_launches(1);
        gret_tc_kernel<<<bh * (p.n_sc - 1), kThreads, kAlloc, st>>>(mq, mk, mv, mo, p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // pass 2 (or the only pass): outputs, each superchunk from its own start state
    p.state_only = 0;
    note_launches(1);
    gret_tc_kernel<<<bh * p.n_sc, kThreads, kAlloc, st>>>(mq, mk, mv, mo, p);
    return cudaGetLastError();
}

int gret_superchunks(int32_t B, int32_t H, int64_t T, int sms) {
    // as many superchunks as leave one per SM, at most kMaxSuperchunks, and
    // at least 8 chunks each; 1 when the sequences alone fill the GPU
    const int64_t bh = (int64_t)B * H;
    const int64_t n_chunks = (T + kC - 1) / kC;
    int64_t n = bh > 0 ? sms / bh : 1;
    n = std::min<int64_t>(n, kMaxSuperchunks);
    n = std::min<int64_t>(n, n_chunks / 8);
    return (int)std::max<int64_t>(n, 1);
}

size_t gret_workspace_bytes(int32_t B, int32_t H, int64_t T, int D) {
    if (D != kD || B < 1 || H < 1 || T < 1) return 0;
    if ((int64_t)B * H >= 148) return 0;   // the sequences alone fill the GPU: no split
    return (size_t)B * H * kMaxSuperchunks * (kD * kD + 1) * sizeof(float);
}

unsigned int read_and_clear_status_gret_tc() {
    unsigned int h = 0, z = 0;
    if (cudaMemcpyFromSymbol(&h, g_status_gret_tc, sizeof(h)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_status_gret_tc, &z, sizeof(z));
    return h;
}

}  // namespace yoco
