// Causal / sliding-window GQA attention prefill on the sm_100a tensor cores
// for even group sizes, two query heads per CTA (bf16 in, fp32 softmax and
// accumulation).
//
// The same attention as prefill_tc.cu ("You Only Cache Once", paperlayer
// summary, sections 1-3; podcast transcript cue 12: every cross layer attends
// causally to the one shared K_g, V_g with grouped-query heads; the
// self-decoder attends within a fixed window), with a different work unit: a
// 128-row query tile of TWO query heads 2hp and 2hp + 1 of one KV group.  The
// two heads read the same K and V tiles and have the same mask, so one KV
// stream feeds both, and each SM sub-partition runs two softmax warps (one per
// head) whose latencies interleave: with one softmax warp per sub-partition
// the softmax chain, not the tensor core, set the pace.
//
// Persistent grid: one CTA per SM walks the work tiles heaviest first in
// snake order.  Warp roles (320 threads):
//   warps 0-3  softmax of head A (= 2hp), warps 4-7 of head B: thread r owns
//              query row r (TMEM lane r).  Per KV tile it reads S from TMEM,
//              masks (diagonal / window / tail tiles), takes the row max,
//              computes P = 2^(S*scale*log2e - m) -- three quarters of the
//              exponentials on MUFU, a quarter on an FMA-pipe polynomial --
//              and writes P as bf16 over the first 64 columns of its S buffer.
//              The running max only moves (and O is rescaled in TMEM) when it
//              grows by more than 2^8.  The same warps run the epilogue, which
//              frees the O columns as soon as they are in registers.
//   warp 8     TMA producer: lane 0 loads the two Q tiles, lane 1 the K tiles
//              (three stages), lane 2 the V tiles (two stages).
//   warp 9     MMA issuer (one thread), in the order
//                PV_A(t-1), S_A(t), PV_B(t-1), S_B(t), PV_A(t), S_A(t+1), ...
//              so that while softmax A works on S_A(t) the tensor core runs
//              PV_B(t-1) and S_B(t), and the other way round.  One thread's
//              MMAs run in issue order, so S_A(t+1) overwrites P_A(t) only
//              after PV_A(t) has read it, and "S_A(t) is ready" also means
//              PV_A(t-1) has finished.
// TMEM (512 columns): S_A/P_A [0,128), S_B/P_B [128,256), O_A [256,384),
// O_B [384,512).  Every barrier phase follows the CTA's running KV tile
// counter g (S, P and O done: one completion per KV tile per head) or its
// work counter k (Q, O free: one per work tile).
// Every mbarrier wait is bounded; a wait that gives up sets the status word,
// and all roles fall through to the common exit, which waits for issued
// copies and MMAs before freeing TMEM.
#include <cuda.h>

#include <algorithm>
#include <cstdint>

#include "common.cuh"
#include "launch.h"
#include "schedule.h"
#include "tc.cuh"

namespace yoco {

static __device__ unsigned int g_status_prefill_pair;

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kThreads = 320;
constexpr int kTmemCols = 512;
constexpr uint32_t kBlk = 128 * 128;  // one [128 rows x 128 bytes] swizzled block

template <int D>
struct Smem {
    static constexpr int KB = D / 64;                  // 64-element column blocks
    static constexpr uint32_t TILE = (uint32_t)KB * kBlk;
    static constexpr int KSTAGES = 3;
    static constexpr int VSTAGES = 2;
    static constexpr uint32_t Q = 0;                   // head A tile, then head B tile
    static constexpr uint32_t K = Q + 2 * TILE;
    static constexpr uint32_t V = K + KSTAGES * TILE;
    static constexpr uint32_t BAR = V + VSTAGES * TILE;
    static constexpr uint32_t BYTES = BAR + 256;
    static constexpr uint32_t ALLOC = BYTES + 1024;    // alignment slack
};

struct PairParams {
    sched::PrefillShape s;
    float scale_log2;
    void *o;
    float *lse;
    int32_t n_work;
    int32_t o_32B;   // o is 32-byte aligned: rows go out in 32-byte stores
};

enum Bar {
    kQFull = 0,    // 2: Q tile of head A / B loaded
    kQEmpty = 2,   // 2: last S MMA of head A / B of the work tile done
    kKFull = 4,    // 3
    kKEmpty = 7,   // 3
    kVFull = 10,   // 2
    kVEmpty = 12,  // 2
    kSFull = 14,   // 2: S of head A / B ready
    kPFull = 16,   // 2: P of head A / B written (128 arrivals)
    kODone = 18,   // 2: P.V of head A / B finished
    kOFree = 20,   // 2: O of head A / B read out by the epilogue (128 arrivals)
    kDrain = 22,
    kNumBars = 23
};

// 32-byte global store (the sm_100 256-bit vector store), not kept in L1; the
// address must be 32-byte aligned.
YOCO_DEV void st_global_32B(void *p, const uint32_t (&w)[8]) {
    asm volatile("st.global.L1::no_allocate.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :: "l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]),
                    "r"(w[7])
                 : "memory");
}

YOCO_DEV bool wait1(uint64_t *bar, uint32_t parity) {
    return mbar_wait(bar, parity, &g_status_prefill_pair);
}
YOCO_DEV bool waitw(uint64_t *bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, &g_status_prefill_pair));
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                             const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const PairParams p) {
    // once any CTA has recorded a timeout, the rest of the grid exits at once
    if (*(volatile unsigned int *)&g_status_prefill_pair) return;
    using L = Smem<D>;
    constexpr int KB = L::KB;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sbase = smem_raw + (base - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sbase + L::BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sbase + L::BAR + kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sbase + L::BAR + kNumBars * 8 + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kQFull + s], 1);
            mbar_init(&bars[kQEmpty + s], 1);
            mbar_init(&bars[kSFull + s], 1);
            mbar_init(&bars[kPFull + s], 128);
            mbar_init(&bars[kODone + s], 1);
            mbar_init(&bars[kOFree + s], 128);
        }
        for (int s = 0; s < L::KSTAGES; ++s) {
            mbar_init(&bars[kKFull + s], 1);
            mbar_init(&bars[kKEmpty + s], 1);
        }
        for (int s = 0; s < L::VSTAGES; ++s) {
            mbar_init(&bars[kVFull + s], 1);
            mbar_init(&bars[kVEmpty + s], 1);
        }
        mbar_init(&bars[kDrain], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 9) {
        tc::tmem_alloc(tmem_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 8) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            // Q tiles of both heads; each half is refilled once the last S MMA
            // of its head in the previous work tile has finished
            int k = 0;
            for (int r = 0; !*abort_flag; ++r, ++k) {
                const int w = sched::prefill_work_index(r, blockIdx.x, gridDim.x);
                if (w >= p.n_work) break;
                const sched::PrefillWork x = sched::prefill_pair_work(p.s, w);
                bool ok = true;
                for (int hh = 0; hh < 2 && ok; ++hh) {
                    if (!wait1(&bars[kQEmpty + hh], (k & 1) ^ 1)) { ok = false; break; }
                    mbar_arrive_expect_tx(&bars[kQFull + hh], BM * D * 2);
                    for (int kb = 0; kb < KB; ++kb)
                        tc::tma_load_4d(base + L::Q + hh * L::TILE + kb * kBlk, &tm_q, kb * 64, x.h + hh,
                                        (int)x.i0, x.b, &bars[kQFull + hh]);
                }
                if (!ok) { *abort_flag = 1; ++k; break; }
            }
            // drain: the last copies issued must land before this CTA may exit
            if (k > 0)
                for (int hh = 0; hh < 2; ++hh)
                    if (!wait1(&bars[kQFull + hh], (k - 1) & 1)) break;
        } else if (lane == 1) {
            int gk = 0;
            for (int r = 0; !*abort_flag; ++r) {
                const int w = sched::prefill_work_index(r, blockIdx.x, gridDim.x);
                if (w >= p.n_work) break;
                const sched::PrefillWork x = sched::prefill_pair_work(p.s, w);
                for (int t = 0; t < x.n_kv; ++t, ++gk) {
                    const int st = gk % L::KSTAGES;
                    if (!wait1(&bars[kKEmpty + st], ((gk / L::KSTAGES) & 1) ^ 1)) { *abort_flag = 1; break; }
                    if (*abort_flag) break;
                    mbar_arrive_expect_tx(&bars[kKFull + st], BN * D * 2);
                    for (int kb = 0; kb < KB; ++kb)
                        tc::tma_load_4d(base + L::K + st * L::TILE + kb * kBlk, &tm_k, kb * 64, x.g,
                                        (x.jt_lo + t) * BN, x.b, &bars[kKFull + st]);
                }
            }
            for (int q = max(0, gk - L::KSTAGES); q < gk; ++q)
                if (!wait1(&bars[kKFull + q % L::KSTAGES], (q / L::KSTAGES) & 1)) break;
        } else if (lane == 2) {
            int gv = 0;
            for (int r = 0; !*abort_flag; ++r) {
                const int w = sched::prefill_work_index(r, blockIdx.x, gridDim.x);
                if (w >= p.n_work) break;
                const sched::PrefillWork x = sched::prefill_pair_work(p.s, w);
                for (int t = 0; t < x.n_kv; ++t, ++gv) {
                    const int st = gv % L::VSTAGES;
                    if (!wait1(&bars[kVEmpty + st], ((gv / L::VSTAGES) & 1) ^ 1)) { *abort_flag = 1; break; }
                    if (*abort_flag) break;
                    mbar_arrive_expect_tx(&bars[kVFull + st], BN * D * 2);
                    for (int kb = 0; kb < KB; ++kb)
                        tc::tma_load_4d(base + L::V + st * L::TILE + kb * kBlk, &tm_v, kb * 64, x.g,
                                        (x.jt_lo + t) * BN, x.b, &bars[kVFull + st]);
                }
            }
            for (int q = max(0, gv - L::VSTAGES); q < gv; ++q)
                if (!wait1(&bars[kVFull + q % L::VSTAGES], (q / L::VSTAGES) & 1)) break;
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------- MMA issue
        if (lane == 0) {
            constexpr uint32_t idS = tc::idesc_bf16(BM, BN, false, false);
            constexpr uint32_t idPV = tc::idesc_bf16(BM, D, false, true);
            bool ok = true;
            // the KV tile whose P.V MMAs are still owed: its tile counter, its
            // work counter, and whether it opens its work tile
            int pend_g = -1, pend_k = 0;
            bool pend_first = false;
            auto issue_pv = [&](int hh) -> bool {
                const int u = pend_g, vs = u % L::VSTAGES;
                if (pend_first && pend_k >= 1 && !wait1(&bars[kOFree + hh], (pend_k - 1) & 1)) return false;
                if (!wait1(&bars[kPFull + hh], u & 1)) return false;
                if (hh == 0 && !wait1(&bars[kVFull + vs], (u / L::VSTAGES) & 1)) return false;
                tc::fence_after_sync();
                const uint32_t vb = base + L::V + vs * L::TILE;
                const uint32_t tp = tmem + hh * 128;        // P over the first 64 columns of S
                const uint32_t to = tmem + 256 + hh * 128;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    tc::mma_bf16_ts(to, tp + kk * 8, tc::smem_desc_sw128(vb + kk * 2048, kBlk, 1024), idPV,
                                    (!pend_first || kk > 0) ? 1u : 0u);
                tc::mma_commit(&bars[kODone + hh]);
                if (hh == 1) tc::mma_commit(&bars[kVEmpty + vs]);
                return true;
            };
            auto issue_s = [&](int hh, uint32_t kbase) {
                const uint32_t qb = base + L::Q + hh * L::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBlk + (kk & 3) * 32;
                    tc::mma_bf16_ss(tmem + hh * 128, tc::smem_desc_sw128(qb + off, 16, 1024),
                                    tc::smem_desc_sw128(kbase + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&bars[kSFull + hh]);
            };
            int g = 0;
            for (int k = 0; ok; ++k) {
                const int w = sched::prefill_work_index(k, blockIdx.x, gridDim.x);
                if (w >= p.n_work) break;
                const sched::PrefillWork x = sched::prefill_pair_work(p.s, w);
                for (int t = 0; t < x.n_kv; ++t, ++g) {
                    const int st = g % L::KSTAGES;
                    if (!wait1(&bars[kKFull + st], (g / L::KSTAGES) & 1) || *abort_flag) { ok = false; break; }
                    const uint32_t kbase = base + L::K + st * L::TILE;
                    if (pend_g >= 0 && !issue_pv(0)) { ok = false; break; }
                    if (t == 0 && !wait1(&bars[kQFull + 0], k & 1)) { ok = false; break; }
                    tc::fence_after_sync();
                    issue_s(0, kbase);
                    if (t == x.n_kv - 1) tc::mma_commit(&bars[kQEmpty + 0]);
                    if (pend_g >= 0 && !issue_pv(1)) { ok = false; break; }
                    if (t == 0 && !wait1(&bars[kQFull + 1], k & 1)) { ok = false; break; }
                    tc::fence_after_sync();
                    issue_s(1, kbase);
                    tc::mma_commit(&bars[kKEmpty + st]);
                    if (t == x.n_kv - 1) tc::mma_commit(&bars[kQEmpty + 1]);
                    pend_g = g;
                    pend_k = k;
                    pend_first = (t == 0);
                }
            }
            if (ok && pend_g >= 0 && !*abort_flag) ok = issue_pv(0) && issue_pv(1);
            if (!ok) *abort_flag = 1;
            // every MMA issued by this thread has finished before TMEM is freed
            tc::mma_commit(&bars[kDrain]);
            wait1(&bars[kDrain], 0);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int hh = warp >> 2;                  // 0: head A, 1: head B
        const int r = threadIdx.x & 127;           // row in tile == TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + hh * 128 + lane_off;
        const uint32_t tO = tmem + 256 + hh * 128 + lane_off;
        const uint64_t sl2 = tc::f2_pack(p.scale_log2, p.scale_log2);
        bool ok = true;
        int g = 0;
        for (int k = 0; ok; ++k) {
            const int w = sched::prefill_work_index(k, blockIdx.x, gridDim.x);
            if (w >= p.n_work) break;
            const sched::PrefillWork x = sched::prefill_pair_work(p.s, w);
            const int h = x.h + hh;
            const int64_t i = x.i0 + r;
            const int64_t pos = p.s.q_pos0 + i;
            float m = -INFINITY, l = 0.f;
            for (int t = 0; t < x.n_kv; ++t, ++g) {
                if (!waitw(&bars[kSFull + hh], g & 1)) { ok = false; break; }
                tc::fence_after_sync();
                float s[BN];
#pragma unroll
                for (int c = 0; c < BN; c += 32) tc::tmem_ld32(tS + c, s + c);
                tc::wait_ld();
                if (sched::prefill_tile_masked(p.s, x, t)) {
                    // visible columns of this row form one range [c_lo, c_hi); the
                    // diagonal tile has c_lo = 0 and a window's lower-edge tile
                    // c_hi = BN, which need one comparison per column, not two
                    const int64_t j0 = (int64_t)(x.jt_lo + t) * BN;
                    const int64_t dg = pos - j0;
                    const int c_hi = (int)max((int64_t)0, min(min(dg + 1, p.s.Tkv - j0), (int64_t)BN));
                    const int c_lo =
                        p.s.window > 0 ? (int)max((int64_t)0, min(dg - p.s.window + 1, (int64_t)BN)) : 0;
                    if (c_lo == 0) {
#pragma unroll
                        for (int c = 0; c < BN; ++c) s[c] = c < c_hi ? s[c] : -INFINITY;
                    } else if (c_hi == BN) {
#pragma unroll
                        for (int c = 0; c < BN; ++c) s[c] = c >= c_lo ? s[c] : -INFINITY;
                    } else {
                        const unsigned width = (unsigned)max(0, c_hi - c_lo);
#pragma unroll
                        for (int c = 0; c < BN; ++c) s[c] = (unsigned)(c - c_lo) < width ? s[c] : -INFINITY;
                    }
                }
                // row max: 3-input max tree, eight independent chains
                float a8[8];
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) a8[kk] = tc::max3(s[kk], s[kk + 8], s[kk + 16]);
#pragma unroll
                for (int c = 24; c < 120; c += 16)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) a8[kk] = tc::max3(a8[kk], s[c + kk], s[c + 8 + kk]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) a8[kk] = fmaxf(a8[kk], s[120 + kk]);
                const float mx = tc::max3(tc::max3(a8[0], a8[1], a8[2]), tc::max3(a8[3], a8[4], a8[5]),
                                          fmaxf(a8[6], a8[7]));
                const float m_cand = mx * p.scale_log2;
                float alpha = 1.f;
                const bool grow = m_cand > m + 8.f;
                if (grow) {
                    alpha = (m == -INFINITY) ? 0.f : tc::ex2(m - m_cand);
                    m = m_cand;
                }
                const float neg_m = (m == -INFINITY) ? 0.f : -m;
                // P = 2^(S * scale * log2e - m) on packed pairs; columns 48-63 and
                // 112-127 of every 64 on the FMA-pipe polynomial, the rest on MUFU.
                // Each half row of P goes to TMEM as soon as it is packed.
                const uint64_t nm2 = tc::f2_pack(neg_m, neg_m);
                uint64_t rs2a = 0, rs2b = 0;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t pk[BN / 4];
#pragma unroll
                    for (int cc = 0; cc < BN / 2; cc += 2) {
                        const int c = half * (BN / 2) + cc;
                        float x0, x1, e0, e1;
                        tc::f2_unpack(tc::f2_fma(tc::f2_pack(s[c], s[c + 1]), sl2, nm2), x0, x1);
                        if ((c & 48) != 48) {
                            e0 = tc::ex2(x0);
                            e1 = tc::ex2(x1);
                        } else {
                            // a masked score (-inf) gives 2^-125 here, not 0: ~1e-38 of the
                            // row's largest weight (>= 1 after the max), below any fp32 sum's
                            // resolution; bound and -inf checked by the exp2 probe test
                            tc::exp2_pair_poly(x0, x1, e0, e1);
                        }
                        if (c & 2)
                            rs2b = tc::f2_add(rs2b, tc::f2_pack(e0, e1));
                        else
                            rs2a = tc::f2_add(rs2a, tc::f2_pack(e0, e1));
                        pk[cc / 2] = tc::pack_bf16x2(e0, e1);
                    }
                    tc::tmem_st32u(tS + half * 32, pk);
                }
                float ra0, ra1, rb0, rb1;
                tc::f2_unpack(rs2a, ra0, ra1);
                tc::f2_unpack(rs2b, rb0, rb1);
                l = l * alpha + ((ra0 + ra1) + (rb0 + rb1));
                // O holds P.V up to the previous KV tile (finished: S_t was issued
                // after it); rescale it before this tile's P.V is issued
                if (t >= 1 && __any_sync(0xffffffffu, grow)) {
                    if (!waitw(&bars[kODone + hh], (g - 1) & 1)) { ok = false; break; }
                    tc::fence_after_sync();
#pragma unroll
                    for (int c = 0; c < D; c += 32) {
                        float o[32];
                        tc::tmem_ld32(tO + c, o);
                        tc::wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= alpha;
                        tc::tmem_st32(tO + c, o);
                    }
                }
                tc::wait_st();
                tc::fence_before_sync();
                mbar_arrive(&bars[kPFull + hh]);
            }
            if (!ok) break;
            // epilogue: the last P.V of this work tile.  O is read out of TMEM
            // whole and its columns handed to the next work tile's first P.V
            // before O / l goes to global memory.  Each thread writes its own
            // row, so a warp's store covers 32 rows: 32-byte stores make that
            // 32 whole sectors per instruction, not 32 half sectors.
            if (!waitw(&bars[kODone + hh], (g - 1) & 1)) { ok = false; break; }
            tc::fence_after_sync();
            float o[D];
#pragma unroll
            for (int c = 0; c < D; c += 32) tc::tmem_ld32(tO + c, o + c);
            tc::wait_ld();
            tc::fence_before_sync();
            mbar_arrive(&bars[kOFree + hh]);
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *dst =
                static_cast<__nv_bfloat16 *>(p.o) + (((int64_t)x.b * p.s.Tq + i) * p.s.Hq + h) * D;
            if (i < p.s.Tq) {
                if (p.o_32B) {
#pragma unroll
                    for (int e = 0; e < D; e += 16) {
                        uint32_t wv[8];
#pragma unroll
                        for (int u = 0; u < 8; ++u) wv[u] = tc::pack_bf16x2(o[e + 2 * u] * inv, o[e + 2 * u + 1] * inv);
                        st_global_32B(dst + e, wv);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < D; e += 8) {
                        uint4 wv;
                        wv.x = tc::pack_bf16x2(o[e] * inv, o[e + 1] * inv);
                        wv.y = tc::pack_bf16x2(o[e + 2] * inv, o[e + 3] * inv);
                        wv.z = tc::pack_bf16x2(o[e + 4] * inv, o[e + 5] * inv);
                        wv.w = tc::pack_bf16x2(o[e + 6] * inv, o[e + 7] * inv);
                        *reinterpret_cast<uint4 *>(dst + e) = wv;
                    }
                }
            }
            if (p.lse && i < p.s.Tq)
                p.lse[((int64_t)x.b * p.s.Hq + h) * p.s.Tq + i] = l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
        }
        if (!ok) *abort_flag = 1;
        tc::wait_st();  // no TMEM store may be in flight when TMEM is freed
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 9) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------- host
namespace {

// 4-D bf16 map over [B, T, H, D] (innermost D), box {64, 1, 128, 1}, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *ptr, int64_t B, int64_t T, int64_t H, int64_t D) {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)H, (uint64_t)T, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)(D * 2), (uint64_t)(H * D * 2), (uint64_t)(T * H * D * 2)};
    const uint32_t box[4] = {64, 1, 128, 1};
    return encode_bf16_map_4d(m, ptr, dims, strides, box);
}

template <int D>
cudaError_t launch_pair_d(const PrefillArgs &a, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.B, a.Tq, a.Hq, D) || !make_map(&mk, a.k, a.B, a.Tkv, a.Hkv, D) ||
        !make_map(&mv, a.v, a.B, a.Tkv, a.Hkv, D))
        return cudaErrorNotSupported;
    PairParams p;
    p.s.B = a.B; p.s.Hq = a.Hq; p.s.Hkv = a.Hkv;
    p.s.Tq = a.Tq; p.s.Tkv = a.Tkv; p.s.q_pos0 = a.q_pos0; p.s.window = a.window;
    p.scale_log2 = a.scale * kLog2e;
    p.o = a.o; p.lse = a.lse;
    p.o_32B = (reinterpret_cast<uintptr_t>(a.o) & 31u) == 0;
    const int64_t n_qtiles = (a.Tq + BM - 1) / BM;
    const int64_t n_work = n_qtiles * (a.Hq / 2) * a.B;
    if (n_work > INT32_MAX / 2) return cudaErrorNotSupported;
    p.s.n_qtiles = (int)n_qtiles;
    p.n_work = (int)n_work;
    const int grid = (int)std::min<int64_t>(n_work, device_sm_count());
    p.s.band = sched::prefill_band(grid, (a.Hq / a.Hkv) / 2, (int64_t)a.B * a.Tkv * a.Hkv * D * 2 * 2, a.window);
    auto kern = attn_prefill_pair_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Smem<D>::ALLOC);
    if (e != cudaSuccess) return e;
    note_launches(1);
    kern<<<grid, kThreads, Smem<D>::ALLOC, st>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_pair(const PrefillArgs &a, cudaStream_t st) {
    if (a.dtype != kBF16 || !sched::prefill_pairs_heads(a.Hq, a.Hkv)) return cudaErrorNotSupported;
    if (a.B == 0 || a.Tq == 0) return cudaSuccess;
    if (a.D == 128) return launch_pair_d<128>(a, st);
    if (a.D == 64) return launch_pair_d<64>(a, st);
    return cudaErrorNotSupported;
}

unsigned int read_and_clear_status_prefill_pair() {
    unsigned int h = 0, z = 0;
    if (cudaMemcpyFromSymbol(&h, g_status_prefill_pair, sizeof(h)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_status_prefill_pair, &z, sizeof(z));
    return h;
}

}  // namespace yoco
