// Causal / sliding-window GQA attention prefill on the sm_100a tensor cores
// (bf16 in, fp32 softmax and accumulation): tcgen05.mma with TMEM
// accumulators, TMA-staged Q/K/V tiles, fp32 online softmax.
//
// It serves the cross-decoder's causal prefill over the one shared KV
// ("You Only Cache Once", paperlayer summary, section 2; podcast transcript
// cue 12: each cross layer has its own Q and attends causally to the shared
// K_g, V_g) and the self-decoder's sliding-window prefill (section 3).  The
// query / key visibility rule is j <= p, plus j > p - window when window > 0,
// for a query at absolute position p = q_pos0 + row.
//
// Persistent grid: one CTA per SM walks work tiles -- a 128-row query tile of
// one (batch, query head) -- heaviest causal tiles first, and streams the KV
// tiles of every work tile through one continuous pipeline, so the next work
// tile's Q load and first S MMA overlap the previous tile's epilogue.  Every
// barrier phase below follows the CTA's running KV-tile counter g (or its
// work-tile counter k for Q and O).  Warp roles:
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r).  For each KV
//              tile it reads S from TMEM, masks (diagonal / window / tail tiles
//              only), takes the row max (3-input max tree), computes
//              P = 2^(S*scale*log2e - m) in fp32 on packed pairs -- three
//              quarters of the exponentials on MUFU, a quarter on an FMA-pipe
//              polynomial -- and writes P as bf16 pairs over the first 64
//              columns of the same S buffer.  The running max is only moved
//              (and O in TMEM rescaled) when it grows by more than 2^8, which
//              keeps O exact after the final 1/l.  At the end of a work tile
//              the same warps normalise O and store it.
//   warp 4     TMA producer: lane 0 loads Q (two buffers) and K tiles (three
//              stages), lane 1 V tiles (two stages); mbarrier complete_tx.
//   warp 5     MMA issuer (one thread): S_g = Q K_g^T into TMEM S buffer g&1,
//              issued one tile ahead so the tensor core computes S_{g+1} while
//              the softmax works on S_g; then O += P_g V_g with P read from
//              TMEM (A operand in tensor memory) and V read MN-major straight
//              from its TMA tile.  One thread's MMAs execute in issue order, so
//              S_{g+2} may overwrite the P_g that P_g V_g read before it; and a
//              commit arrives only when every earlier MMA is done, so "S_g is
//              ready" also means P_{g-2} V has been consumed.
// TMEM (512 columns): S0/P0 [0,128), S1/P1 [128,256), O0 [256,384), O1
// [384,512); work tile k accumulates in O(k&1), so its epilogue can drain
// while work tile k+1 accumulates in the other buffer.
// Every mbarrier wait is bounded; a wait that gives up sets the status word,
// and all roles fall through to the common exit, which waits for issued copies
// and MMAs before freeing TMEM.
#include <cuda.h>

#include <algorithm>
#include <cstdint>

#include "common.cuh"
#include "launch.h"
#include "schedule.h"
#include "tc.cuh"

namespace yoco {

static __device__ unsigned int g_status_prefill_tc;

namespace {

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr uint32_t kBlk = 128 * 128;  // one [128 rows x 128 bytes] swizzled block

template <int D>
struct Smem {
    static constexpr int KB = D / 64;                  // 64-element column blocks
    static constexpr uint32_t TILE = (uint32_t)KB * kBlk;
    static constexpr int KSTAGES = 3;
    static constexpr int VSTAGES = 2;
    static constexpr uint32_t Q = 0;                   // 2 buffers
    static constexpr uint32_t K = Q + 2 * TILE;        // KSTAGES stages
    static constexpr uint32_t V = K + KSTAGES * TILE;  // VSTAGES stages
    static constexpr uint32_t BAR = V + VSTAGES * TILE;
    static constexpr uint32_t BYTES = BAR + 256;
    static constexpr uint32_t ALLOC = BYTES + 1024;    // alignment slack
};

struct TcParams {
    sched::PrefillShape s;
    float scale_log2;
    void *o;
    float *lse;
    int32_t n_work;
};

enum Bar {
    kQFull = 0,    // 2
    kQEmpty = 2,   // 2
    kKFull = 4,    // 3
    kKEmpty = 7,   // 3
    kVFull = 10,   // 2
    kVEmpty = 12,  // 2
    kSFull = 14,   // 2: S of tile g in buffer g&1 ready
    kPFull = 16,   // 2: P of tile g written
    kODone = 18,   // 2: P.V of tile g finished
    kOFree = 20,   // 2: O buffer drained by the epilogue
    kDrain = 22,
    kNumBars = 23
};

YOCO_DEV bool wait1(uint64_t *bar, uint32_t parity) {
    return mbar_wait(bar, parity, &g_status_prefill_tc);
}
YOCO_DEV bool waitw(uint64_t *bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, &g_status_prefill_tc));
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const TcParams p) {
    // once any CTA has recorded a timeout, the rest of the grid exits at once
    if (*(volatile unsigned int *)&g_status_prefill_tc) return;
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
    if (warp == 5) {
        tc::tmem_alloc(tmem_slot, kTmemCols);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS0 = tmem, tS1 = tmem + 128;
    const uint32_t tO0 = tmem + 256, tO1 = tmem + 384;

    if (warp == 4) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int gk = 0, k = 0;  // K tiles issued, Q tiles issued
            for (int r = 0; !*abort_flag; ++r) {
                const int w = sched::prefill_work_index(r, blockIdx.x, gridDim.x);
                if (w >= p.n_work) break;
                const sched::PrefillWork x = sched::prefill_work(p.s, w);
                if (!wait1(&bars[kQEmpty + (k & 1)], ((k >> 1) & 1) ^ 1)) { *abort_flag = 1; break; }
                mbar_arrive_expect_tx(&bars[kQFull + (k & 1)], BM * D * 2);
                for (int kb = 0; kb < KB; ++kb)
                    tc::tma_load_4d(base + L::Q + (k & 1) * L::TILE + kb * kBlk, &tm_q, kb * 64, x.h,
                                    (int)x.i0, x.b, &bars[kQFull + (k & 1)]);
                ++k;
                for (int t = 0; t < x.n_kv; ++t, ++gk) {
                    const int st = gk % L::KSTAGES;
                    if (!wait1(&bars[kKEmpty + st], ((gk / L::KSTAGES) & 1) ^ 1)) { *abort_flag = 1; break; }
                    if (*abort_flag) break;
                    mbar_arrive_expect_tx(&bars[kKFull + st], BN * D * 2);
                    for (int kb = 0; kb < KB; ++kb)
                        tc::tma_load_4d(base + L::K + st * L::TILE + kb * kBlk, &tm_k, kb * 64, x.g,
                                        (x.jt_lo + t) * BN, x.b, &bars[kKFull + st]);
                }
                if (*abort_flag) break;
            }
            // drain: the last copies issued must land before this CTA may exit
            for (int q = max(0, gk - L::KSTAGES); q < gk; ++q)
                if (!wait1(&bars[kKFull + q % L::KSTAGES], (q / L::KSTAGES) & 1)) break;
            for (int q = max(0, k - 2); q < k; ++q)
                if (!wait1(&bars[kQFull + (q & 1)], (q >> 1) & 1)) break;
        } else if (lane == 1) {
            int gv = 0;
            for (int r = 0; !*abort_flag; ++r) {
                const int w = sched::prefill_work_index(r, blockIdx.x, gridDim.x);
                if (w >= p.n_work) break;
                const sched::PrefillWork x = sched::prefill_work(p.s, w);
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
    } else if (warp == 5) {
        // ---------------------------------------------------------- MMA issue
        if (lane == 0) {
            constexpr uint32_t idS = tc::idesc_bf16(BM, BN, false, false);
            constexpr uint32_t idPV = tc::idesc_bf16(BM, D, false, true);
            bool ok = true;
            // the P.V owed for the previous KV tile: its tile counter, work
            // counter and whether it is the first of its work tile
            int pend_g = -1, pend_k = 0;
            bool pend_first = false;
            auto issue_pv = [&]() -> bool {
                const int u = pend_g, kk_ = pend_k;
                const int vs = u % L::VSTAGES;
                if (pend_first && kk_ >= 2 && !wait1(&bars[kOFree + (kk_ & 1)], ((kk_ - 2) >> 1) & 1))
                    return false;
                if (!wait1(&bars[kPFull + (u & 1)], (u >> 1) & 1)) return false;
                if (!wait1(&bars[kVFull + vs], (u / L::VSTAGES) & 1)) return false;
                tc::fence_after_sync();
                const uint32_t vb = base + L::V + vs * L::TILE;
                const uint32_t tp = (u & 1) ? tS1 : tS0;   // P aliases the first 64 columns of S
                const uint32_t to = (kk_ & 1) ? tO1 : tO0;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk)
                    tc::mma_bf16_ts(to, tp + kk * 8, tc::smem_desc_sw128(vb + kk * 2048, kBlk, 1024), idPV,
                                    (!pend_first || kk > 0) ? 1u : 0u);
                tc::mma_commit(&bars[kVEmpty + vs]);
                tc::mma_commit(&bars[kODone + (u & 1)]);
                pend_g = -1;
                return true;
            };
            int gk = 0;
            for (int k = 0; ok; ++k) {
                const int w = sched::prefill_work_index(k, blockIdx.x, gridDim.x);
                if (w >= p.n_work) break;
                const sched::PrefillWork x = sched::prefill_work(p.s, w);
                if (!wait1(&bars[kQFull + (k & 1)], (k >> 1) & 1)) { ok = false; break; }
                const uint32_t qb = base + L::Q + (k & 1) * L::TILE;
                for (int t = 0; t < x.n_kv; ++t, ++gk) {
                    const int st = gk % L::KSTAGES;
                    if (!wait1(&bars[kKFull + st], (gk / L::KSTAGES) & 1) || *abort_flag) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t kbase = base + L::K + st * L::TILE;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kBlk + (kk & 3) * 32;
                        tc::mma_bf16_ss((gk & 1) ? tS1 : tS0, tc::smem_desc_sw128(qb + off, 16, 1024),
                                        tc::smem_desc_sw128(kbase + off, 16, 1024), idS, kk > 0 ? 1u : 0u);
                    }
                    tc::mma_commit(&bars[kKEmpty + st]);
                    tc::mma_commit(&bars[kSFull + (gk & 1)]);
                    if (t == x.n_kv - 1) tc::mma_commit(&bars[kQEmpty + (k & 1)]);
                    if (pend_g >= 0 && !issue_pv()) { ok = false; break; }
                    pend_g = gk;
                    pend_k = k;
                    pend_first = (t == 0);
                }
            }
            if (ok && pend_g >= 0 && !*abort_flag && !issue_pv()) ok = false;
            if (!ok) *abort_flag = 1;
            // every MMA issued by this thread has finished before TMEM is freed
            tc::mma_commit(&bars[kDrain]);
            wait1(&bars[kDrain], 0);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int r = threadIdx.x;                 // row in tile == TMEM lane
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint64_t sl2 = tc::f2_pack(p.scale_log2, p.scale_log2);
        bool ok = true;
        uint32_t pk[BN / 2];
        int gk = 0;
        for (int k = 0; ok; ++k) {
            const int w = sched::prefill_work_index(k, blockIdx.x, gridDim.x);
            if (w >= p.n_work) break;
            const sched::PrefillWork x = sched::prefill_work(p.s, w);
            const int64_t i = x.i0 + r;
            const int64_t pos = p.s.q_pos0 + i;
            const uint32_t tO = ((k & 1) ? tO1 : tO0) + lane_off;
            float m = -INFINITY, l = 0.f;
            for (int t = 0; t < x.n_kv; ++t, ++gk) {
                if (!waitw(&bars[kSFull + (gk & 1)], (gk >> 1) & 1)) { ok = false; break; }
                tc::fence_after_sync();
                const uint32_t tS = ((gk & 1) ? tS1 : tS0) + lane_off;
                float s[BN];
#pragma unroll
                for (int c = 0; c < BN; c += 32) tc::tmem_ld32(tS + c, s + c);
                tc::wait_ld();
                const int64_t j0 = (int64_t)(x.jt_lo + t) * BN;
                if (sched::prefill_tile_masked(p.s, x, t)) {
                    // visible columns of this row form one range [c_lo, c_hi): one
                    // unsigned compare per element against 32-bit bounds
                    const int64_t dg = pos - j0;
                    const int c_hi = (int)max((int64_t)0, min(min(dg + 1, p.s.Tkv - j0), (int64_t)BN));
                    const int c_lo = p.s.window > 0 ? (int)max((int64_t)0, min(dg - p.s.window + 1, (int64_t)BN)) : 0;
                    const unsigned width = (unsigned)max(0, c_hi - c_lo);
#pragma unroll
                    for (int c = 0; c < BN; ++c)
                        s[c] = (unsigned)(c - c_lo) < width ? s[c] : -INFINITY;
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
                // P = 2^(S * scale * log2e - m): scale on packed pairs; exponentials
                // split between MUFU and the FMA-pipe polynomial (columns 48-63 and
                // 112-127, a quarter: the split measured fastest, since MUFU and
                // the issue slots then run out at about the same time)
                const uint64_t nm2 = tc::f2_pack(neg_m, neg_m);
                uint64_t rs2a = 0, rs2b = 0;
#pragma unroll
                for (int c = 0; c < BN; c += 2) {
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
                    pk[c / 2] = tc::pack_bf16x2(e0, e1);
                }
                float ra0, ra1, rb0, rb1;
                tc::f2_unpack(rs2a, ra0, ra1);
                tc::f2_unpack(rs2b, rb0, rb1);
                l = l * alpha + ((ra0 + ra1) + (rb0 + rb1));
                // O must hold the previous tile's P.V before it is rescaled
                if (t >= 1 && __any_sync(0xffffffffu, grow)) {
                    if (!waitw(&bars[kODone + ((gk - 1) & 1)], ((gk - 1) >> 1) & 1)) { ok = false; break; }
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
                    tc::wait_st();
                }
                // P row r (bf16 pairs) over the first 64 columns of this S buffer
                tc::tmem_st32u(tS, pk);
                tc::tmem_st32u(tS + 32, pk + 32);
                tc::wait_st();
                tc::fence_before_sync();
                mbar_arrive(&bars[kPFull + (gk & 1)]);
            }
            if (!ok) break;
            // epilogue: the last P.V of this work tile, then O / l -> global
            const int gl = gk - 1;
            if (!waitw(&bars[kODone + (gl & 1)], (gl >> 1) & 1)) { ok = false; break; }
            tc::fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.o) +
                                 (((int64_t)x.b * p.s.Tq + i) * p.s.Hq + x.h) * D;
#pragma unroll
            for (int c = 0; c < D; c += 32) {
                float o[32];
                tc::tmem_ld32(tO + c, o);
                tc::wait_ld();
                if (i < p.s.Tq) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 wv;
                        wv.x = tc::pack_bf16x2(o[e] * inv, o[e + 1] * inv);
                        wv.y = tc::pack_bf16x2(o[e + 2] * inv, o[e + 3] * inv);
                        wv.z = tc::pack_bf16x2(o[e + 4] * inv, o[e + 5] * inv);
                        wv.w = tc::pack_bf16x2(o[e + 6] * inv, o[e + 7] * inv);
                        *reinterpret_cast<uint4 *>(dst + c + e) = wv;
                    }
                }
            }
            if (p.lse && i < p.s.Tq)
                p.lse[((int64_t)x.b * p.s.Hq + x.h) * p.s.Tq + i] = l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
            tc::fence_before_sync();
            mbar_arrive(&bars[kOFree + (k & 1)]);
        }
        if (!ok) *abort_flag = 1;
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 5) {
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
cudaError_t launch_tc_d(const PrefillArgs &a, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.B, a.Tq, a.Hq, D) || !make_map(&mk, a.k, a.B, a.Tkv, a.Hkv, D) ||
        !make_map(&mv, a.v, a.B, a.Tkv, a.Hkv, D))
        return cudaErrorNotSupported;
    TcParams p;
    p.s.B = a.B; p.s.Hq = a.Hq; p.s.Hkv = a.Hkv;
    p.s.Tq = a.Tq; p.s.Tkv = a.Tkv; p.s.q_pos0 = a.q_pos0; p.s.window = a.window;
    p.scale_log2 = a.scale * kLog2e;
    p.o = a.o; p.lse = a.lse;
    const int64_t n_qtiles = (a.Tq + BM - 1) / BM;
    const int64_t n_work = n_qtiles * a.Hq * a.B;
    if (n_work > INT32_MAX / 2) return cudaErrorNotSupported;
    p.s.n_qtiles = (int)n_qtiles;
    p.n_work = (int)n_work;
    const int grid = (int)std::min<int64_t>(n_work, device_sm_count());
    p.s.band = sched::prefill_band(grid, a.Hq / a.Hkv, (int64_t)a.B * a.Tkv * a.Hkv * D * 2 * 2, a.window);
    auto kern = attn_prefill_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Smem<D>::ALLOC);
    if (e != cudaSuccess) return e;
    note_launches(1);
    kern<<<grid, kThreads, Smem<D>::ALLOC, st>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t st) {
    if (a.dtype != kBF16) return cudaErrorNotSupported;
    if (a.B == 0 || a.Tq == 0) return cudaSuccess;
    if (a.D == 128) return launch_tc_d<128>(a, st);
    if (a.D == 64) return launch_tc_d<64>(a, st);
    return cudaErrorNotSupported;
}

unsigned int read_and_clear_status_prefill_tc() {
    unsigned int h = 0, z = 0;
    if (cudaMemcpyFromSymbol(&h, g_status_prefill_tc, sizeof(h)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_status_prefill_tc, &z, sizeof(z));
    return h;
}

}  // namespace yoco
