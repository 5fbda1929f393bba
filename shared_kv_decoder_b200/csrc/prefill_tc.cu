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
// Per CTA: one 128-row query tile of one (batch, query head); KV tiles of 128
// keys of the matching KV head.  Warp roles:
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r).  For each KV
//              tile it reads S from TMEM, masks (diagonal / window / tail tiles
//              only), takes the row max (3-input max tree), computes
//              P = 2^(S*scale*log2e - m) in fp32 on packed pairs -- three
//              quarters of the exponentials on MUFU, a quarter on an FMA-pipe
//              polynomial -- and writes P as bf16 pairs back into TMEM (two P
//              buffers).  The
//              running max is only moved (and O in TMEM rescaled) when it grows
//              by more than 2^8, which keeps O exact after the final 1/l.
//   warp 4     TMA producer: lane 0 loads Q then K tiles, lane 1 V tiles,
//              into a three-deep ring each (mbarrier complete_tx).
//   warp 5     MMA issuer (one thread): S_t = Q K_t^T into one of two TMEM S
//              buffers, issued one tile ahead so the tensor core computes
//              S_{t+1} while the softmax works on S_t; then O += P_t V_t with
//              P read from TMEM (A operand in tensor memory) and V read
//              MN-major straight from its TMA tile.  Keeping P out of shared
//              memory matters: at N = 128 the operand reads of one MMA already
//              use the whole shared-memory bandwidth.
// TMEM: S0, S1 [128 x 128] fp32, O [128 x D] fp32, P0, P1 [128 x 128] bf16
// (512 columns allocated).
// Every mbarrier wait is bounded; a wait that gives up sets the status word,
// and all roles then fall through to the common exit, which waits for issued
// copies and MMAs before freeing TMEM.
#include <cuda.h>

#include "common.cuh"
#include "launch.h"
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
    static constexpr int STAGES = 3;
    static constexpr uint32_t Q = 0;
    static constexpr uint32_t K = Q + TILE;            // STAGES stages
    static constexpr uint32_t V = K + STAGES * TILE;   // STAGES stages
    static constexpr uint32_t BAR = V + STAGES * TILE;
    static constexpr uint32_t BYTES = BAR + 256;
    static constexpr uint32_t ALLOC = BYTES + 1024;    // alignment slack
};

struct TcParams {
    int32_t B, Hq, Hkv;
    int64_t Tq, Tkv, q_pos0;
    int32_t window;
    float scale_log2;
    void *o;
    float *lse;
    int32_t n_qtiles;
};

enum Bar {
    kQFull = 0,
    kKFull = 1,   // 3
    kKEmpty = 4,  // 3
    kVFull = 7,   // 3
    kVEmpty = 10, // 3
    kSFull = 13,  // 2
    kPFull = 15,  // 2: P buffer t&1 written (tile t)
    kODone = 17,  // 2: P.V of tile u (P buffer u&1) finished
    kDrain = 19,
    kNumBars = 20
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
    using L = Smem<D>;
    constexpr int KB = L::KB;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sbase = smem_raw + (base - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sbase + L::BAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sbase + L::BAR + kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sbase + L::BAR + kNumBars * 8 + 4);

    // once any CTA has recorded a timeout, the rest of the grid exits at once
    if (*(volatile unsigned int *)&g_status_prefill_tc) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x, b = blockIdx.y;
    const int qt = p.n_qtiles - 1 - (int)blockIdx.z;  // heaviest causal tiles first
    const int g = h / (p.Hq / p.Hkv);
    const int64_t i0 = (int64_t)qt * BM;
    const int64_t i_last = min(i0 + BM, p.Tq) - 1;
    const int64_t p_first = p.q_pos0 + i0, p_last = p.q_pos0 + i_last;
    const int64_t j_lo = p.window > 0 ? max((int64_t)0, p_first - p.window + 1) : 0;
    const int64_t j_hi = min(p.Tkv - 1, p_last);
    const int jt_lo = (int)(j_lo / BN);
    const int n_kv = (int)(j_hi / BN) - jt_lo + 1;

    if (threadIdx.x == 0) {
        mbar_init(&bars[kQFull], 1);
        for (int s = 0; s < L::STAGES; ++s) {
            mbar_init(&bars[kKFull + s], 1);
            mbar_init(&bars[kKEmpty + s], 1);
            mbar_init(&bars[kVFull + s], 1);
            mbar_init(&bars[kVEmpty + s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kSFull + s], 1);
            mbar_init(&bars[kPFull + s], 128);
            mbar_init(&bars[kODone + s], 1);
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
    // TMEM columns: S0 [0,128) S1 [128,256) O [256,256+D) P0 [384,448) P1 [448,512)
    const uint32_t tS0 = tmem, tS1 = tmem + 128;
    const uint32_t tO = tmem + 256;
    const uint32_t tP0 = tmem + 384, tP1 = tmem + 448;

    if (warp == 4) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            int issued = 0;
            mbar_arrive_expect_tx(&bars[kQFull], BM * D * 2);
            for (int kb = 0; kb < KB; ++kb)
                tc::tma_load_4d(base + L::Q + kb * kBlk, &tm_q, kb * 64, h, (int)i0, b, &bars[kQFull]);
            for (int t = 0; t < n_kv; ++t) {
                const int st = t % L::STAGES;
                if (!wait1(&bars[kKEmpty + st], ((t / L::STAGES) & 1) ^ 1)) { *abort_flag = 1; break; }
                if (*abort_flag) break;
                mbar_arrive_expect_tx(&bars[kKFull + st], BN * D * 2);
                const int j0 = (jt_lo + t) * BN;
                for (int kb = 0; kb < KB; ++kb)
                    tc::tma_load_4d(base + L::K + st * L::TILE + kb * kBlk, &tm_k, kb * 64, g, j0, b,
                                    &bars[kKFull + st]);
                ++issued;
            }
            // drain: the last copies issued must land before this CTA may exit
            for (int t = max(0, issued - L::STAGES); t < issued; ++t)
                if (!wait1(&bars[kKFull + t % L::STAGES], (t / L::STAGES) & 1)) break;
            wait1(&bars[kQFull], 0);
        } else if (lane == 1) {
            int issued = 0;
            for (int t = 0; t < n_kv; ++t) {
                const int st = t % L::STAGES;
                if (!wait1(&bars[kVEmpty + st], ((t / L::STAGES) & 1) ^ 1)) { *abort_flag = 1; break; }
                if (*abort_flag) break;
                mbar_arrive_expect_tx(&bars[kVFull + st], BN * D * 2);
                const int j0 = (jt_lo + t) * BN;
                for (int kb = 0; kb < KB; ++kb)
                    tc::tma_load_4d(base + L::V + st * L::TILE + kb * kBlk, &tm_v, kb * 64, g, j0, b,
                                    &bars[kVFull + st]);
                ++issued;
            }
            for (int t = max(0, issued - L::STAGES); t < issued; ++t)
                if (!wait1(&bars[kVFull + t % L::STAGES], (t / L::STAGES) & 1)) break;
        }
    } else if (warp == 5) {
        // ---------------------------------------------------------- MMA issue
        if (lane == 0) {
            constexpr uint32_t idS = tc::idesc_bf16(BM, BN, false, false);
            constexpr uint32_t idPV = tc::idesc_bf16(BM, D, false, true);
            bool ok = wait1(&bars[kQFull], 0);
            auto issue_pv = [&](int u) -> bool {
                const int vs = u % L::STAGES;
                if (!wait1(&bars[kPFull + (u & 1)], (u >> 1) & 1)) return false;
                if (!wait1(&bars[kVFull + vs], (u / L::STAGES) & 1)) return false;
                tc::fence_after_sync();
                const uint32_t vb = base + L::V + vs * L::TILE;
                const uint32_t tp = (u & 1) ? tP1 : tP0;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t bd = tc::smem_desc_sw128(vb + kk * 2048, kBlk, 1024);
                    tc::mma_bf16_ts(tO, tp + kk * 8, bd, idPV, (u > 0 || kk > 0) ? 1u : 0u);
                }
                tc::mma_commit(&bars[kVEmpty + vs]);
                tc::mma_commit(&bars[kODone + (u & 1)]);
                return true;
            };
            for (int t = 0; ok && t < n_kv; ++t) {
                const int st = t % L::STAGES;
                if (!wait1(&bars[kKFull + st], (t / L::STAGES) & 1) || *abort_flag) { ok = false; break; }
                tc::fence_after_sync();
                const uint32_t kbase = base + L::K + st * L::TILE;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBlk + (kk & 3) * 32;
                    const uint64_t ad = tc::smem_desc_sw128(base + L::Q + off, 16, 1024);
                    const uint64_t bd = tc::smem_desc_sw128(kbase + off, 16, 1024);
                    tc::mma_bf16_ss((t & 1) ? tS1 : tS0, ad, bd, idS, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&bars[kKEmpty + st]);
                tc::mma_commit(&bars[kSFull + (t & 1)]);
                if (t >= 1 && !issue_pv(t - 1)) { ok = false; break; }
            }
            if (ok && !*abort_flag) ok = issue_pv(n_kv - 1);
            if (!ok) *abort_flag = 1;
            // every MMA issued by this thread has finished before TMEM is freed
            tc::mma_commit(&bars[kDrain]);
            wait1(&bars[kDrain], 0);
        }
    } else {
        // ------------------------------------------------------------ softmax
        const int r = threadIdx.x;                 // row in tile == TMEM lane
        const int64_t i = i0 + r;
        const int64_t pos = p.q_pos0 + i;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        uint32_t pk[BN / 2];
        for (int t = 0; t < n_kv; ++t) {
            if (!waitw(&bars[kSFull + (t & 1)], (t >> 1) & 1)) { ok = false; break; }
            tc::fence_after_sync();
            float s[BN];
#pragma unroll
            for (int c = 0; c < BN; c += 32) tc::tmem_ld32(((t & 1) ? tS1 : tS0) + lane_off + c, s + c);
            tc::wait_ld();
            const int64_t j0 = (int64_t)(jt_lo + t) * BN;
            const bool need_mask = (j0 + BN - 1 > p_first) || (j0 + BN > p.Tkv) ||
                                   (p.window > 0 && j0 <= p_last - p.window);
            if (need_mask) {
#pragma unroll
                for (int c = 0; c < BN; ++c) {
                    const int64_t j = j0 + c;
                    const bool vis = j <= pos && j < p.Tkv && (p.window <= 0 || j > pos - p.window);
                    s[c] = vis ? s[c] : -INFINITY;
                }
            }
            // row max: 3-input max tree, eight independent chains
            float a8[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) a8[k] = tc::max3(s[k], s[k + 8], s[k + 16]);
#pragma unroll
            for (int c = 24; c < 120; c += 16)
#pragma unroll
                for (int k = 0; k < 8; ++k) a8[k] = tc::max3(a8[k], s[c + k], s[c + 8 + k]);
#pragma unroll
            for (int k = 0; k < 8; ++k) a8[k] = fmaxf(a8[k], s[120 + k]);
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
            // 112-127, a quarter: the split measured fastest, since MUFU and the
            // issue slots then run out at about the same time)
            const uint64_t sl2 = tc::f2_pack(p.scale_log2, p.scale_log2);
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
            // O must hold P_{t-1} V before it is rescaled
            if (t >= 1 && __any_sync(0xffffffffu, grow)) {
                if (!waitw(&bars[kODone + ((t - 1) & 1)], ((t - 1) >> 1) & 1)) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll
                for (int c = 0; c < D; c += 32) {
                    float o[32];
                    tc::tmem_ld32(tO + lane_off + c, o);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= alpha;
                    tc::tmem_st32(tO + lane_off + c, o);
                }
                tc::wait_st();
            }
            // P buffer t&1 in TMEM is free once P_{t-2} V has finished
            if (t >= 2) {
                if (!waitw(&bars[kODone + (t & 1)], ((t - 2) >> 1) & 1)) { ok = false; break; }
            }
            // P row r (bf16 pairs) -> TMEM lane r, 64 columns of buffer t&1
            const uint32_t tp = ((t & 1) ? tP1 : tP0) + lane_off;
            tc::tmem_st32u(tp, pk);
            tc::tmem_st32u(tp + 32, pk + 32);
            tc::wait_st();
            tc::fence_before_sync();
            mbar_arrive(&bars[kPFull + (t & 1)]);
        }
        if (ok && waitw(&bars[kODone + ((n_kv - 1) & 1)], ((n_kv - 1) >> 1) & 1)) {
            tc::fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.o) +
                                 (((int64_t)b * p.Tq + i) * p.Hq + h) * D;
#pragma unroll
            for (int c = 0; c < D; c += 32) {
                float o[32];
                tc::tmem_ld32(tO + lane_off + c, o);
                tc::wait_ld();
                if (i < p.Tq) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 w;
                        w.x = tc::pack_bf16x2(o[e] * inv, o[e + 1] * inv);
                        w.y = tc::pack_bf16x2(o[e + 2] * inv, o[e + 3] * inv);
                        w.z = tc::pack_bf16x2(o[e + 4] * inv, o[e + 5] * inv);
                        w.w = tc::pack_bf16x2(o[e + 6] * inv, o[e + 7] * inv);
                        *reinterpret_cast<uint4 *>(dst + c + e) = w;
                    }
                }
            }
            if (p.lse && i < p.Tq)
                p.lse[((int64_t)b * p.Hq + h) * p.Tq + i] = l > 0.f ? (m + __log2f(l)) * kLn2 : -INFINITY;
        } else {
            *abort_flag = 1;
        }
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 4-D bf16 map over [B, T, H, D] (innermost D), box {64, 1, 128, 1}, 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *ptr, int64_t B, int64_t T, int64_t H, int64_t D) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)(D * 2), (cuuint64_t)(H * D * 2), (cuuint64_t)(T * H * D * 2)};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_tc_d(const PrefillArgs &a, cudaStream_t st) {
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.B, a.Tq, a.Hq, D) || !make_map(&mk, a.k, a.B, a.Tkv, a.Hkv, D) ||
        !make_map(&mv, a.v, a.B, a.Tkv, a.Hkv, D))
        return cudaErrorNotSupported;
    TcParams p;
    p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv;
    p.Tq = a.Tq; p.Tkv = a.Tkv; p.q_pos0 = a.q_pos0; p.window = a.window;
    p.scale_log2 = a.scale * kLog2e;
    p.o = a.o; p.lse = a.lse;
    p.n_qtiles = (int)((a.Tq + BM - 1) / BM);
    if (p.n_qtiles > 65535) return cudaErrorNotSupported;
    auto kern = attn_prefill_tc_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Smem<D>::ALLOC);
    if (e != cudaSuccess) return e;
    dim3 grid(a.Hq, a.B, p.n_qtiles);
    note_launches(1);
    kern<<<grid, kThreads, Smem<D>::ALLOC, st>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t st) {
    if (a.dtype != kBF16) return cudaErrorNotSupported;
    if (a.B == 0 || a.Tq == 0) return cudaSuccess;
    if (a.B > 65535 || a.Hq > 65535) return cudaErrorNotSupported;
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
