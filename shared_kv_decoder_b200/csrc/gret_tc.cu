// Gated retention chunkwise prefill on the sm_100a tensor cores (bf16 in,
// fp32 state and accumulation), D = 128.  The same computation as
// gret_prefill_kernel in gret.cu ("You Only Cache Once", paperlayer summary,
// section 3 "Gated Retention" and Appendix B; podcast transcript cue 16):
// per head, S_t = gamma_t S_{t-1} + scale k_t^T v_t and o_t = q_t S_t, taken
// in chunks of 128 tokens.  With c_r the running sum of log gamma over the
// chunk's rows 0..r (base-2 units here):
//   o_r   = sum_{u<=r} 2^{c_r - c_u} scale (q_r . k_u) v_u   +  2^{c_r} q_r S_prev
//   S_new = 2^{c_last} S_prev + sum_u 2^{c_last - c_u} scale k_u^T v_u
// Every exponent is <= 0.
//
// One CTA per (batch, head) walks the chunks in order.  TMEM (512 columns):
//   A/P [0,128)   Q K^T of the chunk, then the decayed, masked P (bf16, first 64)
//   O   [128,256) P V
//   X   [256,384) Q S_prev
//   S   [384,512) the fp32 state (row d = lane d)
// Shared memory: the chunk's Q, K and V tiles (TMA, 128-byte swizzle), K_w
// (K scaled by scale * 2^{c_last - c_u}), and S_prev split into bf16 high and
// low parts laid out like a V tile (about 16 mantissa bits for the cross term).
// Warp roles (320 threads):
//   warps 0-3  output: P from A (decay mask), then o = O + 2^{c_r} X -> global
//   warps 4-7  state: K_w, S *= 2^{c_last} in TMEM, and after the update the
//              high / low split of S into shared memory for the next chunk
//   warp 8     TMA: lane 0 Q tiles, lane 1 K tiles, lane 2 V tiles
//   warp 9     MMA issuer: A = Q K^T; X = Q S_hi + Q S_lo; O = P V;
//              S += K_w^T V (A operand MN-major from the K_w tile)
// Every mbarrier wait is bounded; a wait that gives up sets the status word,
// and all roles fall through to the common exit, which waits for issued
// copies and MMAs before freeing TMEM.
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
constexpr int kThreads = 320;
constexpr uint32_t kBlk = 128 * 128;      // one [128 rows x 128 bytes] swizzled block
constexpr uint32_t kTile = 2 * kBlk;      // a [128, 128] bf16 tile (two 64-column blocks)

enum Smem : uint32_t {
    kQ = 0,
    kK = kQ + kTile,
    kV = kK + kTile,
    kKw = kV + kTile,
    kShi = kKw + kTile,
    kSlo = kShi + kTile,
    kC2 = kSlo + kTile,                   // 8 warps x 128 floats of running sums
    kBars = kC2 + 8 * kC * 4,
    kBytes = kBars + 256,
    kAlloc = kBytes + 1024,
};

enum Bar {
    kQFull = 0, kKFull, kVFull,
    kQEmpty, kKEmpty, kVEmpty,
    kAFull,       // Q K^T done
    kPFull,       // P written (128 arrivals)
    kOFull,       // P V (and the cross term before it) done
    kOFree,       // O and X read out (128 arrivals)
    kSScaled,     // K_w written and S decayed (128 arrivals)
    kSUpdated,    // S += K_w^T V done
    kSplit,       // S_hi / S_lo ready for the next chunk (128 arrivals)
    kDrain,
    kNumBars
};

struct GretTcParams {
    const float *g;
    float *state;
    __nv_bfloat16 *o;
    int32_t B, H;
    int64_t T;
    float lg_scale;   // log2(e) / tau
    float scale;
    int32_t n_chunks;
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
                   const __grid_constant__ CUtensorMap tm_v, const GretTcParams p) {
    if (*(volatile unsigned int *)&g_status_gret_tc) return;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sb = smem_raw + (base - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sb + kBars);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sb + kBars + kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sb + kBars + kNumBars * 8 + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int NC = p.n_chunks;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i)
            mbar_init(&bars[i], (i == kPFull || i == kOFree || i == kSScaled || i == kSplit) ? 128 : 1);
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
        if (lane < 3) {
            const CUtensorMap *map = lane == 0 ? &tm_q : lane == 1 ? &tm_k : &tm_v;
            const uint32_t dst = base + (lane == 0 ? kQ : lane == 1 ? kK : kV);
            uint64_t *full = &bars[kQFull + lane], *empty = &bars[kQEmpty + lane];
            int j = 0;
            for (; j < NC && !*abort_flag; ++j) {
                if (j > 0 && !wait1(empty, (j - 1) & 1)) { *abort_flag = 1; break; }
                mbar_arrive_expect_tx(full, kC * kD * 2);
                for (int kb = 0; kb < 2; ++kb)
                    tc::tma_load_4d(dst + kb * kBlk, map, kb * 64, h, j * kC, b, full);
            }
            if (j > 0) wait1(full, (j - 1) & 1);  // the last copy has landed before exit
        }
    } else if (warp == 9) {
        // ---------------------------------------------------------- MMA issue
        if (lane == 0) {
            constexpr uint32_t idQK = tc::idesc_bf16(128, 128, false, false);
            constexpr uint32_t idMNB = tc::idesc_bf16(128, 128, false, true);
            constexpr uint32_t idUpd = tc::idesc_bf16(128, 128, true, true);
            bool ok = true;
            for (int j = 0; ok && j < NC; ++j) {
                const uint32_t ph = j & 1;
                // A = Q K^T
                if (!wait1(&bars[kQFull], ph) || !wait1(&bars[kKFull], ph) || *abort_flag) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kBlk + (kk & 3) * 32;
                    tc::mma_bf16_ss(tA, tc::smem_desc_sw128(base + kQ + off, 16, 1024),
                                    tc::smem_desc_sw128(base + kK + off, 16, 1024), idQK, kk > 0 ? 1u : 0u);
                }
                tc::mma_commit(&bars[kAFull]);
                // X = Q S_prev (high and low parts); X and O must have been read out
                if (!wait1(&bars[kSplit], ph)) { ok = false; break; }
                if (j > 0 && !wait1(&bars[kOFree], (j - 1) & 1)) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll
                for (int part = 0; part < 2; ++part) {
                    const uint32_t sm = base + (part == 0 ? kShi : kSlo);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kBlk + (kk & 3) * 32;
                        tc::mma_bf16_ss(tX, tc::smem_desc_sw128(base + kQ + off, 16, 1024),
                                        tc::smem_desc_sw128(sm + kk * 2048, kBlk, 1024), idMNB,
                                        (part > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                tc::mma_commit(&bars[kQEmpty]);
                // O = P V
                if (!wait1(&bars[kPFull], ph) || !wait1(&bars[kVFull], ph)) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    tc::mma_bf16_ts(tO, tA + kk * 8, tc::smem_desc_sw128(base + kV + kk * 2048, kBlk, 1024), idMNB,
                                    kk > 0 ? 1u : 0u);
                tc::mma_commit(&bars[kOFull]);
                // S += K_w^T V
                if (!wait1(&bars[kSScaled], ph)) { ok = false; break; }
                tc::fence_after_sync();
                tc::mma_commit(&bars[kKEmpty]);   // the state warps are done reading K
#pragma unroll
                for (int kk = 0; kk < kC / 16; ++kk)
                    tc::mma_bf16_ss(tS, tc::smem_desc_sw128(base + kKw + kk * 2048, kBlk, 1024),
                                    tc::smem_desc_sw128(base + kV + kk * 2048, kBlk, 1024), idUpd, 1u);
                tc::mma_commit(&bars[kVEmpty]);
                tc::mma_commit(&bars[kSUpdated]);
            }
            if (!ok) *abort_flag = 1;
            tc::mma_commit(&bars[kDrain]);
            wait1(&bars[kDrain], 0);
        }
    } else {
        // ------------------------------------------- output and state warps
        const bool state_role = warp >= 4;
        const int r = (warp & 3) * 32 + lane;                 // TMEM lane = chunk row / state row
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        float *c2w = reinterpret_cast<float *>(sb + kC2) + warp * kC;
        const float *gb = p.g + (int64_t)b * p.T * p.H + h;
        bool ok = true;

        if (state_role) {
            // initial state: TMEM rows, then the high / low split for chunk 0
            const float *s0 = p.state ? p.state + ((int64_t)b * p.H + h) * kD * kD + (int64_t)r * kD : nullptr;
#pragma unroll
            for (int c = 0; c < kD; c += 32) {
                float v[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] = s0 ? s0[c + e] : 0.f;
                tc::tmem_st32(tS + lane_off + c, v);
            }
            tc::wait_st();
        }

        for (int j = 0; ok && j < NC; ++j) {
            const uint32_t ph = j & 1;
            const int64_t t0 = (int64_t)j * kC;
            // running base-2 log-decay sums of the chunk, computed by every warp
            // for itself (lane l: rows 4l..4l+3; padded rows decay by 1)
            __syncwarp();  // the previous chunk's reads of this warp's copy are done
            {
                float x[4], run = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int64_t t = t0 + 4 * lane + i;
                    run += t < p.T ? log2_decay(gb[t * p.H], p.lg_scale) : 0.f;
                    x[i] = run;
                }
                float incl = run;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += y;
                }
                const float excl = incl - run;
#pragma unroll
                for (int i = 0; i < 4; ++i) c2w[4 * lane + i] = excl + x[i];
                __syncwarp();
            }
            const float c_r = c2w[r], c_last = c2w[kC - 1];

            if (!state_role) {
                // ---- P = scale * 2^{c_r - c_u} A for u <= r, else 0
                if (!waitw(&bars[kAFull], ph)) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    float a[64];
                    tc::tmem_ld32(tA + lane_off + half * 64, a);
                    tc::tmem_ld32(tA + lane_off + half * 64 + 32, a + 32);
                    tc::wait_ld();
                    uint32_t pk[32];
#pragma unroll
                    for (int u2 = 0; u2 < 64; u2 += 2) {
                        const int u = half * 64 + u2;
                        const float w0 = u <= r ? p.scale * tc::ex2(c_r - c2w[u]) : 0.f;
                        const float w1 = u + 1 <= r ? p.scale * tc::ex2(c_r - c2w[u + 1]) : 0.f;
                        pk[u2 / 2] = tc::pack_bf16x2(a[u2] * w0, a[u2 + 1] * w1);
                    }
                    tc::tmem_st32u(tA + lane_off + half * 32, pk);
                }
                tc::wait_st();
                tc::fence_before_sync();
                mbar_arrive(&bars[kPFull]);
                // ---- o = O + 2^{c_r} X
                if (!waitw(&bars[kOFull], ph)) { ok = false; break; }
                tc::fence_after_sync();
                const float f = tc::ex2(c_r);
                __nv_bfloat16 *dst = p.o + (((int64_t)b * p.T + t0 + r) * p.H + h) * kD;
#pragma unroll
                for (int c = 0; c < kD; c += 32) {
                    float ov[32], xv[32];
                    tc::tmem_ld32(tO + lane_off + c, ov);
                    tc::tmem_ld32(tX + lane_off + c, xv);
                    tc::wait_ld();
                    if (t0 + r < p.T) {
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            uint4 w;
                            w.x = tc::pack_bf16x2(fmaf(f, xv[e], ov[e]), fmaf(f, xv[e + 1], ov[e + 1]));
                            w.y = tc::pack_bf16x2(fmaf(f, xv[e + 2], ov[e + 2]), fmaf(f, xv[e + 3], ov[e + 3]));
                            w.z = tc::pack_bf16x2(fmaf(f, xv[e + 4], ov[e + 4]), fmaf(f, xv[e + 5], ov[e + 5]));
                            w.w = tc::pack_bf16x2(fmaf(f, xv[e + 6], ov[e + 6]), fmaf(f, xv[e + 7], ov[e + 7]));
                            *reinterpret_cast<uint4 *>(dst + c + e) = w;
                        }
                    }
                }
                tc::fence_before_sync();
                mbar_arrive(&bars[kOFree]);
            } else {
                // ---- the state's split for this chunk's cross term (chunk 0: the
                // initial state; later: done at the end of the previous chunk)
                if (j == 0) {
#pragma unroll
                    for (int c = 0; c < kD; c += 32) {
                        float v[32];
                        tc::tmem_ld32(tS + lane_off + c, v);
                        tc::wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            uint4 hi, lo;
                            uint32_t *hp = &hi.x, *lp = &lo.x;
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float x0 = v[e + 2 * q], x1 = v[e + 2 * q + 1];
                                hp[q] = tc::pack_bf16x2(x0, x1);
                                lp[q] = tc::pack_bf16x2(x0 - __uint_as_float(hp[q] << 16),
                                                        x1 - __uint_as_float(hp[q] & 0xffff0000u));
                            }
                            *reinterpret_cast<uint4 *>(sb + kShi + sw_off(r, c + e)) = hi;
                            *reinterpret_cast<uint4 *>(sb + kSlo + sw_off(r, c + e)) = lo;
                        }
                    }
                    fence_proxy_async_smem();
                    tc::fence_before_sync();
                    mbar_arrive(&bars[kSplit]);
                }
                // ---- K_w = K * scale * 2^{c_last - c_u} (row u = r of the K tile)
                if (!waitw(&bars[kKFull], ph)) { ok = false; break; }
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
                // ---- S *= 2^{c_last} in TMEM (row d = r)
                {
                    const float f = tc::ex2(c_last);
                    tc::fence_after_sync();
#pragma unroll
                    for (int c = 0; c < kD; c += 32) {
                        float v[32];
                        tc::tmem_ld32(tS + lane_off + c, v);
                        tc::wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] *= f;
                        tc::tmem_st32(tS + lane_off + c, v);
                    }
                    tc::wait_st();
                }
                fence_proxy_async_smem();
                tc::fence_before_sync();
                mbar_arrive(&bars[kSScaled]);
                // ---- after the update: split S for the next chunk (and, at the
                // end, write the final state)
                if (!waitw(&bars[kSUpdated], ph)) { ok = false; break; }
                tc::fence_after_sync();
                float *sfin = (j == NC - 1 && p.state) ? p.state + ((int64_t)b * p.H + h) * kD * kD + (int64_t)r * kD
                                                      : nullptr;
#pragma unroll
                for (int c = 0; c < kD; c += 32) {
                    float v[32];
                    tc::tmem_ld32(tS + lane_off + c, v);
                    tc::wait_ld();
                    if (sfin) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4 *>(sfin + c + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                    }
                    if (j + 1 < NC) {
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            uint4 hi, lo;
                            uint32_t *hp = &hi.x, *lp = &lo.x;
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float x0 = v[e + 2 * q], x1 = v[e + 2 * q + 1];
                                hp[q] = tc::pack_bf16x2(x0, x1);
                                lp[q] = tc::pack_bf16x2(x0 - __uint_as_float(hp[q] << 16),
                                                        x1 - __uint_as_float(hp[q] & 0xffff0000u));
                            }
                            *reinterpret_cast<uint4 *>(sb + kShi + sw_off(r, c + e)) = hi;
                            *reinterpret_cast<uint4 *>(sb + kSlo + sw_off(r, c + e)) = lo;
                        }
                    }
                }
                if (j + 1 < NC) {
                    fence_proxy_async_smem();
                    tc::fence_before_sync();
                    mbar_arrive(&bars[kSplit]);
                }
            }
        }
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
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.B, a.T, a.H) || !make_map(&mk, a.k, a.B, a.T, a.H) || !make_map(&mv, a.v, a.B, a.T, a.H))
        return cudaErrorNotSupported;
    GretTcParams p;
    p.g = a.g;
    p.state = a.state;
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.B = a.B; p.H = a.H; p.T = a.T;
    p.lg_scale = kLog2e / a.tau;
    p.scale = a.scale;
    p.n_chunks = (int)((a.T + kC - 1) / kC);
    cudaError_t e = cudaFuncSetAttribute(gret_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kAlloc);
    if (e != cudaSuccess) return e;
    note_launches(1);
    gret_tc_kernel<<<a.B * a.H, kThreads, kAlloc, st>>>(mq, mk, mv, p);
    return cudaGetLastError();
}

unsigned int read_and_clear_status_gret_tc() {
    unsigned int h = 0, z = 0;
    if (cudaMemcpyFromSymbol(&h, g_status_gret_tc, sizeof(h)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_status_gret_tc, &z, sizeof(z));
    return h;
}

}  // namespace yoco
