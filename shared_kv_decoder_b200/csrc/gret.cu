// Gated retention, the alternative self-decoder ("You Only Cache Once",
// paperlayer summary, section 3 "Design Choices of Self-Decoder", bullets
// "Gated Retention", and Appendix B "Chunk-wise Representation of Gated
// Retention"; podcast transcript cue 16: a data-dependent head-wise decay
// gate, sigmoid of the input raised to one over a temperature; a d x d state
// per head for decoding; chunkwise computation for prefill -- parallel inside
// a chunk, recurrent across chunks).  Per head:
//
//   gamma_t = sigmoid(g_t)^(1/tau)
//   S_t     = gamma_t S_{t-1} + scale * k_t^T v_t       (S: D x D, fp32)
//   o_t     = q_t S_t
//
// gret_prefill_kernel (bf16, head dim 64; head dim 128 runs on the tensor-core
// kernel in gret_tc.cu): one CTA of eight warps per (batch, head) walks the
// sequence in chunks of 64 tokens.  With c_r the running sum of log gamma
// over the chunk's rows 0..r:
//   o_r   = sum_{u<=r} e^{c_r - c_u} scale (q_r . k_u) v_u      (inner part)
//         + e^{c_r} q_r S_prev                                   (cross part)
//   S_new = e^{c_last} S_prev + sum_u e^{c_last - c_u} scale k_u^T v_u
// Every exponent is <= 0, so nothing overflows however strong the decay.  The
// products are warp-wide mma.sync tiles (bf16 in, fp32 accumulate): Q K^T
// with the decay mask applied to the fp32 accumulators, P V with P taken
// straight from those accumulators, Q S_prev against S_prev split into a
// bf16 high and low part (about 16 mantissa bits, so the state keeps its fp32
// accuracy through the cross term), and the state update K_w^T V into the
// fp32 state, which each warp keeps in registers for its 16 rows.  The next
// chunk's Q, K and V stream in with cp.async while the current one computes.
//
// gret_decode_kernel: one step of the recurrence, one CTA of 256 threads per
// (batch, head); a thread owns four adjacent state columns over a group of
// rows (16-byte row reads and writes of S, up to eight rows in flight at a
// time), and the row groups' partial outputs add up in shared memory.  With
// one column per thread and one row at a time (128 threads), too few bytes
// were in flight: 22.5 us against 18.5 us for a batch-16 step of 32 heads.
#include "common.cuh"
#include "launch.h"

#include <algorithm>
#include <type_traits>

namespace yoco {

namespace {

constexpr int kChunk = 64;
constexpr int kGretWarps = 8;
constexpr int kGretThreads = 32 * kGretWarps;
constexpr int kGretDecodeThreads = 256;   // 128 and 512 threads, batches of 16: no faster or slower
constexpr int kGretDecodeBatch = 8;

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
// c += A * B, one m16n8k16 tile (bf16 in, fp32 accumulate)
YOCO_DEV void mma16816(float *c, const uint32_t *a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
YOCO_DEV uint32_t bf2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}
YOCO_DEV void cp_async16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
YOCO_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
YOCO_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// log gamma = log(sigmoid(g)) / tau, stable for large |g|
YOCO_DEV float log_decay(float g, float inv_tau) {
    return (fminf(g, 0.f) - log1pf(expf(-fabsf(g)))) * inv_tau;
}

template <int D>
struct GretSmem {
    static constexpr int LD = D + 8;                      // padded row (elements): conflict-free ldmatrix
    static constexpr uint32_t TILE = kChunk * LD * 2;     // one [64, D] bf16 tile
    static constexpr uint32_t SMAT = D * LD * 2;          // one [D, D] bf16 matrix
    static constexpr uint32_t QKV = 0;                    // 2 buffers x (Q, K, V)
    static constexpr uint32_t KW = QKV + 6 * TILE;        // decayed, scaled K of the chunk
    static constexpr uint32_t SHI = KW + TILE;            // state, bf16 high part
    static constexpr uint32_t SLO = SHI + SMAT;           // state, bf16 low part
    static constexpr uint32_t CUM = SLO + SMAT;           // running log-decay sums [64]
    static constexpr uint32_t BYTES = CUM + kChunk * 4;
};

struct GretParams {
    const __nv_bfloat16 *q, *k, *v;
    const float *g;
    float *state;          // [B, H, D, D] or null
    __nv_bfloat16 *o;
    int32_t B, H;
    int64_t T;
    float inv_tau, scale;
};

}  // namespace

template <int D>
__global__ void __launch_bounds__(kGretThreads, 1) gret_prefill_kernel(const GretParams p) {
    using L = GretSmem<D>;
    constexpr int LD = L::LD;
    constexpr int MT = D / 16;                 // 16-row strips of the state
    constexpr int WPM = kGretWarps / MT;       // warps per state strip
    constexpr int SNT = (D / 8) / WPM;         // state n-tiles per warp
    constexpr int ONT = D / 16;                // output n-tiles per warp (half of D)
    constexpr int CPR = D / 8;                 // 16-byte chunks per row
    extern __shared__ __align__(128) unsigned char smem[];
    const uint32_t s0 = smem_u32(smem);
    float *cum = reinterpret_cast<float *>(smem + L::CUM);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const int b = blockIdx.x / p.H, h = blockIdx.x % p.H;
    const int64_t T = p.T;
    const int64_t row_stride = (int64_t)p.H * D;  // elements between consecutive tokens
    const __nv_bfloat16 *qb = p.q + ((int64_t)b * T * p.H + h) * D;
    const __nv_bfloat16 *kb = p.k + ((int64_t)b * T * p.H + h) * D;
    const __nv_bfloat16 *vb = p.v + ((int64_t)b * T * p.H + h) * D;
    const int n_chunks = (int)((T + kChunk - 1) / kChunk);

    auto load_chunk = [&](int j, int buf) {
        const int64_t t0 = (int64_t)j * kChunk;
        for (int c = threadIdx.x; c < 3 * kChunk * CPR; c += kGretThreads) {
            const int tsr = c / (kChunk * CPR), rem = c % (kChunk * CPR);
            const int r = rem / CPR, ch = rem % CPR;
            const bool valid = t0 + r < T;
            const int64_t tok = valid ? t0 + r : 0;
            const __nv_bfloat16 *src = (tsr == 0 ? qb : tsr == 1 ? kb : vb) + tok * row_stride + ch * 8;
            cp_async16(s0 + L::QKV + (uint32_t)(buf * 3 + tsr) * L::TILE + (uint32_t)(r * LD + ch * 8) * 2, src,
                       valid);
        }
        cp_async_commit();
    };

    // the state strip this warp owns: rows d0..d0+15, columns [e0, e0 + 8*SNT)
    const int d0 = (warp % MT) * 16, e0 = (warp / MT) * SNT * 8;
    float st[SNT][4];
    const float *sg = p.state ? p.state + ((int64_t)b * p.H + h) * D * D : nullptr;
#pragma unroll
    for (int n = 0; n < SNT; ++n) {
        const int e = e0 + 8 * n + 2 * tq;
        st[n][0] = sg ? sg[(d0 + gq) * D + e] : 0.f;
        st[n][1] = sg ? sg[(d0 + gq) * D + e + 1] : 0.f;
        st[n][2] = sg ? sg[(d0 + gq + 8) * D + e] : 0.f;
        st[n][3] = sg ? sg[(d0 + gq + 8) * D + e + 1] : 0.f;
    }
    // bf16 high / low parts of the state for the cross term
    auto store_state_split = [&]() {
        __nv_bfloat16 *shi = reinterpret_cast<__nv_bfloat16 *>(smem + L::SHI);
        __nv_bfloat16 *slo = reinterpret_cast<__nv_bfloat16 *>(smem + L::SLO);
#pragma unroll
        for (int n = 0; n < SNT; ++n) {
            const int e = e0 + 8 * n + 2 * tq;
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {
                const int d = d0 + gq + 8 * hr;
                const float x0 = st[n][2 * hr], x1 = st[n][2 * hr + 1];
                const uint32_t hi = bf2(x0, x1);
                const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xffff0000u);
                *reinterpret_cast<uint32_t *>(shi + d * LD + e) = hi;
                *reinterpret_cast<uint32_t *>(slo + d * LD + e) = bf2(x0 - h0, x1 - h1);
            }
        }
    };
    store_state_split();
    load_chunk(0, 0);

    // output-phase role: rows 16*mt .. of the chunk, output columns [oh * D/2, (oh+1) * D/2)
    const int mt = warp & 3, oh = warp >> 2;
    const int mat = lane >> 3, rr = lane & 7;

    for (int j = 0; j < n_chunks; ++j) {
        const int buf = j & 1;
        const int64_t t0 = (int64_t)j * kChunk;
        const int len = (int)std::min<int64_t>(kChunk, T - t0);
        cp_async_wait_all();
        __syncthreads();  // chunk j landed; every warp is done with chunk j-1
        if (j + 1 < n_chunks) load_chunk(j + 1, buf ^ 1);
        // running log-decay sums over the chunk (padded rows decay by 1)
        if (warp == 0) {
            float x0 = lane < len ? log_decay(p.g[((int64_t)b * T + t0 + lane) * p.H + h], p.inv_tau) : 0.f;
            float x1 = lane + 32 < len ? log_decay(p.g[((int64_t)b * T + t0 + lane + 32) * p.H + h], p.inv_tau) : 0.f;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float y0 = __shfl_up_sync(0xffffffffu, x0, o), y1 = __shfl_up_sync(0xffffffffu, x1, o);
                if (lane >= o) { x0 += y0; x1 += y1; }
            }
            x1 += __shfl_sync(0xffffffffu, x0, 31);
            cum[lane] = x0;
            cum[lane + 32] = x1;
        }
        __syncthreads();
        const float c_last = cum[kChunk - 1];
        const uint32_t qs = s0 + L::QKV + (uint32_t)(buf * 3 + 0) * L::TILE;
        const uint32_t ks = s0 + L::QKV + (uint32_t)(buf * 3 + 1) * L::TILE;
        const uint32_t vs = s0 + L::QKV + (uint32_t)(buf * 3 + 2) * L::TILE;
        // K_w = K * scale * e^{c_last - c_u}, for the state update
        {
            const __nv_bfloat16 *kt = reinterpret_cast<const __nv_bfloat16 *>(smem + (ks - s0));
            __nv_bfloat16 *kw = reinterpret_cast<__nv_bfloat16 *>(smem + L::KW);
            for (int c = threadIdx.x; c < kChunk * (D / 2); c += kGretThreads) {
                const int r = c / (D / 2), d = (c % (D / 2)) * 2;
                const float w = p.scale * __expf(c_last - cum[r]);
                const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162 *>(kt + r * LD + d);
                *reinterpret_cast<uint32_t *>(kw + r * LD + d) =
                    bf2(__bfloat162float(x.x) * w, __bfloat162float(x.y) * w);
            }
        }

        // ---------------------------------------------------------- output
        {
            // A = Q K^T for rows 16mt..16mt+15 and all 64 keys
            float sc[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
            const uint32_t qrow = qs + (uint32_t)((16 * mt + (lane & 15)) * LD + (lane >> 4) * 8) * 2;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t a[4];
                ldsm_x4(qrow + kk * 32, a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int n = 0; n < 8; n += 2) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(ks + (uint32_t)((8 * n + 8 * (mat >> 1) + rr) * LD + 16 * kk + 8 * (mat & 1)) * 2,
                            b0, b1, b2, b3);
                    mma16816(sc[n], a, b0, b1);
                    mma16816(sc[n + 1], a, b2, b3);
                }
            }
            // decay mask: weight scale * e^{c_r - c_u} for u <= r, else 0
            const int r0 = 16 * mt + gq, r1 = r0 + 8;
            const float cr0 = cum[r0], cr1 = cum[r1];
#pragma unroll
            for (int n = 0; n < 8; ++n) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int u = 8 * n + 2 * tq + e;
                    const float cu = cum[u];
                    sc[n][e] = u <= r0 ? sc[n][e] * p.scale * __expf(cr0 - cu) : 0.f;
                    sc[n][2 + e] = u <= r1 ? sc[n][2 + e] * p.scale * __expf(cr1 - cu) : 0.f;
                }
            }
            // O = P V for this warp's output columns
            float oc[ONT][4];
#pragma unroll
            for (int n = 0; n < ONT; ++n) oc[n][0] = oc[n][1] = oc[n][2] = oc[n][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk) {
                uint32_t a[4];
                a[0] = bf2(sc[2 * kk][0], sc[2 * kk][1]);
                a[1] = bf2(sc[2 * kk][2], sc[2 * kk][3]);
                a[2] = bf2(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
                a[3] = bf2(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
#pragma unroll
                for (int n = 0; n < ONT; n += 2) {
                    uint32_t b0, b1, b2, b3;
                    const int col = oh * (D / 2) + 8 * n;
                    ldsm_x4_t(vs + (uint32_t)((16 * kk + 8 * (mat & 1) + rr) * LD + col + 8 * (mat >> 1)) * 2,
                              b0, b1, b2, b3);
                    mma16816(oc[n], a, b0, b1);
                    mma16816(oc[n + 1], a, b2, b3);
                }
            }
            // cross part: e^{c_r} q_r S_prev, S_prev = S_hi + S_lo
            float xc[ONT][4];
#pragma unroll
            for (int n = 0; n < ONT; ++n) xc[n][0] = xc[n][1] = xc[n][2] = xc[n][3] = 0.f;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const uint32_t sm = s0 + (part == 0 ? L::SHI : L::SLO);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    uint32_t a[4];
                    ldsm_x4(qrow + kk * 32, a[0], a[1], a[2], a[3]);
#pragma unroll
                    for (int n = 0; n < ONT; n += 2) {
                        uint32_t b0, b1, b2, b3;
                        const int col = oh * (D / 2) + 8 * n;
                        ldsm_x4_t(sm + (uint32_t)((16 * kk + 8 * (mat & 1) + rr) * LD + col + 8 * (mat >> 1)) * 2,
                                  b0, b1, b2, b3);
                        mma16816(xc[n], a, b0, b1);
                        mma16816(xc[n + 1], a, b2, b3);
                    }
                }
            }
            const float f0 = __expf(cr0), f1 = __expf(cr1);
#pragma unroll
            for (int n = 0; n < ONT; ++n) {
                const int col = oh * (D / 2) + 8 * n + 2 * tq;
                if (r0 < len)
                    *reinterpret_cast<uint32_t *>(p.o + (((int64_t)b * T + t0 + r0) * p.H + h) * D + col) =
                        bf2(oc[n][0] + f0 * xc[n][0], oc[n][1] + f0 * xc[n][1]);
                if (r1 < len)
                    *reinterpret_cast<uint32_t *>(p.o + (((int64_t)b * T + t0 + r1) * p.H + h) * D + col) =
                        bf2(oc[n][2] + f1 * xc[n][2], oc[n][3] + f1 * xc[n][3]);
            }
        }
        __syncthreads();  // K_w complete; every warp done reading S_hi / S_lo

        // ---------------------------------------------------- state update
        {
            const float fe = __expf(c_last);
#pragma unroll
            for (int n = 0; n < SNT; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) st[n][e] *= fe;
            const uint32_t kw = s0 + L::KW;
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk) {
                // A = K_w^T: rows d0..d0+15, tokens 16kk..16kk+15 (transposed loads)
                uint32_t a[4];
                ldsm_x4_t(kw + (uint32_t)((16 * kk + 8 * (mat >> 1) + rr) * LD + d0 + 8 * (mat & 1)) * 2, a[0],
                          a[1], a[2], a[3]);
#pragma unroll
                for (int n = 0; n < SNT; n += 2) {
                    uint32_t b0, b1, b2, b3;
                    const int col = e0 + 8 * n;
                    ldsm_x4_t(vs + (uint32_t)((16 * kk + 8 * (mat & 1) + rr) * LD + col + 8 * (mat >> 1)) * 2,
                              b0, b1, b2, b3);
                    mma16816(st[n], a, b0, b1);
                    mma16816(st[n + 1], a, b2, b3);
                }
            }
            store_state_split();
        }
    }
    if (p.state) {
        float *sgo = p.state + ((int64_t)b * p.H + h) * D * D;
#pragma unroll
        for (int n = 0; n < SNT; ++n) {
            const int e = e0 + 8 * n + 2 * tq;
            *reinterpret_cast<float2 *>(sgo + (d0 + gq) * D + e) = make_float2(st[n][0], st[n][1]);
            *reinterpret_cast<float2 *>(sgo + (d0 + gq + 8) * D + e) = make_float2(st[n][2], st[n][3]);
        }
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(kGretDecodeThreads) gret_decode_kernel(const T *q, const T *k, const T *v,
                                                                         const float *g, int32_t H, float inv_tau,
                                                                         float scale, float *state, T *o) {
    constexpr int CQ = D / 4;                       // column quads
    constexpr int RG = kGretDecodeThreads / CQ;     // row groups
    constexpr int RPG = D / RG;                     // rows per group
    constexpr int NB = RPG < kGretDecodeBatch ? RPG : kGretDecodeBatch;   // rows in flight
    static_assert(RPG % NB == 0, "rows per group in whole batches");
    __shared__ float sq[D], sk[D];
    __shared__ float4 part[RG][CQ];
    const int tid = threadIdx.x, cq = tid % CQ, rg = tid / CQ;
    const int64_t bh = blockIdx.x;
    for (int i = tid; i < D; i += kGretDecodeThreads) {
        sq[i] = to_f32(q[bh * D + i]);
        sk[i] = to_f32(k[bh * D + i]) * scale;
    }
    const float v0 = to_f32(v[bh * D + 4 * cq]), v1 = to_f32(v[bh * D + 4 * cq + 1]);
    const float v2 = to_f32(v[bh * D + 4 * cq + 2]), v3 = to_f32(v[bh * D + 4 * cq + 3]);
    const float gam = __expf(log_decay(g[bh], inv_tau));
    __syncthreads();
    float4 *S = reinterpret_cast<float4 *>(state + bh * D * D);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int d0 = rg * RPG; d0 < (rg + 1) * RPG; d0 += NB) {
        // a batch of rows' column quads in flight before any is used
        float4 sv[NB];
#pragma unroll
        for (int u = 0; u < NB; ++u) sv[u] = S[(d0 + u) * CQ + cq];
#pragma unroll
        for (int u = 0; u < NB; ++u) {
            const int d = d0 + u;
            float4 s4;
            s4.x = fmaf(gam, sv[u].x, sk[d] * v0);
            s4.y = fmaf(gam, sv[u].y, sk[d] * v1);
            s4.z = fmaf(gam, sv[u].z, sk[d] * v2);
            s4.w = fmaf(gam, sv[u].w, sk[d] * v3);
            S[d * CQ + cq] = s4;
            acc.x = fmaf(sq[d], s4.x, acc.x);
            acc.y = fmaf(sq[d], s4.y, acc.y);
            acc.z = fmaf(sq[d], s4.z, acc.z);
            acc.w = fmaf(sq[d], s4.w, acc.w);
        }
    }
    part[rg][cq] = acc;
    __syncthreads();
    if (rg == 0) {
        float4 t = part[0][cq];
#pragma unroll
        for (int r = 1; r < RG; ++r) {
            t.x += part[r][cq].x;
            t.y += part[r][cq].y;
            t.z += part[r][cq].z;
            t.w += part[r][cq].w;
        }
        o[bh * D + 4 * cq] = from_f32<T>(t.x);
        o[bh * D + 4 * cq + 1] = from_f32<T>(t.y);
        o[bh * D + 4 * cq + 2] = from_f32<T>(t.z);
        o[bh * D + 4 * cq + 3] = from_f32<T>(t.w);
    }
}

// ------------------------------------------------------------------- host
template <int D>
static cudaError_t launch_gret_prefill_d(const GretArgs &a, cudaStream_t st) {
    GretParams p;
    p.q = static_cast<const __nv_bfloat16 *>(a.q);
    p.k = static_cast<const __nv_bfloat16 *>(a.k);
    p.v = static_cast<const __nv_bfloat16 *>(a.v);
    p.g = a.g;
    p.state = a.state;
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.B = a.B; p.H = a.H; p.T = a.T;
    p.inv_tau = 1.f / a.tau;
    p.scale = a.scale;
    auto kern = gret_prefill_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)GretSmem<D>::BYTES);
    if (e != cudaSuccess) return e;
    note_launches(1);
    kern<<<a.B * a.H, kGretThreads, GretSmem<D>::BYTES, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_gret_prefill(const GretArgs &a, cudaStream_t st) {
    if (a.dtype != kBF16) return cudaErrorNotSupported;
    if (a.B == 0 || a.T == 0 || a.H == 0) return cudaSuccess;
    // D = 128: the tcgen05 kernel (gret_tc.cu); otherwise the mma.sync kernel here
    const cudaError_t e = launch_gret_prefill_tc(a, st);
    if (e != cudaErrorNotSupported) return e;
    cudaGetLastError();
    if ((int64_t)a.B * a.H > INT32_MAX) return cudaErrorNotSupported;
    if (a.D == 128) return launch_gret_prefill_d<128>(a, st);
    if (a.D == 64) return launch_gret_prefill_d<64>(a, st);
    return cudaErrorNotSupported;
}

template <typename T>
static cudaError_t launch_gret_decode_t(const GretArgs &a, cudaStream_t st) {
    const int grid = a.B * a.H;
    const float inv_tau = 1.f / a.tau;
    note_launches(1);
    if (a.D == 128)
        gret_decode_kernel<T, 128><<<grid, kGretDecodeThreads, 0, st>>>(
            static_cast<const T *>(a.q), static_cast<const T *>(a.k), static_cast<const T *>(a.v), a.g, a.H, inv_tau,
            a.scale, a.state, static_cast<T *>(a.o));
    else
        gret_decode_kernel<T, 64><<<grid, kGretDecodeThreads, 0, st>>>(
            static_cast<const T *>(a.q), static_cast<const T *>(a.k), static_cast<const T *>(a.v), a.g, a.H, inv_tau,
            a.scale, a.state, static_cast<T *>(a.o));
    return cudaGetLastError();
}

cudaError_t launch_gret_decode(const GretArgs &a, cudaStream_t st) {
    if (a.B == 0 || a.H == 0) return cudaSuccess;
    if ((int64_t)a.B * a.H > INT32_MAX || (a.D != 64 && a.D != 128)) return cudaErrorNotSupported;
    return a.dtype == kBF16 ? launch_gret_decode_t<__nv_bfloat16>(a, st) : launch_gret_decode_t<float>(a, st);
}

}  // namespace yoco
