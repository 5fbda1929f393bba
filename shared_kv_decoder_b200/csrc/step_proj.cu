// The K/V projection of a decode step (a few new tokens) with the weight rows
// streamed through registers:
//
//   out[r, c] = N(x)[r, :] . W[c, :] + w * base[r, c]      (r < n <= 4)
//
// -- the K/V producer of the self-decoder with the YOCO++ weighted residual
// (podcast transcript "YOCO: Caching Once ...", cue 12; YOCO++ Abstract), the
// same result as the other projection kernels of linear.cu.
//
// A CTA takes 16 output columns (one m16 tile of weight rows, 128 KB at
// d_in = 4096) and holds no weights in shared memory: its eight warps each
// load their d_in / 8 columns of the 16 rows as 16-byte register loads,
// twelve 32-column blocks in flight at a time, and multiply them with the n
// token rows on the tensor cores (the MMA's N columns: tokens 0..n-1, and a
// column of ones at 7 whose products are the rows' weight sums, for the folded
// LayerNorm).  The token rows are bulk-copied into shared memory; the warps
// also add up their columns' share of each row's LayerNorm sums.  A CTA takes
// ~37 KB of shared memory and 140 registers a thread (256 threads, one CTA an
// SM).  Measured in CUDA graphs of 4096 layer-steps (4 x 4096 -> 2048, then
// the window decode over a 4 x 1024 ring): 15.2 us a layer-step, against
// 16.2-16.6 with 126 registers (two CTAs an SM) and 16.6 for linear.cu's
// few-row projection followed by the decode.
//
// Programmatic launch: the weight rows and the token rows are prefetched into
// L2 before the wait (a prefetch changes no data).

#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace yoco {

static __device__ unsigned int g_status_step_proj;

namespace {

typedef __nv_bfloat16 bf16;

constexpr int kPWarps = 8;
constexpr int kPThreads = 32 * kPWarps;
constexpr int kPRows = 16;      // output columns (weight rows) per CTA
constexpr int kPMaxTok = 4;     // token rows
constexpr int kPBatch = 12;     // 32-column k-blocks per batch of weight loads (24 loads a thread)

YOCO_DEV uint4 ldg_stream(const uint4 *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}
YOCO_DEV void mma16816(float *c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// shared memory: x [n][d_in + 32] bf16 (the 64-byte pad puts the two rows of
// one 16-byte load phase in distinct banks), the warps' partial tiles
// [8][16][8] and LayerNorm sums [8][4][2] (floats), the mbarrier
__host__ __device__ inline size_t proj_x_bytes(int n, int d_in) { return ((size_t)n * (d_in + 32) * 2 + 15) / 16 * 16; }
inline size_t proj_smem_bytes(int n, int d_in) {
    return proj_x_bytes(n, d_in) + (size_t)kPWarps * kPRows * 8 * 4 + (size_t)kPWarps * kPMaxTok * 2 * 4 + 16;
}

}  // namespace

__global__ void __launch_bounds__(kPThreads, 1) linear_few_reg_kernel(const LinearArgs a) {
    extern __shared__ __align__(16) unsigned char sm[];
    __shared__ float mu[kPMaxTok], rs[kPMaxTok];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, t = lane & 3;
    const int n = (int)a.n, K = a.d_in, ldx = K + 32;
    bf16 *xs = reinterpret_cast<bf16 *>(sm);
    float *part = reinterpret_cast<float *>(sm + proj_x_bytes(n, K));   // [8 warps][16 rows][8 columns]
    float *lsum = part + kPWarps * kPRows * 8;                            // [8 warps][4 tokens][2]
    uint64_t *bar = reinterpret_cast<uint64_t *>(lsum + kPWarps * kPMaxTok * 2);
    const bf16 *w = static_cast<const bf16 *>(a.w);
    const bf16 *x = static_cast<const bf16 *>(a.x);
    const int r0 = blockIdx.x * kPRows;

    if (threadIdx.x < kPRows)   // this CTA's weight rows into L2 while the previous kernel finishes
        bulk_prefetch_l2(w + (int64_t)(r0 + threadIdx.x) * K, (uint32_t)K * 2u);
    if (threadIdx.x == kPRows && blockIdx.x < 8)   // the token rows (the first CTAs; the rest hit L2)
        bulk_prefetch_l2(x, (uint32_t)(n * K * 2));
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar, (uint32_t)(n * K * 2));
        for (int r = 0; r < n; ++r) bulk_g2s(xs + (size_t)r * ldx, x + (int64_t)r * K, (uint32_t)K * 2u, bar);
    }
    // A k-block is 32 columns; a thread's 16-byte load covers columns
    // 8t..8t+7 of it, which feed two MMAs (columns 8t+0..3, then 8t+4..7, in
    // the slots of k = 2t, 2t+1, 2t+8, 2t+9) -- the same order for the weight
    // rows (A) and the token rows (B), so the sum is unchanged.
    const int kbw = K / 32 / kPWarps;   // k-blocks of this warp
    const int kb0 = warp * kbw;
    const uint4 *wa = reinterpret_cast<const uint4 *>(w + (int64_t)(r0 + gq) * K) + t;
    const uint4 *wb = reinterpret_cast<const uint4 *>(w + (int64_t)(r0 + gq + 8) * K) + t;
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    float s1 = 0.f, s2 = 0.f;   // this lane's share of token gq's LayerNorm sums (shifted by x[gq][0])
    bool ok = true;
    const uint32_t kOnes = 0x3F803F80u;   // two bf16 1.0
    for (int k0 = 0; k0 < kbw && ok; k0 += kPBatch) {
        const int nk = min(kPBatch, kbw - k0);
        uint4 ra[kPBatch], rb[kPBatch];
#pragma unroll
        for (int u = 0; u < kPBatch; ++u)
            if (u < nk) {
                ra[u] = ldg_stream(wa + (kb0 + k0 + u) * 4);
                rb[u] = ldg_stream(wb + (kb0 + k0 + u) * 4);
            }
        if (k0 == 0) ok = __all_sync(0xffffffffu, mbar_wait(bar, 0, &g_status_step_proj));
        if (!ok) break;
        const bf16 *xg = xs + (size_t)gq * ldx + 8 * t;
        const float x0 = gq < n ? __bfloat162float(xs[(size_t)gq * ldx]) : 0.f;
#pragma unroll
        for (int u = 0; u < kPBatch; ++u)
            if (u < nk) {
                uint4 xv;
                if (gq < n) {
                    xv = *reinterpret_cast<const uint4 *>(xg + (kb0 + k0 + u) * 32);
                    float f[8];
                    Chunk<bf16>::unpack(xv, f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float d = f[i] - x0;
                        s1 += d;
                        s2 = fmaf(d, d, s2);
                    }
                } else {
                    xv = gq == 7 ? make_uint4(kOnes, kOnes, kOnes, kOnes) : make_uint4(0u, 0u, 0u, 0u);
                }
                mma16816(c, ra[u].x, rb[u].x, ra[u].y, rb[u].y, xv.x, xv.y);
                mma16816(c, ra[u].z, rb[u].z, ra[u].w, rb[u].w, xv.z, xv.w);
            }
    }
    // the row's four lanes hold disjoint columns
    s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
    s2 += __shfl_xor_sync(0xffffffffu, s2, 1);
    s2 += __shfl_xor_sync(0xffffffffu, s2, 2);
    if (t == 0 && gq < n) {
        lsum[(warp * kPMaxTok + gq) * 2] = s1;
        lsum[(warp * kPMaxTok + gq) * 2 + 1] = s2;
    }
    float *pw = part + warp * kPRows * 8;
    pw[gq * 8 + 2 * t] = c[0];
    pw[gq * 8 + 2 * t + 1] = c[1];
    pw[(gq + 8) * 8 + 2 * t] = c[2];
    pw[(gq + 8) * 8 + 2 * t + 1] = c[3];
    ok = __syncthreads_and(ok);
    if (!ok) return;
    if ((int)threadIdx.x < n) {
        const int r = threadIdx.x;
        float mean = 0.f, rstd = 1.f;
        if (a.apply_ln) {
            float S1 = 0.f, S2 = 0.f;
            for (int ww = 0; ww < kPWarps; ++ww) {
                S1 += lsum[(ww * kPMaxTok + r) * 2];
                S2 += lsum[(ww * kPMaxTok + r) * 2 + 1];
            }
            const float m1 = S1 / (float)K;
            const float var = fmaxf(S2 / (float)K - m1 * m1, 0.f);
            mean = __bfloat162float(xs[(size_t)r * ldx]) + m1;
            rstd = rsqrtf(var + a.eps);
        }
        mu[r] = mean;
        rs[r] = rstd;
    }
    __syncthreads();
    // one thread per (token, column): the warps' partial sums, the fold, the blend
    const int i = threadIdx.x, r = i / kPRows, cc = i % kPRows;
    if (r >= n || r0 + cc >= a.d_out) return;
    float tot = 0.f, wsum = 0.f;
#pragma unroll
    for (int ww = 0; ww < kPWarps; ++ww) {
        tot += part[(ww * kPRows + cc) * 8 + r];
        wsum += part[(ww * kPRows + cc) * 8 + 7];
    }
    const int col = r0 + cc, w1 = a.d_out - a.split_col;
    const int64_t dr = a.dst_rows ? a.dst_rows[r] : r;
    float val = a.apply_ln ? rs[r] * (tot - mu[r] * wsum) : tot;
    if (col < a.split_col) {
        if (a.base0) val = fmaf(a.w0, __bfloat162float(static_cast<const bf16 *>(a.base0)[(int64_t)r * a.split_col + col]), val);
        static_cast<bf16 *>(a.out0)[dr * a.split_col + col] = __float2bfloat16_rn(val);
    } else {
        const int c1 = col - a.split_col;
        if (a.base1) val = fmaf(a.w1, __bfloat162float(static_cast<const bf16 *>(a.base1)[(int64_t)r * w1 + c1]), val);
        static_cast<bf16 *>(a.out1)[dr * w1 + c1] = __float2bfloat16_rn(val);
    }
}

cudaError_t launch_linear_few_reg(const LinearArgs &a, cudaStream_t st) {
    if (a.dtype != kBF16 || a.n < 1 || a.n > kPMaxTok || a.d_in % (32 * kPWarps) != 0 || a.d_out % kPRows != 0)
        return cudaErrorNotSupported;
    const size_t smem = proj_smem_bytes((int)a.n, a.d_in);
    if (smem > 100 * 1024) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(linear_few_reg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    note_launches(1);
    return launch_pdl(linear_few_reg_kernel, dim3(a.d_out / kPRows), dim3(kPThreads), smem, st, a);
}

unsigned int read_and_clear_status_step_proj() {
    unsigned int h = 0, z = 0;
    if (cudaMemcpyFromSymbol(&h, g_status_step_proj, sizeof(h)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_status_step_proj, &z, sizeof(z));
    return h;
}

}  // namespace yoco
