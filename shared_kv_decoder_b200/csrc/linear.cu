// Projection with an optional LayerNorm prologue and a weighted-residual
// epilogue, on CUDA cores:
//
//   out[r, c] = N(x)[r, :] . W[c, :] + w * base[r, c]
//
// This is the K/V producer of the self-decoder and of the global KV (podcast
// transcript "YOCO: Caching Once ...", cue 12: normalised once, projected by
// one pair of matrices) with the YOCO++ weighted residual to the bottom
// layer's KV fused into the epilogue (YOCO++ Abstract), so the blend costs no
// extra pass over HBM.  The same kernel serves the query / output
// projections of the small end-to-end stack.
//
// LayerNorm statistics (mean, biased variance) are computed per CTA row tile
// in fp32 before the main loop, and rows are normalised while they are
// staged into shared memory.  Output columns below split_col go to out0, the
// rest to out1 (K and V of one fused [K | V] weight); dst_rows, when given,
// scatters output rows (appending to the shared cache).
#include <algorithm>

#include "common.cuh"
#include "launch.h"

namespace yoco {

constexpr int kLinBM = 64, kLinBN = 64, kLinBK = 16;

template <typename T>
__global__ void __launch_bounds__(256) linear_simt_kernel(const LinearArgs a) {
    __shared__ float As[kLinBK][kLinBM + 4];
    __shared__ float Bs[kLinBK][kLinBN + 4];
    __shared__ float mu[kLinBM], rs[kLinBM];

    const T *x = static_cast<const T *>(a.x);
    const T *w = static_cast<const T *>(a.w);
    const int64_t r0 = (int64_t)blockIdx.y * kLinBM;
    const int c0 = blockIdx.x * kLinBN;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // LayerNorm statistics of this CTA's rows (two passes, fp32)
    for (int rr = warp; rr < kLinBM; rr += 8) {
        const int64_t r = r0 + rr;
        float mean = 0.f, rstd = 1.f;
        if (a.apply_ln && r < a.n) {
            const T *xr = x + r * a.d_in;
            float s = 0.f;
            for (int c = lane; c < a.d_in; c += 32) s += to_f32(xr[c]);
            mean = warp_sum(s) / (float)a.d_in;
            float q = 0.f;
            for (int c = lane; c < a.d_in; c += 32) {
                const float t = to_f32(xr[c]) - mean;
                q = fmaf(t, t, q);
            }
            rstd = rsqrtf(warp_sum(q) / (float)a.d_in + a.eps);
        }
        if (lane == 0) {
            mu[rr] = a.apply_ln ? mean : 0.f;
            rs[rr] = a.apply_ln ? rstd : 1.f;
        }
    }
    __syncthreads();

    const int ty = tid / 16, tx = tid % 16;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < a.d_in; k0 += kLinBK) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int idx = tid + 256 * e;       // 0 .. 1023
            const int rr = idx / kLinBK, kk = idx % kLinBK;
            const int64_t r = r0 + rr;
            const int kc = k0 + kk;
            As[kk][rr] = (r < a.n && kc < a.d_in) ? (to_f32(x[r * a.d_in + kc]) - mu[rr]) * rs[rr] : 0.f;
            const int c = c0 + rr;
            Bs[kk][rr] = (c < a.d_out && kc < a.d_in) ? to_f32(w[(int64_t)c * a.d_in + kc]) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kLinBK; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }

    const int w1 = a.d_out - a.split_col;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t r = r0 + ty * 4 + i;
        if (r >= a.n) continue;
        const int64_t dr = a.dst_rows ? a.dst_rows[r] : r;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int c = c0 + tx * 4 + j;
            if (c >= a.d_out) continue;
            float val = acc[i][j];
            if (c < a.split_col) {
                if (a.base0) val = fmaf(a.w0, to_f32(static_cast<const T *>(a.base0)[r * a.split_col + c]), val);
                static_cast<T *>(a.out0)[dr * a.split_col + c] = from_f32<T>(val);
            } else {
                const int cc = c - a.split_col;
                if (a.base1) val = fmaf(a.w1, to_f32(static_cast<const T *>(a.base1)[r * w1 + cc]), val);
                static_cast<T *>(a.out1)[dr * w1 + cc] = from_f32<T>(val);
            }
        }
    }
}

// A few rows (decode-step projections, n <= 16): the weight is read once,
// from HBM, and all of a CTA's share is in flight at once.  A CTA owns eight
// output columns (one per warp; 256 CTAs for a 2048-wide [K | V]).  One thread
// issues bulk copies of the CTA's eight weight rows and of the n x rows into
// shared memory, all completing on one mbarrier, so the bytes in flight cost
// no registers; before that, while the previous kernel finishes, every warp
// asks L2 for its weight row.  Each row's LayerNorm statistics come from one
// pass over its staged copy, shifted by the row's first value, and LayerNorm
// is folded out of the dot products,
//   N(x) . w = rstd (x . w - mean * sum(w)),
// so the inner loop is one packed f32x2 FMA per two weights and row.  NR
// bounds the row count at compile time (4, 8 or 16).
// Earlier versions, measured on a 4 x 4096 -> 2048 projection: four columns
// per warp and 64 CTAs, ~16 us (too few loads in flight); one column per warp
// with the weight in registers and the loop unrolled for 16 rows, 17 us
// (instruction-fetch bound); the same unrolled for 4 rows, 10 us (latency of
// each warp's own dependent loads, 0.4 eligible warps per cycle).
constexpr int kSmallRows = 16, kSmallWarps = 8;
constexpr size_t kSmallMaxSmem = 200 * 1024;

static __device__ unsigned int g_status_linear;

// 8 bf16 (one 16-byte chunk) as four packed fp32 pairs; 4 fp32 as two
template <typename T> YOCO_DEV void chunk_pairs(const uint4 &c, uint64_t *p);
template <> YOCO_DEV void chunk_pairs<__nv_bfloat16>(const uint4 &c, uint64_t *p) {
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint64_t r;
        asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(w[i] << 16), "r"(w[i] & 0xffff0000u));
        p[i] = r;
    }
}
template <> YOCO_DEV void chunk_pairs<float>(const uint4 &c, uint64_t *p) {
    uint64_t r0, r1;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r0) : "r"(c.x), "r"(c.y));
    asm("mov.b64 %0, {%1, %2};" : "=l"(r1) : "r"(c.z), "r"(c.w));
    p[0] = r0;
    p[1] = r1;
}
YOCO_DEV uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
YOCO_DEV uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
YOCO_DEV uint64_t pack2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
YOCO_DEV float hsum2(uint64_t a) {
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(a));
    return lo + hi;
}

// shared memory of the few-row projection: the CTA's weight rows, then the x
// rows (both [rows][d_in] of T), then the mbarrier
static inline size_t small_smem_bytes(int n, int d_in, int elem) {
    return ((size_t)(kSmallWarps + n) * d_in * elem + 15) / 16 * 16 + 16;
}

template <typename T, int NR>
__global__ void __launch_bounds__(32 * kSmallWarps, 2) linear_small_kernel(const LinearArgs a) {
    constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte chunk
    constexpr int NP = VEC / 2;          // packed pairs per chunk
    extern __shared__ __align__(16) uint4 sm4[];
    __shared__ float mu[NR], rs[NR];
    const T *w = static_cast<const T *>(a.w);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = (int)a.n;
    const int row_chunks = a.d_in / VEC;            // 16-byte chunks per row
    const int c0 = blockIdx.x * kSmallWarps;        // the CTA's first output column
    const int n_cols = min(kSmallWarps, a.d_out - c0);
    const int c = c0 + warp;                        // this warp's output column
    uint4 *ws4 = sm4;                               // [n_cols][row_chunks]
    uint4 *xs4 = sm4 + (size_t)kSmallWarps * row_chunks;   // [n][row_chunks]
    uint64_t *bar = reinterpret_cast<uint64_t *>(xs4 + (size_t)n * row_chunks);
    const uint32_t row_bytes = (uint32_t)row_chunks * 16u;

    // while the previous kernel finishes: ask L2 for this warp's weight row
    // (a prefetch only warms the cache; nothing is read before pdl_wait)
    pdl_trigger();
    if (warp < n_cols) {
        const uint4 *wrow = reinterpret_cast<const uint4 *>(w + (int64_t)c * a.d_in);
        for (int ch = lane * 8; ch < row_chunks; ch += 256) asm volatile("prefetch.global.L2 [%0];" ::"l"(wrow + ch));
    }
    if (threadIdx.x == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(bar, (uint32_t)(n_cols + n) * row_bytes);
        for (int j = 0; j < n_cols; ++j)
            bulk_g2s(ws4 + (size_t)j * row_chunks, w + (int64_t)(c0 + j) * a.d_in, row_bytes, bar);
        for (int r = 0; r < n; ++r)
            bulk_g2s(xs4 + (size_t)r * row_chunks, static_cast<const T *>(a.x) + (int64_t)r * a.d_in, row_bytes, bar);
    }
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar, 0, &g_status_linear));
    // the row statistics (warp r: row r)
    if (ok) {
        for (int r = warp; r < n; r += kSmallWarps) {
            float mean = 0.f, rstd = 1.f;
            if (a.apply_ln) {
                const float x0 = to_f32(reinterpret_cast<const T *>(xs4 + (size_t)r * row_chunks)[0]);
                const uint64_t sh = pack2(-x0, -x0);
                uint64_t s1 = 0, s2 = 0;
                for (int ch = lane; ch < row_chunks; ch += 32) {
                    uint64_t p[NP];
                    chunk_pairs<T>(xs4[(size_t)r * row_chunks + ch], p);
#pragma unroll
                    for (int i = 0; i < NP; ++i) {
                        const uint64_t d = add2(p[i], sh);
                        s1 = add2(s1, d);
                        s2 = fma2(d, d, s2);
                    }
                }
                const float m1 = warp_sum(hsum2(s1)) / (float)a.d_in;   // mean of x - x0
                const float var = fmaxf(warp_sum(hsum2(s2)) / (float)a.d_in - m1 * m1, 0.f);
                mean = x0 + m1;
                rstd = rsqrtf(var + a.eps);
            }
            if (lane == 0) {
                mu[r] = mean;
                rs[r] = rstd;
            }
        }
    }
    __syncthreads();
    if (!ok || warp >= n_cols) return;
    uint64_t acc[NR], wsum = 0;
#pragma unroll
    for (int r = 0; r < NR; ++r) acc[r] = 0;
    const uint4 *wr = ws4 + (size_t)warp * row_chunks;
#pragma unroll 4
    for (int ch = lane; ch < row_chunks; ch += 32) {
        uint64_t wp[NP];
        chunk_pairs<T>(wr[ch], wp);
#pragma unroll
        for (int i = 0; i < NP; ++i) wsum = add2(wsum, wp[i]);
#pragma unroll
        for (int r = 0; r < NR; ++r) {
            if (r < n) {
                uint64_t xp[NP];
                chunk_pairs<T>(xs4[(size_t)r * row_chunks + ch], xp);
#pragma unroll
                for (int i = 0; i < NP; ++i) acc[r] = fma2(xp[i], wp[i], acc[r]);
            }
        }
    }
    const float wsm = warp_sum(hsum2(wsum));
    const int w1 = a.d_out - a.split_col;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        if (r >= n) break;
        const float tot = warp_sum(hsum2(acc[r]));
        if (lane != r) continue;
        const int64_t dr = a.dst_rows ? a.dst_rows[r] : r;
        float val = a.apply_ln ? rs[r] * (tot - mu[r] * wsm) : tot;
        if (c < a.split_col) {
            if (a.base0) val = fmaf(a.w0, to_f32(static_cast<const T *>(a.base0)[(int64_t)r * a.split_col + c]), val);
            static_cast<T *>(a.out0)[dr * a.split_col + c] = from_f32<T>(val);
        } else {
            const int cc = c - a.split_col;
            if (a.base1) val = fmaf(a.w1, to_f32(static_cast<const T *>(a.base1)[(int64_t)r * w1 + cc]), val);
            static_cast<T *>(a.out1)[dr * w1 + cc] = from_f32<T>(val);
        }
    }
}

// The same projection on the tensor cores, for bf16, n <= 15 rows and d_in a
// multiple of 128: a CTA's eight output columns are one m16n8 MMA tile (A = the
// n x rows, padded with zeros and a row of ones at row 15, whose products are
// the columns' weight sums for the folded LayerNorm; B = the eight weight
// rows), the CTA's eight warps split K and add their partial tiles through
// shared memory.  The weight and x rows are bulk-copied in four K-quarters on
// four mbarriers, so a warp starts on its quarter as soon as it lands.  Rows
// are padded by 16 bytes in shared memory, so the eight rows one fragment load
// touches fall in distinct banks.
constexpr int kFewMaxRows = 15;   // row 15 carries the ones

YOCO_DEV void mma_bf16_16816(float *c, const uint32_t *a, const uint32_t *b) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

static inline size_t few_tc_smem_bytes(int n, int d_in) {
    return (size_t)(kSmallWarps + n) * (d_in + 8) * 2 + (size_t)kSmallWarps * 16 * 8 * 4 + 4 * 8;
}

__global__ void __launch_bounds__(32 * kSmallWarps, 2) linear_few_tc_kernel(const LinearArgs a) {
    typedef __nv_bfloat16 T;
    extern __shared__ __align__(16) unsigned char sm[];
    __shared__ float mu[kFewMaxRows], rs[kFewMaxRows];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t4 = lane & 3;
    const int n = (int)a.n, K = a.d_in, ldr = K + 8, Kq = K / 4, Kw = K / kSmallWarps;
    const int c0 = blockIdx.x * kSmallWarps;
    const int n_cols = min(kSmallWarps, a.d_out - c0);
    T *ws = reinterpret_cast<T *>(sm);                 // [8][ldr]
    T *xs = ws + (size_t)kSmallWarps * ldr;            // [n][ldr]
    float *part = reinterpret_cast<float *>(xs + (size_t)n * ldr);   // [8 warps][16][8]
    uint64_t *bars = reinterpret_cast<uint64_t *>(part + kSmallWarps * 16 * 8);
    const T *w = static_cast<const T *>(a.w);
    const T *x = static_cast<const T *>(a.x);

    pdl_trigger();
    if (warp < n_cols) {   // warm L2 with this warp's weight row while the previous kernel finishes
        const uint4 *wrow = reinterpret_cast<const uint4 *>(w + (int64_t)(c0 + warp) * K);
        for (int ch = lane * 8; ch < K / 8; ch += 256) asm volatile("prefetch.global.L2 [%0];" ::"l"(wrow + ch));
    }
    if (threadIdx.x == 0) {
        for (int q = 0; q < 4; ++q) mbar_init(&bars[q], 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    if (threadIdx.x == 0) {
        const uint32_t qb = (uint32_t)Kq * 2;
        for (int q = 0; q < 4; ++q) {
            mbar_arrive_expect_tx(&bars[q], (uint32_t)(n_cols + n) * qb);
            for (int j = 0; j < n_cols; ++j)
                bulk_g2s(ws + (size_t)j * ldr + q * Kq, w + (int64_t)(c0 + j) * K + q * Kq, qb, &bars[q]);
            for (int r = 0; r < n; ++r)
                bulk_g2s(xs + (size_t)r * ldr + q * Kq, x + (int64_t)r * K + q * Kq, qb, &bars[q]);
        }
    }
    // this warp's K range lies in quarter warp / 2
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[warp / 2], 0, &g_status_linear));
    float c[4] = {0.f, 0.f, 0.f, 0.f};
    if (ok) {
        const uint32_t kOnes = 0x3F803F80u;   // two bf16 1.0
        const T *xa = xs + (size_t)g * ldr, *xb = xs + (size_t)(g + 8) * ldr;
        const T *wb = ws + (size_t)g * ldr;
        for (int kk = warp * Kw; kk < (warp + 1) * Kw; kk += 16) {
            const int k0 = kk + 2 * t4;
            uint32_t af[4], bfr[2];
            af[0] = g < n ? *reinterpret_cast<const uint32_t *>(xa + k0) : 0u;
            af[2] = g < n ? *reinterpret_cast<const uint32_t *>(xa + k0 + 8) : 0u;
            af[1] = g + 8 < n ? *reinterpret_cast<const uint32_t *>(xb + k0) : (g == 7 ? kOnes : 0u);
            af[3] = g + 8 < n ? *reinterpret_cast<const uint32_t *>(xb + k0 + 8) : (g == 7 ? kOnes : 0u);
            bfr[0] = *reinterpret_cast<const uint32_t *>(wb + k0);
            bfr[1] = *reinterpret_cast<const uint32_t *>(wb + k0 + 8);
            mma_bf16_16816(c, af, bfr);
        }
    }
    float *pw = part + warp * 16 * 8;
    pw[g * 8 + 2 * t4] = c[0];
    pw[g * 8 + 2 * t4 + 1] = c[1];
    pw[(g + 8) * 8 + 2 * t4] = c[2];
    pw[(g + 8) * 8 + 2 * t4 + 1] = c[3];
    // every quarter has landed before the row statistics read whole rows
    for (int q = 0; q < 4 && ok; ++q) ok = __all_sync(0xffffffffu, mbar_wait(&bars[q], 0, &g_status_linear));
    if (ok && warp < n) {
        const int r = warp;
        float mean = 0.f, rstd = 1.f;
        if (a.apply_ln) {
            const T *xr = xs + (size_t)r * ldr;
            const float x0 = to_f32(xr[0]);
            const uint64_t sh = pack2(-x0, -x0);
            uint64_t s1 = 0, s2 = 0;
            for (int ch = lane; ch < K / 8; ch += 32) {
                uint64_t p[4];
                chunk_pairs<T>(*reinterpret_cast<const uint4 *>(xr + ch * 8), p);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint64_t d = add2(p[i], sh);
                    s1 = add2(s1, d);
                    s2 = fma2(d, d, s2);
                }
            }
            const float m1 = warp_sum(hsum2(s1)) / (float)K;
            const float var = fmaxf(warp_sum(hsum2(s2)) / (float)K - m1 * m1, 0.f);
            mean = x0 + m1;
            rstd = rsqrtf(var + a.eps);
        }
        if (lane == 0) {
            mu[r] = mean;
            rs[r] = rstd;
        }
    }
    __syncthreads();
    // one thread per (row, column): the warps' partial sums, the fold, the blend
    const int i = threadIdx.x, r = i / kSmallWarps, cc = i % kSmallWarps;
    if (!ok || r >= n || cc >= n_cols) return;
    float tot = 0.f, wsum = 0.f;
#pragma unroll
    for (int ww = 0; ww < kSmallWarps; ++ww) {
        tot += part[(ww * 16 + r) * 8 + cc];
        wsum += part[(ww * 16 + 15) * 8 + cc];
    }
    const int col = c0 + cc, w1 = a.d_out - a.split_col;
    const int64_t dr = a.dst_rows ? a.dst_rows[r] : r;
    float val = a.apply_ln ? rs[r] * (tot - mu[r] * wsum) : tot;
    if (col < a.split_col) {
        if (a.base0) val = fmaf(a.w0, to_f32(static_cast<const T *>(a.base0)[(int64_t)r * a.split_col + col]), val);
        static_cast<T *>(a.out0)[dr * a.split_col + col] = from_f32<T>(val);
    } else {
        const int c1 = col - a.split_col;
        if (a.base1) val = fmaf(a.w1, to_f32(static_cast<const T *>(a.base1)[(int64_t)r * w1 + c1]), val);
        static_cast<T *>(a.out1)[dr * w1 + c1] = from_f32<T>(val);
    }
}

template <typename T, int NR>
static cudaError_t launch_small(const LinearArgs &a, size_t smem, cudaStream_t st) {
    auto kern = linear_small_kernel<T, NR>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmallMaxSmem);
    if (e != cudaSuccess) return e;
    note_launches(1);
    const int grid = (a.d_out + kSmallWarps - 1) / kSmallWarps;
    return launch_pdl(kern, dim3(grid), dim3(32 * kSmallWarps), smem, st, a);
}

template <typename T>
static cudaError_t launch_small_t(const LinearArgs &a, size_t smem, cudaStream_t st) {
    if (a.n <= 4) return launch_small<T, 4>(a, smem, st);
    if (a.n <= 8) return launch_small<T, 8>(a, smem, st);
    return launch_small<T, 16>(a, smem, st);
}

cudaError_t launch_linear_simt(const LinearArgs &a, cudaStream_t st) {
    if (a.n == 0 || a.d_out == 0) return cudaSuccess;
    const int vec = a.dtype == kBF16 ? 8 : 4;
    if (a.dtype == kBF16 && a.n <= kFewMaxRows && a.d_in % 128 == 0) {
        const size_t fsm = few_tc_smem_bytes((int)a.n, a.d_in);
        if (fsm <= kSmallMaxSmem) {
            const cudaError_t e = cudaFuncSetAttribute(linear_few_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       (int)kSmallMaxSmem);
            if (e != cudaSuccess) return e;
            note_launches(1);
            const int grid = (a.d_out + kSmallWarps - 1) / kSmallWarps;
            return launch_pdl(linear_few_tc_kernel, dim3(grid), dim3(32 * kSmallWarps), fsm, st, a);
        }
    }
    const size_t smem = small_smem_bytes((int)std::min<int64_t>(a.n, kSmallRows), a.d_in, (int)dtype_bytes(a.dtype));
    if (a.n <= kSmallRows && a.d_in % vec == 0 && smem <= kSmallMaxSmem)
        return a.dtype == kBF16 ? launch_small_t<__nv_bfloat16>(a, smem, st) : launch_small_t<float>(a, smem, st);
    dim3 grid((unsigned)((a.d_out + kLinBN - 1) / kLinBN), (unsigned)((a.n + kLinBM - 1) / kLinBM));
    note_launches(1);
    if (a.dtype == kBF16)
        linear_simt_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
    else
        linear_simt_kernel<float><<<grid, 256, 0, st>>>(a);
    return cudaGetLastError();
}

unsigned int read_and_clear_status_linear() {
    unsigned int h = 0, z = 0;
    if (cudaMemcpyFromSymbol(&h, g_status_linear, sizeof(h)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_status_linear, &z, sizeof(z));
    return h;
}

}  // namespace yoco
