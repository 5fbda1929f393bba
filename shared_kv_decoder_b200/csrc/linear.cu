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
// from HBM, and all of it is in flight at once.  One output column per warp
// (256 CTAs for a 2048-wide [K | V]); each lane first asks L2 for its slice of
// the column's weight row, waits for the previous kernel (pdl_wait), then
// issues every 16-byte load of that slice before using any.  The CTA stages
// its x rows in shared memory and takes each row's LayerNorm statistics in
// one pass shifted by the row's first value (mean and variance of x - x_0).
// LayerNorm is folded out of the dot products:
//   N(x) . w = rstd (x . w - mean * sum(w)),
// so the inner loop is one packed f32x2 FMA per two weights and row.  NR
// bounds the row count at compile time (4, 8 or 16): a loop unrolled for 16
// rows when 4 are used ran ~4000 instructions per warp, bound by instruction
// fetch, for 17 us where the weight streams in a few.
constexpr int kSmallRows = 16, kSmallWarps = 8, kSmallChunks = 16;
constexpr size_t kSmallMaxSmem = 200 * 1024;

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

// x staged in shared memory: fp32 for up to four rows (converted once, so the
// inner loop reads ready pairs), else in its own type
template <typename T, int NR> struct SmallStage { using type = T; };
template <> struct SmallStage<__nv_bfloat16, 4> { using type = float; };

template <typename T, int NR>
__global__ void __launch_bounds__(32 * kSmallWarps, 2) linear_small_kernel(const LinearArgs a) {
    using XS = typename SmallStage<T, NR>::type;
    constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte chunk of T
    constexpr int NP = VEC / 2;          // packed pairs per chunk
    constexpr int XC = sizeof(XS) / sizeof(T);  // 16-byte staged chunks per chunk of T
    extern __shared__ uint4 xs4[];       // the n x rows, [n][d_in] of XS
    __shared__ float mu[NR], rs[NR];
    const T *w = static_cast<const T *>(a.w);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = (int)a.n;
    const int row_chunks = a.d_in / VEC;            // 16-byte chunks per row
    const int c = blockIdx.x * kSmallWarps + warp;  // this warp's output column
    const uint4 *wrow = reinterpret_cast<const uint4 *>(w + (int64_t)min(c, a.d_out - 1) * a.d_in);
    // while the previous kernel finishes: ask L2 for this warp's weight row
    // (a prefetch only warms the cache; nothing is read before pdl_wait)
    pdl_trigger();
    for (int ch = lane * 8; ch < row_chunks; ch += 256) asm volatile("prefetch.global.L2 [%0];" ::"l"(wrow + ch));
    pdl_wait();
    uint4 wr[kSmallChunks];
#pragma unroll
    for (int k = 0; k < kSmallChunks; ++k)
        if (lane + 32 * k < row_chunks) wr[k] = wrow[lane + 32 * k];
    // stage x (every thread, eight 16-byte loads in flight each), then the
    // statistics of each row
    const uint4 *x4 = static_cast<const uint4 *>(a.x);
    const int total = n * row_chunks;
    for (int i0 = 0; i0 < total; i0 += 8 * (int)blockDim.x) {
        uint4 t[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * (int)blockDim.x + (int)threadIdx.x;
            if (i < total) t[u] = x4[i];
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * (int)blockDim.x + (int)threadIdx.x;
            if (i < total) {
                if constexpr (XC == 1) {
                    xs4[i] = t[u];
                } else {   // bf16 -> fp32: one chunk of T becomes two staged chunks
                    uint64_t p[NP];
                    chunk_pairs<T>(t[u], p);
                    uint4 lo, hi;
                    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo.x), "=r"(lo.y) : "l"(p[0]));
                    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo.z), "=r"(lo.w) : "l"(p[1]));
                    asm("mov.b64 {%0, %1}, %2;" : "=r"(hi.x), "=r"(hi.y) : "l"(p[2]));
                    asm("mov.b64 {%0, %1}, %2;" : "=r"(hi.z), "=r"(hi.w) : "l"(p[3]));
                    xs4[2 * i] = lo;
                    xs4[2 * i + 1] = hi;
                }
            }
        }
    }
    __syncthreads();
    // the NP pairs of chunk ch of staged row r
    auto x_pairs = [&](int r, int ch, uint64_t *p) {
        if constexpr (XC == 1) {
            chunk_pairs<T>(xs4[(int64_t)r * row_chunks + ch], p);
        } else {
            const uint4 lo = xs4[2 * ((int64_t)r * row_chunks + ch)], hi = xs4[2 * ((int64_t)r * row_chunks + ch) + 1];
            asm("mov.b64 %0, {%1, %2};" : "=l"(p[0]) : "r"(lo.x), "r"(lo.y));
            asm("mov.b64 %0, {%1, %2};" : "=l"(p[1]) : "r"(lo.z), "r"(lo.w));
            asm("mov.b64 %0, {%1, %2};" : "=l"(p[2]) : "r"(hi.x), "r"(hi.y));
            asm("mov.b64 %0, {%1, %2};" : "=l"(p[3]) : "r"(hi.z), "r"(hi.w));
        }
    };
    for (int r = warp; r < n; r += kSmallWarps) {
        float mean = 0.f, rstd = 1.f;
        if (a.apply_ln) {
            const float x0 = to_f32(static_cast<const T *>(a.x)[(int64_t)r * a.d_in]);
            const uint64_t sh = pack2(-x0, -x0);
            uint64_t s1 = 0, s2 = 0;
            for (int ch = lane; ch < row_chunks; ch += 32) {
                uint64_t p[NP];
                x_pairs(r, ch, p);
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    const uint64_t d = add2(p[i], sh);
                    s1 = add2(s1, d);
                    s2 = fma2(d, d, s2);
                }
            }
            const float m1 = warp_sum(hsum2(s1)) / (float)a.d_in;          // mean of x - x0
            const float var = fmaxf(warp_sum(hsum2(s2)) / (float)a.d_in - m1 * m1, 0.f);
            mean = x0 + m1;
            rstd = rsqrtf(var + a.eps);
        }
        if (lane == 0) {
            mu[r] = mean;
            rs[r] = rstd;
        }
    }
    __syncthreads();
    if (c >= a.d_out) return;
    uint64_t acc[NR], wsum = 0;
#pragma unroll
    for (int r = 0; r < NR; ++r) acc[r] = 0;
    for (int k0 = 0; k0 * 32 < row_chunks; k0 += kSmallChunks) {
        if (k0 > 0) {  // rows longer than 16 chunks per lane: the next block of loads
#pragma unroll
            for (int k = 0; k < kSmallChunks; ++k)
                if (lane + 32 * (k0 + k) < row_chunks) wr[k] = wrow[lane + 32 * (k0 + k)];
        }
#pragma unroll
        for (int k = 0; k < kSmallChunks; ++k) {
            const int ch = lane + 32 * (k0 + k);
            if (ch >= row_chunks) break;
            uint64_t wp[NP];
            chunk_pairs<T>(wr[k], wp);
#pragma unroll
            for (int i = 0; i < NP; ++i) wsum = add2(wsum, wp[i]);
#pragma unroll
            for (int r = 0; r < NR; ++r) {
                if (r < n) {
                    uint64_t xp[NP];
                    x_pairs(r, ch, xp);
#pragma unroll
                    for (int i = 0; i < NP; ++i) acc[r] = fma2(xp[i], wp[i], acc[r]);
                }
            }
        }
    }
    const float ws = warp_sum(hsum2(wsum));
    const int w1 = a.d_out - a.split_col;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
        if (r >= n) break;
        const float tot = warp_sum(hsum2(acc[r]));
        if (lane != r) continue;
        const int64_t dr = a.dst_rows ? a.dst_rows[r] : r;
        float val = a.apply_ln ? rs[r] * (tot - mu[r] * ws) : tot;
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

template <typename T, int NR>
static cudaError_t launch_small(const LinearArgs &a, size_t xs_bytes, cudaStream_t st) {
    auto kern = linear_small_kernel<T, NR>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmallMaxSmem);
    if (e != cudaSuccess) return e;
    note_launches(1);
    const int grid = (a.d_out + kSmallWarps - 1) / kSmallWarps;
    return launch_pdl(kern, dim3(grid), dim3(32 * kSmallWarps), xs_bytes, st, a);
}

template <typename T>
static cudaError_t launch_small_t(const LinearArgs &a, size_t xs_bytes, cudaStream_t st) {
    // up to four rows are staged in fp32: twice the bytes of bf16
    if (a.n <= 4) return launch_small<T, 4>(a, xs_bytes * sizeof(typename SmallStage<T, 4>::type) / sizeof(T), st);
    if (a.n <= 8) return launch_small<T, 8>(a, xs_bytes, st);
    return launch_small<T, 16>(a, xs_bytes, st);
}

cudaError_t launch_linear_simt(const LinearArgs &a, cudaStream_t st) {
    if (a.n == 0 || a.d_out == 0) return cudaSuccess;
    const int vec = a.dtype == kBF16 ? 8 : 4;
    const size_t xs_bytes = (size_t)a.n * a.d_in * dtype_bytes(a.dtype);
    const size_t staged = (a.n <= 4 && a.dtype == kBF16) ? 2 * xs_bytes : xs_bytes;   // fp32 staging
    if (a.n <= kSmallRows && a.d_in % vec == 0 && staged <= kSmallMaxSmem)
        return a.dtype == kBF16 ? launch_small_t<__nv_bfloat16>(a, xs_bytes, st) : launch_small_t<float>(a, xs_bytes, st);
    dim3 grid((unsigned)((a.d_out + kLinBN - 1) / kLinBN), (unsigned)((a.n + kLinBM - 1) / kLinBM));
    note_launches(1);
    if (a.dtype == kBF16)
        linear_simt_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
    else
        linear_simt_kernel<float><<<grid, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace yoco
