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
// (256 CTAs for a 2048-wide [K | V]); each lane first issues every 16-byte
// load of its slice of the column's weight row (up to 16 in flight per lane),
// then the CTA stages its x rows in shared memory, takes each row's
// LayerNorm statistics from there, and the warp forms the n dot products
// against the registers, normalising x as it reads it.  An earlier version
// with four columns per warp and 64 CTAs kept too few loads in flight: the
// 16.8 MB weight of a d=4096 K/V projection took ~16 us to stream.
constexpr int kSmallRows = 16, kSmallWarps = 8, kSmallChunks = 16;
constexpr size_t kSmallMaxSmem = 200 * 1024;

template <typename T>
__global__ void __launch_bounds__(32 * kSmallWarps, 2) linear_small_kernel(const LinearArgs a) {
    constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte chunk
    extern __shared__ uint4 xs4[];       // the n x rows, [n][d_in]
    __shared__ float mu[kSmallRows], rs[kSmallRows];
    const T *x = static_cast<const T *>(a.x);
    const T *w = static_cast<const T *>(a.w);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = (int)a.n;
    const int row_chunks = a.d_in / VEC;          // 16-byte chunks per row
    const int c = blockIdx.x * kSmallWarps + warp;  // this warp's output column
    const uint4 *wrow = reinterpret_cast<const uint4 *>(w + (int64_t)min(c, a.d_out - 1) * a.d_in);
    // while the previous kernel finishes: ask L2 for this warp's weight row
    // (a prefetch only warms the cache; nothing is read before pdl_wait)
    pdl_trigger();
    for (int ch = lane * 8; ch < row_chunks; ch += 256)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(wrow + ch));
    pdl_wait();
    // this lane's chunks of the weight row: lane, lane + 32, ... (blocks of 16)
    uint4 wr[kSmallChunks];
#pragma unroll
    for (int k = 0; k < kSmallChunks; ++k)
        if (lane + 32 * k < row_chunks) wr[k] = wrow[lane + 32 * k];
    // stage x (every thread), then the statistics of each row
    const uint4 *x4 = reinterpret_cast<const uint4 *>(x);
    for (int i = threadIdx.x; i < n * row_chunks; i += blockDim.x) xs4[i] = x4[i];
    __syncthreads();
    const T *xs = reinterpret_cast<const T *>(xs4);
    for (int r = warp; r < n; r += kSmallWarps) {
        float mean = 0.f, rstd = 1.f;
        if (a.apply_ln) {
            const T *xr = xs + (int64_t)r * a.d_in;
            float s1 = 0.f;
            for (int cc = lane; cc < a.d_in; cc += 32) s1 += to_f32(xr[cc]);
            mean = warp_sum(s1) / (float)a.d_in;
            float q = 0.f;
            for (int cc = lane; cc < a.d_in; cc += 32) {
                const float t = to_f32(xr[cc]) - mean;
                q = fmaf(t, t, q);
            }
            rstd = rsqrtf(warp_sum(q) / (float)a.d_in + a.eps);
        }
        if (lane == 0) {
            mu[r] = mean;
            rs[r] = rstd;
        }
    }
    __syncthreads();
    if (c >= a.d_out) return;
    float acc[kSmallRows];
#pragma unroll
    for (int r = 0; r < kSmallRows; ++r) acc[r] = 0.f;
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
            const T *we = reinterpret_cast<const T *>(&wr[k]);
            float wv[VEC];
#pragma unroll
            for (int u = 0; u < VEC; ++u) wv[u] = to_f32(we[u]);
#pragma unroll
            for (int r = 0; r < kSmallRows; ++r) {
                if (r >= n) break;
                const uint4 raw = xs4[(int64_t)r * row_chunks + ch];
                const T *e = reinterpret_cast<const T *>(&raw);
                const float m = mu[r], sc = rs[r];
                float d = 0.f;
#pragma unroll
                for (int u = 0; u < VEC; ++u) d = fmaf((to_f32(e[u]) - m) * sc, wv[u], d);
                acc[r] += d;
            }
        }
    }
    const int w1 = a.d_out - a.split_col;
#pragma unroll
    for (int r = 0; r < kSmallRows; ++r) {
        if (r >= n) break;
        const float tot = warp_sum(acc[r]);
        if (lane != (r & 31)) continue;
        const int64_t dr = a.dst_rows ? a.dst_rows[r] : r;
        float val = tot;
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

cudaError_t launch_linear_simt(const LinearArgs &a, cudaStream_t st) {
    if (a.n == 0 || a.d_out == 0) return cudaSuccess;
    const int vec = a.dtype == kBF16 ? 8 : 4;
    const size_t xs_bytes = (size_t)a.n * a.d_in * dtype_bytes(a.dtype);
    if (a.n <= kSmallRows && a.d_in % vec == 0 && xs_bytes <= kSmallMaxSmem) {
        const int grid = (a.d_out + kSmallWarps - 1) / kSmallWarps;
        cudaError_t e;
        if (a.dtype == kBF16) {
            auto kern = linear_small_kernel<__nv_bfloat16>;
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmallMaxSmem);
            if (e != cudaSuccess) return e;
            note_launches(1);
            e = launch_pdl(kern, dim3(grid), dim3(32 * kSmallWarps), xs_bytes, st, a);
        } else {
            auto kern = linear_small_kernel<float>;
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmallMaxSmem);
            if (e != cudaSuccess) return e;
            note_launches(1);
            e = launch_pdl(kern, dim3(grid), dim3(32 * kSmallWarps), xs_bytes, st, a);
        }
        return e;
    }
    dim3 grid((unsigned)((a.d_out + kLinBN - 1) / kLinBN), (unsigned)((a.n + kLinBM - 1) / kLinBM));
    note_launches(1);
    if (a.dtype == kBF16)
        linear_simt_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a);
    else
        linear_simt_kernel<float><<<grid, 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace yoco
