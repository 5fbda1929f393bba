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

// A few rows (decode-step projections): the weight is read once, from HBM,
// by warps that each own four output columns and every row; x (a few KB per
// row) comes from L2.  LayerNorm statistics per row first, then each x value
// is normalised as it is loaded.
constexpr int kSmallRows = 16, kSmallCols = 4, kSmallWarps = 8;

template <typename T>
__global__ void __launch_bounds__(32 * kSmallWarps, 1) linear_small_kernel(const LinearArgs a) {
    constexpr int VEC = 16 / sizeof(T);  // elements per 16-byte load
    __shared__ float mu[kSmallRows], rs[kSmallRows];
    const T *x = static_cast<const T *>(a.x);
    const T *w = static_cast<const T *>(a.w);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = (int)a.n;
    for (int r = warp; r < n; r += kSmallWarps) {
        float mean = 0.f, rstd = 1.f;
        if (a.apply_ln) {
            const T *xr = x + (int64_t)r * a.d_in;
            float s1 = 0.f;
            for (int c = lane; c < a.d_in; c += 32) s1 += to_f32(xr[c]);
            mean = warp_sum(s1) / (float)a.d_in;
            float q = 0.f;
            for (int c = lane; c < a.d_in; c += 32) {
                const float t = to_f32(xr[c]) - mean;
                q = fmaf(t, t, q);
            }
            rstd = rsqrtf(warp_sum(q) / (float)a.d_in + a.eps);
        }
        if (lane == 0) {
            mu[r] = a.apply_ln ? mean : 0.f;
            rs[r] = a.apply_ln ? rstd : 1.f;
        }
    }
    __syncthreads();
    const int c0 = (blockIdx.x * kSmallWarps + warp) * kSmallCols;
    if (c0 >= a.d_out) return;
    float acc[kSmallRows][kSmallCols];
#pragma unroll
    for (int r = 0; r < kSmallRows; ++r)
#pragma unroll
        for (int j = 0; j < kSmallCols; ++j) acc[r][j] = 0.f;
    for (int d0 = lane * VEC; d0 < a.d_in; d0 += 32 * VEC) {
        float wv[kSmallCols][VEC];
#pragma unroll
        for (int j = 0; j < kSmallCols; ++j) {
            const int c = min(c0 + j, a.d_out - 1);
            const uint4 raw = *reinterpret_cast<const uint4 *>(w + (int64_t)c * a.d_in + d0);
            const T *e = reinterpret_cast<const T *>(&raw);
#pragma unroll
            for (int u = 0; u < VEC; ++u) wv[j][u] = to_f32(e[u]);
        }
#pragma unroll
        for (int r = 0; r < kSmallRows; ++r) {
            if (r >= n) break;
            const uint4 raw = *reinterpret_cast<const uint4 *>(x + (int64_t)r * a.d_in + d0);
            const T *e = reinterpret_cast<const T *>(&raw);
            const float m = mu[r], sc = rs[r];
#pragma unroll
            for (int u = 0; u < VEC; ++u) {
                const float xv = (to_f32(e[u]) - m) * sc;
#pragma unroll
                for (int j = 0; j < kSmallCols; ++j) acc[r][j] = fmaf(xv, wv[j][u], acc[r][j]);
            }
        }
    }
    const int w1 = a.d_out - a.split_col;
#pragma unroll
    for (int r = 0; r < kSmallRows; ++r) {
        if (r >= n) break;
#pragma unroll
        for (int j = 0; j < kSmallCols; ++j) {
            const float tot = warp_sum(acc[r][j]);
            const int c = c0 + j;
            if (lane != ((r * kSmallCols + j) & 31) || c >= a.d_out) continue;
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
}

cudaError_t launch_linear_simt(const LinearArgs &a, cudaStream_t st) {
    if (a.n == 0 || a.d_out == 0) return cudaSuccess;
    const int vec = a.dtype == kBF16 ? 8 : 4;
    if (a.n <= kSmallRows && a.d_in % vec == 0) {
        const int cols_per_cta = kSmallWarps * kSmallCols;
        note_launches(1);
        const int grid = (a.d_out + cols_per_cta - 1) / cols_per_cta;
        if (a.dtype == kBF16)
            linear_small_kernel<__nv_bfloat16><<<grid, 32 * kSmallWarps, 0, st>>>(a);
        else
            linear_small_kernel<float><<<grid, 32 * kSmallWarps, 0, st>>>(a);
        return cudaGetLastError();
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
