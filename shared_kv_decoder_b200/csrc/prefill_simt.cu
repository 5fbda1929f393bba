// CUDA-core causal / sliding-window GQA attention prefill.
//
// This is the fp32 path (the small fp32 stack) and the shape-agnostic
// path; bf16 prefill at scale runs on the tcgen05 kernel instead.
// Masks: "You Only Cache Once" (paperlayer summary), section 1
// "Architecture" (both halves causal) and section 3 "Sliding-Window
// Attention" (fixed window).  A query at position p sees keys j with
// j <= p and, when window > 0, j > p - window.
//
// One CTA owns 16 query rows of one (batch, query head); K/V tiles of 32
// keys are staged in shared memory as fp32 (K padded by one column so that
// lane-per-key dot products are bank-conflict free); each warp runs an
// online softmax (exp2 domain) for 4 rows: lanes own keys for Q.K^T and own
// head-dim slices for P.V.
#include "common.cuh"
#include "launch.h"

namespace yoco {

constexpr int kSimtBQ = 16;
constexpr int kSimtBK = 32;
constexpr int kSimtWarps = 4;
constexpr int kRowsPerWarp = kSimtBQ / kSimtWarps;

template <typename T, int D>
__global__ void __launch_bounds__(128) attn_prefill_simt_kernel(const PrefillArgs a, float scale_log2) {
    __shared__ float Qs[kSimtBQ][D];
    __shared__ float Ks[kSimtBK][D + 1];
    __shared__ float Vs[kSimtBK][D];
    __shared__ float Ps[kSimtWarps][kSimtBK];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t i0 = (int64_t)blockIdx.x * kSimtBQ;
    const int h = blockIdx.y, b = blockIdx.z;
    const int g = h / (a.Hq / a.Hkv);
    const T *q = static_cast<const T *>(a.q);
    const T *k = static_cast<const T *>(a.k);
    const T *v = static_cast<const T *>(a.v);
    T *o = static_cast<T *>(a.o);

    for (int idx = threadIdx.x; idx < kSimtBQ * D; idx += blockDim.x) {
        const int r = idx / D, d = idx % D;
        const int64_t i = i0 + r;
        Qs[r][d] = (i < a.Tq) ? to_f32(q[(((int64_t)b * a.Tq + i) * a.Hq + h) * D + d]) * scale_log2 : 0.f;
    }

    const int64_t i_last = min(i0 + kSimtBQ, a.Tq) - 1;
    const int64_t p_first = a.q_pos0 + i0, p_last = a.q_pos0 + i_last;
    const int64_t j_lo = a.window > 0 ? max((int64_t)0, p_first - a.window + 1) : 0;
    const int64_t j_hi = min(a.Tkv - 1, p_last);

    constexpr int DL = D / 32;
    float m[kRowsPerWarp], l[kRowsPerWarp], acc[kRowsPerWarp][DL];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.f;
#pragma unroll
        for (int e = 0; e < DL; ++e) acc[r][e] = 0.f;
    }

    for (int64_t j0 = j_lo; j0 <= j_hi; j0 += kSimtBK) {
        __syncthreads();
        for (int idx = threadIdx.x; idx < kSimtBK * D; idx += blockDim.x) {
            const int jj = idx / D, d = idx % D;
            const int64_t j = j0 + jj;
            const bool in = j <= j_hi;
            const int64_t off = (((int64_t)b * a.Tkv + j) * a.Hkv + g) * D + d;
            Ks[jj][d] = in ? to_f32(k[off]) : 0.f;
            Vs[jj][d] = in ? to_f32(v[off]) : 0.f;
        }
        __syncthreads();
        const int64_t j = j0 + lane;
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const int row = warp * kRowsPerWarp + r;
            const int64_t i = i0 + row;
            if (i >= a.Tq) break;
            const int64_t p = a.q_pos0 + i;
            const bool vis = j <= j_hi && j <= p && (a.window <= 0 || j > p - a.window);
            float s = 0.f;
#pragma unroll 8
            for (int d = 0; d < D; ++d) s = fmaf(Qs[row][d], Ks[lane][d], s);
            s = vis ? s : -INFINITY;
            const float mt = warp_max(s);
            const float mn = fmaxf(m[r], mt);
            const float alpha = (mn == -INFINITY) ? 1.f : exp2f(m[r] - mn);
            const float pj = vis ? exp2f(s - mn) : 0.f;
            l[r] = l[r] * alpha + warp_sum(pj);
            m[r] = mn;
            Ps[warp][lane] = pj;
            __syncwarp();
#pragma unroll
            for (int e = 0; e < DL; ++e) acc[r][e] *= alpha;
            for (int jj = 0; jj < kSimtBK; ++jj) {
                const float pv = Ps[warp][jj];
#pragma unroll
                for (int e = 0; e < DL; ++e) acc[r][e] = fmaf(pv, Vs[jj][lane + 32 * e], acc[r][e]);
            }
            __syncwarp();
        }
    }

#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
        const int64_t i = i0 + warp * kRowsPerWarp + r;
        if (i >= a.Tq) break;
        const float inv = l[r] > 0.f ? 1.f / l[r] : 0.f;
        T *dst = o + (((int64_t)b * a.Tq + i) * a.Hq + h) * D;
#pragma unroll
        for (int e = 0; e < DL; ++e) dst[lane + 32 * e] = from_f32<T>(acc[r][e] * inv);
        if (a.lse && lane == 0)
            a.lse[((int64_t)b * a.Hq + h) * a.Tq + i] = l[r] > 0.f ? (m[r] + log2f(l[r])) * kLn2 : -INFINITY;
    }
}

template <typename T>
static cudaError_t launch_simt_t(const PrefillArgs &a, cudaStream_t st) {
    dim3 grid((unsigned)((a.Tq + kSimtBQ - 1) / kSimtBQ), a.Hq, a.B);
    const float sl2 = a.scale * kLog2e;
    note_launches(1);
    if (a.D == 128)
        attn_prefill_simt_kernel<T, 128><<<grid, 128, 0, st>>>(a, sl2);
    else if (a.D == 64)
        attn_prefill_simt_kernel<T, 64><<<grid, 128, 0, st>>>(a, sl2);
    else
        return cudaErrorNotSupported;
    return cudaGetLastError();
}

cudaError_t launch_prefill_simt(const PrefillArgs &a, cudaStream_t st) {
    if (a.B == 0 || a.Tq == 0) return cudaSuccess;
    return a.dtype == kBF16 ? launch_simt_t<__nv_bfloat16>(a, st) : launch_simt_t<float>(a, st);
}

}  // namespace yoco
