// K/V producer on the sm_100a tensor cores: LayerNorm, projection and the
// YOCO++ weighted residual in one kernel (bf16 in, fp32 accumulate).
//
//   out[t, c] = rstd_t * (x[t, :] . W[c, :] - mu_t * colsum_c) + w * base[t, c]
//
// which equals LN(x)[t, :] . W[c, :] + w * base[t, c] (podcast transcript
// "YOCO: Caching Once ...", cue 12: normalised once, projected by one pair
// of matrices; "YOCO++ ...", Abstract: weighted residual to the bottom
// layer's KV), so x is read from HBM once, un-normalised, and the blend is
// applied while the accumulator drains -- no extra pass over memory.
//
//  * Tile: 127 token rows x 256 output features per MMA chunk; a CTA sweeps
//    a group of 256-wide chunks of the same rows, so its x rows stream from
//    L2 after the first chunk.  A = x tile [128 x 64] K-major, 128-byte
//    swizzle, loaded by TMA as 127 rows; row 127 of every A stage is a fixed
//    row of ones, so accumulator row 127 is colsum_c = sum_k W[c, k], computed
//    by the tensor core for free.
//  * Row statistics (mean, variance, shifted by the row's first element for
//    accuracy) come from the A tiles already in shared memory: during the
//    first chunk the epilogue warps read each stage once before it is
//    recycled.
//  * Warp roles: 0-3 epilogue (thread r = TMEM lane r = tile row r), 4 TMA
//    producer, 5 MMA issuer.  TMEM holds two 256-column accumulators so the
//    epilogue of chunk i overlaps the MMAs of chunk i+1.  Four-stage
//    A/B ring.  Output columns below split_col go to out0, the rest to out1;
//    dst_rows scatters rows (appending to the shared cache).
// All mbarrier waits are bounded (status word + abort flag); see prefill_tc.cu.
// The epilogue warps' one named barrier is a vote that all four reach on
// every chunk, so a wait that gives up in one of them releases all of them.
#include <cuda.h>

#include <algorithm>

#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace yoco {

static __device__ unsigned int g_status_project_tc;

namespace {

constexpr int kRowsA = 127;           // token rows per tile (row 127 = ones)
constexpr int kBN = 256;              // output features per chunk
constexpr int kBK = 64;               // K per stage (one 128-byte swizzle atom)
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr uint32_t kABytes = 128 * 128;           // [128 rows x 128 B]
constexpr uint32_t kBBytes = kBN * 128;           // [256 rows x 128 B]
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kSmemStages = kStages * kStageBytes;
constexpr uint32_t kSmemColsum = kSmemStages;             // [2][256] fp32
constexpr uint32_t kSmemBar = kSmemColsum + 2 * kBN * 4;
constexpr uint32_t kSmemBytes = kSmemBar + 256;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;

enum Bar {
    kFull = 0,        // kStages
    kEmpty = 4,       // kStages
    kARead = 8,       // kStages (epilogue read a stage for statistics)
    kAccFull = 12,    // 2
    kAccEmpty = 14,   // 2
    kDrain = 16,
    kNumBars = 17
};

struct ProjParams {
    int64_t n;
    int32_t d, m;
    int32_t apply_ln;
    float eps;
    int32_t split_col;
    void *out0, *out1;
    const void *base0, *base1;
    float w0, w1;
    const int64_t *dst_rows;
    int32_t chunks_per_cta;
    int32_t groups;  // CTAs per row tile (column groups), adjacent in launch order
};

YOCO_DEV bool wait1(uint64_t *bar, uint32_t parity) {
    return mbar_wait(bar, parity, &g_status_project_tc);
}
YOCO_DEV bool waitw(uint64_t *bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, &g_status_project_tc));
}
// Named barrier of the four epilogue warps with an OR vote: true for every
// thread if any thread passed true.
YOCO_DEV bool epi_bar_any(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    project_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                      const ProjParams p) {
    if (*(volatile unsigned int *)&g_status_project_tc) return;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t *sbase = smem_raw + (base - raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sbase + kSmemBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sbase + kSmemBar + kNumBars * 8);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sbase + kSmemBar + kNumBars * 8 + 4);
    float *colsum = reinterpret_cast<float *>(sbase + kSmemColsum);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the column groups of one row tile are adjacent CTAs, so they run at the
    // same time and their reads of the row tile's x are shared through L2
    const int64_t row0 = (int64_t)(blockIdx.x / p.groups) * kRowsA;
    const int chunk0 = (int)(blockIdx.x % p.groups) * p.chunks_per_cta;
    const int n_chunks = min(p.chunks_per_cta, p.m / kBN - chunk0);
    const int kblocks = (p.d + kBK - 1) / kBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars[kFull + s], 1);
            mbar_init(&bars[kEmpty + s], 1);
            mbar_init(&bars[kARead + s], 4);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bars[kAccFull + s], 1);
            mbar_init(&bars[kAccEmpty + s], 128);
        }
        mbar_init(&bars[kDrain], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    // row 127 of every A stage: bf16 ones (every 16-byte chunk identical, so
    // the swizzle does not matter); TMA only ever writes rows 0..126
    for (int s = 0; s < kStages; ++s)
        if (threadIdx.x < 8)
            *reinterpret_cast<uint4 *>(sbase + s * kStageBytes + 127 * 128 + threadIdx.x * 16) =
                make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    fence_proxy_async_smem();
    if (warp == 5) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const int total = n_chunks * kblocks;  // pipeline iterations

    if (warp == 4) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            int issued = 0;
            for (int itr = 0; itr < total; ++itr) {
                const int st = itr % kStages;
                const uint32_t ph = ((itr / kStages) & 1) ^ 1;
                if (!wait1(&bars[kEmpty + st], ph)) { *abort_flag = 1; break; }
                const int prev = itr - kStages;  // previous user of this stage
                if (prev >= 0 && prev < kblocks && !wait1(&bars[kARead + st], (prev / kStages) & 1)) {
                    *abort_flag = 1;
                    break;
                }
                if (*abort_flag) break;
                const int c = chunk0 + itr / kblocks, kb = itr % kblocks;
                const uint32_t sa = base + st * kStageBytes;
                mbar_arrive_expect_tx(&bars[kFull + st], kRowsA * 128 + kBBytes);
                tc::tma_load_4d(sa, &tm_x, kb * kBK, (int)row0, 0, 0, &bars[kFull + st]);
                tc::tma_load_4d(sa + kABytes, &tm_w, kb * kBK, c * kBN, 0, 0, &bars[kFull + st]);
                ++issued;
            }
            for (int itr = max(0, issued - kStages); itr < issued; ++itr)
                if (!wait1(&bars[kFull + itr % kStages], (itr / kStages) & 1)) break;
        }
    } else if (warp == 5) {
        // -------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_bf16(128, kBN, false, false);
            bool ok = true;
            for (int ci = 0; ci < n_chunks && ok; ++ci) {
                const int ab = ci & 1;
                if (ci >= 2 && !wait1(&bars[kAccEmpty + ab], ((ci - 2) >> 1) & 1)) { ok = false; break; }
                tc::fence_after_sync();
                for (int kb = 0; kb < kblocks; ++kb) {
                    const int itr = ci * kblocks + kb;
                    const int st = itr % kStages;
                    if (!wait1(&bars[kFull + st], (itr / kStages) & 1) || *abort_flag) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t sa = base + st * kStageBytes;
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const uint64_t ad = tc::smem_desc_sw128(sa + kk * 32, 16, 1024);
                        const uint64_t bd = tc::smem_desc_sw128(sa + kABytes + kk * 32, 16, 1024);
                        tc::mma_bf16_ss(tmem + ab * kBN, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc::mma_commit(&bars[kEmpty + st]);
                }
                if (ok) tc::mma_commit(&bars[kAccFull + ab]);
            }
            if (!ok) *abort_flag = 1;
            tc::mma_commit(&bars[kDrain]);
            wait1(&bars[kDrain], 0);
        }
    } else {
        // --------------------------------------------------------- epilogue
        const int r = threadIdx.x;
        const int64_t tok = row0 + r;
        const bool real_row = r < kRowsA && tok < p.n;
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        bool ok = true;
        // row statistics from the A stages of the first chunk
        float mu = 0.f, rstd = 1.f;
        {
            float shift = 0.f, s1 = 0.f, s2 = 0.f;
            for (int kb = 0; kb < kblocks && n_chunks > 0; ++kb) {
                const int st = kb % kStages;
                if (!waitw(&bars[kFull + st], (kb / kStages) & 1)) { ok = false; break; }
                if (p.apply_ln) {
                    const uint8_t *rowp = sbase + st * kStageBytes + r * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint4 raw4 = *reinterpret_cast<const uint4 *>(rowp + ((c ^ (r & 7)) << 4));
                        float f[8];
                        Chunk<__nv_bfloat16>::unpack(raw4, f);
                        if (kb == 0 && c == 0) shift = f[0];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int kk = kb * kBK + c * 8 + e;
                            const float v = kk < p.d ? f[e] - shift : 0.f;
                            s1 += v;
                            s2 = fmaf(v, v, s2);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[kARead + st]);
            }
            if (p.apply_ln) {
                const float inv_d = 1.f / (float)p.d;
                const float m1 = s1 * inv_d;
                const float var = fmaxf(s2 * inv_d - m1 * m1, 0.f);
                mu = shift + m1;
                rstd = rsqrtf(var + p.eps);
            }
        }
        const int w1 = p.m - p.split_col;
        const int64_t drow = real_row ? (p.dst_rows ? p.dst_rows[tok] : tok) : 0;
        // every epilogue warp enters this loop and reaches the vote on each
        // chunk (a failed statistics wait included); any failure ends all four
        for (int ci = 0; ci < n_chunks; ++ci) {
            const int ab = ci & 1;
            const bool got = ok && waitw(&bars[kAccFull + ab], (ci >> 1) & 1);
            const uint32_t tacc = tmem + lane_off + ab * kBN;
            float *cs = colsum + ab * kBN;
            if (got) {
                tc::fence_after_sync();
                if (warp == 3) {  // lane 31 of warp 3 holds row 127: colsum of W
#pragma unroll 1
                    for (int cc = 0; cc < kBN; cc += 32) {
                        float v[32];
                        tc::tmem_ld32(tacc + cc, v);
                        tc::wait_ld();
                        if (lane == 31)
#pragma unroll
                            for (int e = 0; e < 32; ++e) cs[cc + e] = v[e];
                    }
                }
            }
            if (epi_bar_any(!got)) { ok = false; break; }
            const int col0 = (chunk0 + ci) * kBN;
#pragma unroll 1
            for (int cc = 0; cc < kBN; cc += 32) {
                float v[32];
                tc::tmem_ld32(tacc + cc, v);
                tc::wait_ld();
                if (real_row) {
                    const int c = col0 + cc;  // 32 columns, all on one side of split_col
                    const bool first = c < p.split_col;
                    const int cl = first ? c : c - p.split_col;
                    const int wd = first ? p.split_col : w1;
                    const __nv_bfloat16 *bp = static_cast<const __nv_bfloat16 *>(first ? p.base0 : p.base1);
                    const float bw = first ? p.w0 : p.w1;
                    __nv_bfloat16 *op = static_cast<__nv_bfloat16 *>(first ? p.out0 : p.out1) + drow * wd + cl;
                    float bv[32];
                    if (bp) {
                        const uint4 *b4 = reinterpret_cast<const uint4 *>(bp + tok * wd + cl);
#pragma unroll
                        for (int q = 0; q < 4; ++q) Chunk<__nv_bfloat16>::unpack(b4[q], bv + 8 * q);
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float y[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int j = 8 * q + e;
                            float t = rstd * (v[j] - mu * cs[cc + j]);
                            if (bp) t = fmaf(bw, bv[j], t);
                            y[e] = t;
                        }
                        uint4 w;
                        w.x = tc::pack_bf16x2(y[0], y[1]);
                        w.y = tc::pack_bf16x2(y[2], y[3]);
                        w.z = tc::pack_bf16x2(y[4], y[5]);
                        w.w = tc::pack_bf16x2(y[6], y[7]);
                        reinterpret_cast<uint4 *>(op)[q] = w;
                    }
                }
            }
            tc::fence_before_sync();
            mbar_arrive(&bars[kAccEmpty + ab]);
        }
        if (!ok) *abort_flag = 1;
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------- host
namespace {

// 4-D view {K, rows, 1, 1} of a row-major bf16 matrix, box {64, box_rows, 1, 1}.
bool make_map(CUtensorMap *m, const void *ptr, int64_t rows, int64_t K, uint32_t box_rows) {
    const uint64_t dims[4] = {(uint64_t)K, (uint64_t)rows, 1, 1};
    const uint64_t strides[3] = {(uint64_t)(K * 2), (uint64_t)(rows * K * 2), (uint64_t)(rows * K * 2)};
    const uint32_t box[4] = {64, box_rows, 1, 1};
    return encode_bf16_map_4d(m, ptr, dims, strides, box);
}

}  // namespace

// Small token counts stay on the CUDA-core kernel (a weight-read-bound GEMV
// there); the tensor-core kernel needs bf16, 256-multiple outputs and
// 128-multiple column splits.
cudaError_t launch_linear_tc(const LinearArgs &a, cudaStream_t st) {
    if (a.dtype != kBF16 || a.n < 512 || a.d_out % kBN != 0 || a.split_col % 32 != 0 ||
        (a.d_out - a.split_col) % 32 != 0 || (int64_t)a.d_in * 2 % 16 != 0)
        return cudaErrorNotSupported;
    CUtensorMap mx, mw;
    if (!make_map(&mx, a.x, a.n, a.d_in, kRowsA) || !make_map(&mw, a.w, a.d_out, a.d_in, kBN))
        return cudaErrorNotSupported;
    ProjParams p;
    p.n = a.n; p.d = a.d_in; p.m = a.d_out; p.apply_ln = a.apply_ln; p.eps = a.eps;
    p.split_col = a.split_col; p.out0 = a.out0; p.out1 = a.out1; p.base0 = a.base0;
    p.base1 = a.base1; p.w0 = a.w0; p.w1 = a.w1; p.dst_rows = a.dst_rows;
    const int64_t mtiles = (a.n + kRowsA - 1) / kRowsA;
    const int nchunks = a.d_out / kBN;
    // four 256-column chunks per CTA: the measured best of 1, 2, 4 and all 8 at
    // 32K and 256K tokens (the epilogue of one chunk overlaps the next chunk's
    // MMAs, and the few CTAs of a row tile share its x reads in L2)
    p.chunks_per_cta = std::min(nchunks, 4);
    p.groups = (nchunks + p.chunks_per_cta - 1) / p.chunks_per_cta;
    if (mtiles * p.groups > 0x7fffffff) return cudaErrorNotSupported;
    cudaError_t e = cudaFuncSetAttribute(project_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemAlloc);
    if (e != cudaSuccess) return e;
    note_launches(1);
    project_tc_kernel<<<(unsigned)(mtiles * p.groups), kThreads, kSmemAlloc, st>>>(mx, mw, p);
    return cudaGetLastError();
}

unsigned int read_and_clear_status_project_tc() {
    unsigned int h = 0, z = 0;
    if (cudaMemcpyFromSymbol(&h, g_status_project_tc, sizeof(h)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_status_project_tc, &z, sizeof(z));
    return h;
}

}  // namespace yoco
