// Sliding-window decode step over the ring in ONE launch: the window read,
// the merge of its partials, the new token, and the new token's ring write.
//
// What it computes is the decode step of the self-decoder ("You Only Cache
// Once", paperlayer summary, section 3 "Sliding-Window Attention": each layer
// keeps only the last W tokens' K/V; the new token attends to the visible
// slots of its window and then takes the slot of the token that falls out):
//   o_h = softmax over {visible ring slots} + {new token} of (q_h . k / sqrt(D)) v
// with GQA (query head h reads KV head h / G).  A ring slot is visible when it
// is not the new token's slot (pos mod W, whose old token leaves the window)
// and its position p satisfies pos - W < p <= pos, p >= 0.
//
// Work split: one thread-block cluster per (sequence b, KV head g), C <= 8
// CTAs.  CTA `rank` reads slots [rank * per, (rank + 1) * per) of head g in
// chunks of 128 slots (one TMA box of K and of V per 64-column block; the box
// covers a single KV head, so the bytes of other heads are never touched).
// Eight consumer warps take 16 slots of a chunk each: S = q K^T and O += P V
// are m16n8k16 tensor-core MMAs with the G query heads as the M rows (as in
// the split-KV decode), under an online softmax in the log2 domain.  The
// warps' partials (m, l, o) merge in shared memory into the CTA's partial,
// which the CTA stores straight into rank 0's shared memory (distributed
// shared memory, one slot per rank).  After one cluster barrier rank 0 merges
// the C partials from its own shared memory, adds the new token as one more
// partial (q . k_new and v_new, read while the copies were in flight), writes
// o, and writes k_new / v_new into slot pos mod W (and, in the g = 0 cluster,
// slot_pos).
//
// Against the split kernel + merge kernel of the cross decode, this saves a
// launch and its dependent latency per step, and no partials go through
// global memory.  No CTA waits on another CTA outside its cluster, so there is
// no global counter and no grid-wide wait.
//
// Every mbarrier wait is bounded; a wait that gives up sets the status word
// and the CTA skips the rest of its arithmetic but still takes the cluster
// barrier (and waits, bounded, for its own copies in flight) so that no
// thread of the cluster waits for it.
#include <cuda.h>

#include <algorithm>
#include <cstdint>

#include "cluster.cuh"
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace yoco {

static __device__ unsigned int g_status_ring;

namespace {

using namespace wmma16;

constexpr int kWarps = 8;                   // consumer warps
constexpr int kThreads = 32 * (kWarps + 1); // + one producer warp
constexpr int kChunk = 128;                 // slots per chunk (TMA box rows)
constexpr int kWarpTok = kChunk / kWarps;   // 16 slots per warp per chunk
constexpr int kMaxCluster = 8;
constexpr uint32_t kBoxBytes = kChunk * 128;  // 128 rows of 128 bytes

struct RingParams {
    const __nv_bfloat16 *q;              // [B, Hq, D]
    const __nv_bfloat16 *k_new, *v_new;  // [B, Hkv, D]
    const int64_t *pos;                  // [B]
    __nv_bfloat16 *ring_k, *ring_v;      // [B, W, Hkv, D]
    int32_t *slot_pos;                   // [B, W]
    __nv_bfloat16 *o;                    // [B, Hq, D]
    int32_t B, Hq, Hkv, window;
    int32_t per;       // slots per CTA (a multiple of 16)
    int32_t chunks;    // chunks per CTA
    int32_t stages;    // 1 or 2
    float scale_log2;
};

// Shared memory: the stages, then 64 bytes of barriers, then (floats) the
// gathered partials [kMaxCluster][G][D + 2] (o, then m and l), the new
// token's scores s_new[G] and value row v_new[D], and the skip flag.
template <int D, int G>
struct RingSmem {
    static constexpr int KB = D / 64;
    static constexpr uint32_t STAGE = 2 * KB * kBoxBytes;  // K boxes then V boxes
    static constexpr int PART = D + 2;                     // floats of one head's partial
    static constexpr uint32_t FLOATS = kMaxCluster * G * PART + G + D + 1;
    static size_t bytes(int stages) { return (size_t)stages * STAGE + 64 + FLOATS * sizeof(float) + 1024; }
};

YOCO_DEV void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(32 * kWarps) : "memory"); }

YOCO_DEV bool wait_bar(uint64_t *bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, &g_status_ring));
}

}  // namespace

// two 288-thread CTAs an SM (ptxas then keeps a thread within 96 registers;
// a 112-register cap measured 25% slower)
template <int D, int G>
__global__ void __launch_bounds__(kThreads, 2) ring_decode_cluster_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                                          const __grid_constant__ CUtensorMap tm_v,
                                                                          const RingParams p) {
    static_assert(G >= 1 && G <= 8, "query heads per KV head");
    using L = RingSmem<D, G>;
    constexpr int PART = L::PART;
    constexpr int KB = L::KB;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;  // the 128-byte swizzle repeats every 1024 bytes
    unsigned char *smem = smem_raw + (sbase - raw);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + (size_t)p.stages * L::STAGE);
    uint64_t *empty = full + 2;
    float *gather = reinterpret_cast<float *>(smem + (size_t)p.stages * L::STAGE + 64);
    float *s_new = gather + kMaxCluster * G * PART;
    float *v_new = s_new + G;
    volatile int *skip = reinterpret_cast<volatile int *>(v_new + D);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const uint32_t rank = clu::rank(), C = clu::size();
    const int bg = (int)(blockIdx.x / C);
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int s0 = (int)rank * p.per;
    const int s1 = min(p.window, s0 + p.per);

    pdl_trigger();
    if (threadIdx.x == 32 * kWarps) {
        // the CTA's K and V boxes into L2 while the previous kernel finishes
        // (a prefetch changes no data, so it may run before the wait)
        for (int c = 0; c < p.chunks; ++c)
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                tc::tma_prefetch_4d(&tm_k, kb * 64, g, s0 + c * kChunk, b);
                tc::tma_prefetch_4d(&tm_v, kb * 64, g, s0 + c * kChunk, b);
            }
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kWarps);
        }
        fence_mbar_init();
    }
    pdl_wait();
    if (threadIdx.x == 0) *skip = (*(volatile unsigned int *)&g_status_ring) != 0;
    __syncthreads();
    // first cluster phase: every CTA of the cluster is running before any
    // writes into another's shared memory (waited for just before that)
    clu::arrive_relaxed();

    const int64_t pos_b = p.pos[b];
    const int W = p.window;
    const int new_slot = (int)(((pos_b % W) + W) % W);

    if (warp == kWarps) {
        // ------------------------------------------------------------ producer
        uint32_t issued = 0;
        auto issue = [&](int c) -> bool {
            const int st = c % p.stages;
            const uint32_t ph = (uint32_t)(c / p.stages) & 1u;
            if (!mbar_wait(&empty[st], ph ^ 1u, &g_status_ring)) return false;
            const uint32_t dst = sbase + (uint32_t)st * L::STAGE;
            mbar_arrive_expect_tx(&full[st], L::STAGE);
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                tc::tma_load_4d(dst + kb * kBoxBytes, &tm_k, kb * 64, g, s0 + c * kChunk, b, &full[st]);
                tc::tma_load_4d(dst + (KB + kb) * kBoxBytes, &tm_v, kb * 64, g, s0 + c * kChunk, b, &full[st]);
            }
            ++issued;
            return true;
        };
        const int first = min(p.chunks, p.stages);   // their stages are free: no wait
        if (lane == 0 && !*skip)
            for (int c = 0; c < first; ++c) issue(c);
        __syncwarp();
        if (rank == 0) {
            // rank 0's merge needs the new token: its score for each query
            // head of the group (log2 domain) and its value row, read while
            // the copies are in flight
            const __nv_bfloat16 *kn = p.k_new + ((int64_t)b * p.Hkv + g) * D;
            float kv[D / 32];
#pragma unroll
            for (int i = 0; i < D / 32; ++i) kv[i] = __bfloat162float(kn[lane + 32 * i]);
#pragma unroll
            for (int hq = 0; hq < G; ++hq) {
                const __nv_bfloat16 *qr = p.q + ((int64_t)b * p.Hq + (int64_t)g * G + hq) * D;
                float dot = 0.f;
#pragma unroll
                for (int i = 0; i < D / 32; ++i) dot = fmaf(__bfloat162float(qr[lane + 32 * i]), kv[i], dot);
                dot = warp_sum(dot);
                if (lane == 0) s_new[hq] = dot * p.scale_log2;
            }
            for (int i = lane; i < D; i += 32) v_new[i] = __bfloat162float(p.v_new[((int64_t)b * p.Hkv + g) * D + i]);
        }
        if (lane == 0 && !*skip) {
            bool ok = issued == (uint32_t)first;
            for (int c = first; c < p.chunks && ok; ++c) ok = issue(c);
            // the copies issued must have landed before this CTA's shared
            // memory is reused or released (at once on the normal path)
            for (uint32_t c = issued > (uint32_t)p.stages ? issued - p.stages : 0; c < issued; ++c)
                if (!mbar_wait(&full[c % p.stages], (c / p.stages) & 1u, &g_status_ring)) break;
        }
        __syncwarp();
        clu::wait();
    } else {
        // ----------------------------------------------------------- consumers
        const int gq = lane >> 2;   // fragment row: query head of the group
        const int t = lane & 3;
        uint32_t qa[D / 16][2];
        if (gq < G) {
            const __nv_bfloat16 *qr = p.q + ((int64_t)b * p.Hq + (int64_t)g * G + gq) * D;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                qa[kk][0] = *reinterpret_cast<const uint32_t *>(qr + 16 * kk + 2 * t);
                qa[kk][1] = *reinterpret_cast<const uint32_t *>(qr + 16 * kk + 8 + 2 * t);
            }
        } else {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) qa[kk][0] = qa[kk][1] = 0u;
        }
        float o[D / 8][4];
#pragma unroll
        for (int n = 0; n < D / 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
        float m = -INFINITY, l = 0.f;
        const int tok0 = warp * kWarpTok;
        // ldmatrix rows and swizzle terms (row R keeps 16-byte chunk c at c ^ (R & 7))
        const int mat = lane >> 3, rr = lane & 7;
        const uint32_t rowS = (uint32_t)(tok0 + 8 * (mat >> 1) + rr) * 128u;
        const uint32_t xs = (uint32_t)((mat & 1) ^ rr);
        const uint32_t rowP = (uint32_t)(tok0 + 8 * (mat & 1) + rr) * 128u;
        const uint32_t xp = (uint32_t)((mat >> 1) ^ rr);
        const int32_t *sp = p.slot_pos + (int64_t)b * W;
        bool ok = !*skip;
        for (int c = 0; c < p.chunks && ok; ++c) {
            const int st = c % p.stages;
            const uint32_t ph = (uint32_t)(c / p.stages) & 1u;
            // the positions of this lane's four slots, read before the wait
            // (-1 marks a slot that is out of range or is the new token's)
            int32_t ps[2][2];
#pragma unroll
            for (int n = 0; n < 2; ++n)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int slot = s0 + c * kChunk + tok0 + 8 * n + 2 * t + e;
                    ps[n][e] = (slot < s1 && slot != new_slot) ? sp[slot] : -1;
                }
            if (!wait_bar(&full[st], ph)) { ok = false; break; }
            const uint32_t kst = sbase + (uint32_t)st * L::STAGE;
            const uint32_t vst = kst + KB * kBoxBytes;
            float sc[2][4];
#pragma unroll
            for (int n = 0; n < 2; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(kst + (uint32_t)(kk >> 2) * kBoxBytes + rowS + (((uint32_t)((kk & 3) << 1) ^ xs) << 4),
                        b0, b1, b2, b3);
                mma_rows8(sc[0], qa[kk][0], qa[kk][1], b0, b1);
                mma_rows8(sc[1], qa[kk][0], qa[kk][1], b2, b3);
            }
            float pv[2][2];
            float mx = -INFINITY;
#pragma unroll
            for (int n = 0; n < 2; ++n) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int32_t q_ps = ps[n][e];
                    const bool vld = q_ps >= 0 && q_ps <= pos_b && (int64_t)q_ps > pos_b - W;
                    const float v = vld ? sc[n][e] * p.scale_log2 : -INFINITY;
                    pv[n][e] = v;
                    mx = fmaxf(mx, v);
                }
            }
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            if (mx > m + 8.f) {
                // the reference max moves only when it grows by more than 2^8
                const float alpha = (m == -INFINITY) ? 0.f : tc::ex2(m - mx);
                m = mx;
                l *= alpha;
#pragma unroll
                for (int n = 0; n < D / 8; ++n) {
                    o[n][0] *= alpha;
                    o[n][1] *= alpha;
                }
            }
            const float neg_m = (m == -INFINITY) ? 0.f : -m;
            const float p00 = tc::ex2(pv[0][0] + neg_m), p01 = tc::ex2(pv[0][1] + neg_m);
            const float p10 = tc::ex2(pv[1][0] + neg_m), p11 = tc::ex2(pv[1][1] + neg_m);
            l += (p00 + p01) + (p10 + p11);
            const uint32_t a0 = tc::pack_bf16x2(p00, p01);
            const uint32_t a2 = tc::pack_bf16x2(p10, p11);
#pragma unroll
            for (int n = 0; n < D / 8; n += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(vst + (uint32_t)(n >> 3) * kBoxBytes + rowP + ((((uint32_t)n & 7u) ^ xp) << 4), b0, b1,
                          b2, b3);
                mma_rows8(o[n], a0, a2, b0, b1);
                mma_rows8(o[n + 1], a0, a2, b2, b3);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
        }
        if (!ok) *skip = 1;
        // l over the quad of lanes that share a row; o columns are disjoint
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);

        // the warps' partials into stage 0, once every warp is done with it
        consumers_sync();
        float *wp = reinterpret_cast<float *>(smem);          // [warp][G][D + 2]
        if (gq < G) {
            float *dst = wp + ((size_t)warp * G + gq) * (D + 2);
#pragma unroll
            for (int n = 0; n < D / 8; ++n) {
                dst[8 * n + 2 * t] = o[n][0];
                dst[8 * n + 2 * t + 1] = o[n][1];
            }
            if (t == 0) {
                dst[D] = m;
                dst[D + 1] = l;
            }
        }
        consumers_sync();
        clu::wait();
        // the CTA's partial: the warps' partials under one reference max,
        // stored into slot `rank` of rank 0's gather area
        const uint32_t dst0 = clu::map_rank(smem_u32(gather), 0) + 4u * (rank * G * PART);
        for (int idx = threadIdx.x; idx < G * D; idx += 32 * kWarps) {
            const int hq = idx / D, d = idx % D;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) M = fmaxf(M, wp[((size_t)w * G + hq) * (D + 2) + D]);
            float acc = 0.f, Ls = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
                const float *src = wp + ((size_t)w * G + hq) * (D + 2);
                const float f = (src[D] == -INFINITY) ? 0.f : tc::ex2(src[D] - M);
                acc = fmaf(src[d], f, acc);
                Ls = fmaf(src[D + 1], f, Ls);
            }
            clu::st_f32(dst0 + 4u * (hq * PART + d), acc);
            if (d == 0) {
                clu::st_f32(dst0 + 4u * (hq * PART + D), M);
                clu::st_f32(dst0 + 4u * (hq * PART + D + 1), Ls);
            }
        }
    }

    // ---------------------------------------------------- cluster merge (rank 0)
    // the barrier's release / acquire makes every rank's stores into the
    // gather area visible here; after it no CTA touches another's memory
    clu::sync_all();
    if (rank == 0 && warp < kWarps && !*skip) {
        for (int idx = threadIdx.x; idx < G * D; idx += 32 * kWarps) {
            const int hq = idx / D, d = idx % D;
            float M = s_new[hq];
            for (uint32_t r = 0; r < C; ++r) M = fmaxf(M, gather[(r * G + hq) * PART + D]);
            float acc = 0.f, Ls = 0.f;
            for (uint32_t r = 0; r < C; ++r) {
                const float *src = gather + (r * G + hq) * PART;
                const float f = (src[D] == -INFINITY) ? 0.f : tc::ex2(src[D] - M);
                acc = fmaf(src[d], f, acc);
                Ls = fmaf(src[D + 1], f, Ls);
            }
            const float fn = tc::ex2(s_new[hq] - M);
            acc = fmaf(v_new[d], fn, acc);
            Ls += fn;
            p.o[((int64_t)b * p.Hq + (int64_t)g * G + hq) * D + d] = __float2bfloat16_rn(acc / Ls);
        }
        // the new token into its slot: every CTA of this cluster has read
        // the ring (the cluster barrier), and no other cluster reads head g
        const int64_t row = ((int64_t)b * W + new_slot) * p.Hkv + g;
        for (int i = threadIdx.x; i < D; i += 32 * kWarps) {
            p.ring_k[row * D + i] = p.k_new[((int64_t)b * p.Hkv + g) * D + i];
            p.ring_v[row * D + i] = p.v_new[((int64_t)b * p.Hkv + g) * D + i];
        }
        if (g == 0 && threadIdx.x == 0) p.slot_pos[(int64_t)b * W + new_slot] = (int32_t)pos_b;
    }
}

// ------------------------------------------------------------------- host
namespace {

// 4-D bf16 map over the ring [B, W, Hkv, D] as {D, Hkv, W, B}, box {64, 1,
// 128, 1}: 128 slots of one KV head, 64 columns, 128-byte swizzle.  Slots
// past W read as zeros (and are masked).
bool make_ring_map(CUtensorMap *m, const void *ring, int64_t B, int64_t W, int64_t Hkv, int64_t D) {
    const uint64_t dims[4] = {(uint64_t)D, (uint64_t)Hkv, (uint64_t)W, (uint64_t)B};
    const uint64_t strides[3] = {(uint64_t)(D * 2), (uint64_t)(Hkv * D * 2), (uint64_t)(W * Hkv * D * 2)};
    const uint32_t box[4] = {64, 1, (uint32_t)kChunk, 1};
    return encode_bf16_map_4d(m, ring, dims, strides, box);
}

template <int D, int G>
cudaError_t launch_ring_dg(const DecodeArgs &a, cudaStream_t st, bool compact) {
    CUtensorMap mk, mv;
    if (!make_ring_map(&mk, a.k, a.B, a.window, a.Hkv, D) || !make_ring_map(&mv, a.v, a.B, a.window, a.Hkv, D))
        return cudaErrorNotSupported;
    RingParams p;
    p.q = static_cast<const __nv_bfloat16 *>(a.q);
    p.k_new = static_cast<const __nv_bfloat16 *>(a.k_new);
    p.v_new = static_cast<const __nv_bfloat16 *>(a.v_new);
    p.pos = a.pos;
    p.ring_k = static_cast<__nv_bfloat16 *>(const_cast<void *>(a.k));
    p.ring_v = static_cast<__nv_bfloat16 *>(const_cast<void *>(a.v));
    p.slot_pos = const_cast<int32_t *>(a.slot_pos);
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv; p.window = a.window;
    p.scale_log2 = a.scale * kLog2e;
    // C CTAs per (sequence, KV head): one 128-slot chunk each up to W = 1024,
    // then eight CTAs of several chunks.  The compact layout takes at most
    // four CTAs, each with two chunks in flight (one CTA an SM at W = 1024).
    const int cmax = compact ? kMaxCluster / 2 : kMaxCluster;
    const int C = (int)std::min<int64_t>(cmax, ((int64_t)a.window + kChunk - 1) / kChunk);
    const int64_t per = (((int64_t)a.window + C - 1) / C + kWarpTok - 1) / kWarpTok * kWarpTok;
    p.per = (int32_t)per;
    p.chunks = (int32_t)((per + kChunk - 1) / kChunk);
    p.stages = p.chunks > 1 ? 2 : 1;
    const int64_t grid = (int64_t)a.B * a.Hkv * C;
    if (grid > INT32_MAX) return cudaErrorNotSupported;
    const size_t smem = RingSmem<D, G>::bytes(p.stages);
    auto kern = ring_decode_cluster_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    note_launches(1);
    return cudaLaunchKernelEx(&cfg, kern, mk, mv, p);
}

template <int D>
cudaError_t launch_ring_d(const DecodeArgs &a, cudaStream_t st, bool compact) {
    switch (a.Hq / a.Hkv) {
        case 1: return launch_ring_dg<D, 1>(a, st, compact);
        case 2: return launch_ring_dg<D, 2>(a, st, compact);
        case 4: return launch_ring_dg<D, 4>(a, st, compact);
        case 8: return launch_ring_dg<D, 8>(a, st, compact);
        default: return cudaErrorNotSupported;
    }
}

}  // namespace

cudaError_t launch_ring_decode(const DecodeArgs &a, cudaStream_t st, bool compact) {
    if (a.dtype != kBF16 || !a.k_new || !a.pos || !a.slot_pos || a.window < 1) return cudaErrorNotSupported;
    if (a.D == 128) return launch_ring_d<128>(a, st, compact);
    if (a.D == 64) return launch_ring_d<64>(a, st, compact);
    return cudaErrorNotSupported;
}

unsigned int read_and_clear_status_ring() {
    unsigned int h = 0, z = 0;
    if (cudaMemcpyFromSymbol(&h, g_status_ring, sizeof(h)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_status_ring, &z, sizeof(z));
    return h;
}

}  // namespace yoco
