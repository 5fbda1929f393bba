// Device-side helpers shared by the sm_100a kernels of libyoco: element
// conversion, mbarrier and bulk-copy wrappers (inline PTX), and bounded
// waits that report a timeout through a per-translation-unit status word
// instead of spinning forever.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define YOCO_DEV __device__ __forceinline__

namespace yoco {

// ----------------------------------------------------------------- dtypes
YOCO_DEV float to_f32(float x) { return x; }
YOCO_DEV float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> YOCO_DEV T from_f32(float x);
template <> YOCO_DEV float from_f32<float>(float x) { return x; }
template <> YOCO_DEV __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Unpack one 16-byte chunk into fp32 values (8 for bf16, 4 for fp32).
template <typename T> struct Chunk;
template <> struct Chunk<__nv_bfloat16> {
    static constexpr int N = 8;
    YOCO_DEV static void unpack(const uint4 &c, float *f) {
        const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};
template <> struct Chunk<float> {
    static constexpr int N = 4;
    YOCO_DEV static void unpack(const uint4 &c, float *f) {
        f[0] = __uint_as_float(c.x);
        f[1] = __uint_as_float(c.y);
        f[2] = __uint_as_float(c.z);
        f[3] = __uint_as_float(c.w);
    }
};

// ------------------------------------------------------------- addresses
YOCO_DEV uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// -------------------------------------------------------------- mbarrier
YOCO_DEV void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
YOCO_DEV void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
YOCO_DEV void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
YOCO_DEV void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
YOCO_DEV void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
YOCO_DEV bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// A wait gives up after this many SM clock cycles (about 0.1 s at the B200's
// clocks): far above any legitimate wait (microseconds), short enough that a
// lost arrive becomes an error status rather than a hung GPU.
constexpr long long kWaitLimitCycles = 200000000LL;

// Bounded wait on an mbarrier phase.  Returns false (and sets *status) when
// the limit passes without the phase completing.
YOCO_DEV bool mbar_wait(uint64_t *bar, uint32_t parity, unsigned int *status) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0 && clock64() - t0 > kWaitLimitCycles) {
            atomicOr(status, 1u);
            return false;
        }
    }
}

// --------------------------------------------------------------- bulk copy
// One contiguous global -> shared copy completed on an mbarrier (bytes and
// both addresses multiples of 16).
YOCO_DEV void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Ask L2 for a contiguous range (address and size multiples of 16 bytes); a
// prefetch only warms the cache, so it may precede pdl_wait().
YOCO_DEV void bulk_prefetch_l2(const void *src_gmem, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src_gmem), "r"(bytes) : "memory");
}

// ------------------------------------------- programmatic dependent launch
// The decode-step kernels (small projections, ring write, split decode,
// merge) are launched with programmatic stream serialization (launch_pdl): the
// next kernel on the stream is launched while this one runs and its CTAs wait
// in pdl_wait() -- which returns once every earlier kernel on the stream has
// finished and its writes are visible -- so the launch gap between the short
// kernels of a decode step disappears.  Every such kernel calls pdl_wait()
// before it reads any input (and before any early exit), which also keeps the
// ordering transitive along the stream.  Without the launch attribute both
// are no-ops.
YOCO_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
YOCO_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------ warp helpers
YOCO_DEV float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
YOCO_DEV float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace yoco
