// Cross-decoder decode step for callers that cannot allocate device memory.
//
// yoco_cross_decode needs a caller-provided workspace for its split-KV
// partials.  Some callers have no way to provide one: a plugin or C host that
// is handed only its input and output buffers and holds no allocator, or a
// process whose framework has already reserved nearly all device memory in
// its own pool, where an extra cudaMalloc fails or stalls the whole device.
// yoco_cross_decode_static serves them: its scratch is a fixed array compiled
// into this library, so a call allocates nothing.
//
// Facts a user needs:
//  * Capacity: kStaticScratchBytes (32 MiB) of device memory, reserved on
//    every GPU that loads the library and held until the process exits.  A
//    call whose split plan needs more returns YOCO_ERR_WORKSPACE and launches
//    nothing (yoco_cross_decode_workspace_size tells the need in advance).
//  * Set-up: the first call on a device looks up the array's device address
//    on that device (the device must be current, as for any launch on its
//    streams).  Make that first call before any stream capture.  The address
//    is kept for the life of the process: it does not survive a
//    cudaDeviceReset (or any other teardown of the device's primary context)
//    in the same process, after which this entry point must not be called.
//  * Sharing: every call on a device uses the same array and leaves its
//    contents behind.  Nothing in it needs to start at zero: each call writes
//    every partial it later reads.  Calls whose kernels overlap on the GPU
//    (two streams, or two host threads) race on the array; serialise them.
#include <mutex>

#include "../../include/yoco.h"
#include "launch.h"

namespace {

constexpr size_t kStaticScratchBytes = (size_t)32 << 20;
static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device.  In host code the array's name is only a stand-in for it.
cudaError_t scratch_on_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" yoco_status yoco_cross_decode_static(const void *q, const void *k_cache,
                                                const void *v_cache, int64_t cache_rows,
                                                const int64_t *seq_start, const int32_t *seq_len,
                                                int32_t B, int64_t max_len, void *o, float *lse,
                                                const yoco_attn_cfg *cfg, cudaStream_t stream) {
    // every argument check of yoco_cross_decode first: without a workspace it
    // launches nothing and answers YOCO_ERR_WORKSPACE only when all else is valid
    const yoco_status st = yoco_cross_decode(q, k_cache, v_cache, cache_rows, seq_start, seq_len, B,
                                             max_len, o, lse, nullptr, 0, cfg, stream);
    if (st != YOCO_ERR_WORKSPACE) return st;
    if (yoco_cross_decode_workspace_size(B, max_len, cfg) > kStaticScratchBytes) return YOCO_ERR_WORKSPACE;
    void *scratch = nullptr;
    if (scratch_on_current_device(&scratch) != cudaSuccess) return YOCO_ERR_CUDA;
    return yoco_cross_decode(q, k_cache, v_cache, cache_rows, seq_start, seq_len, B, max_len, o,
                             lse, scratch, kStaticScratchBytes, cfg, stream);
}
