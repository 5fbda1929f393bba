// tcgen05 / TMEM / TMA attention prefill (bf16) for sm_100a.
#include "common.cuh"
#include "launch.h"

namespace yoco {

static __device__ unsigned int g_status_prefill_tc;

cudaError_t launch_prefill_tc(const PrefillArgs &, cudaStream_t) { return cudaErrorNotSupported; }

unsigned int read_and_clear_status_prefill_tc() {
    unsigned int h = 0, z = 0;
    if (cudaMemcpyFromSymbol(&h, g_status_prefill_tc, sizeof(h)) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_status_prefill_tc, &z, sizeof(z));
    return h;
}

}  // namespace yoco
