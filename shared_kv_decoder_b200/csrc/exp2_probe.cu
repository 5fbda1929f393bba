// Test-only entry point: the prefill kernels' polynomial 2^x (tc.cuh,
// exp2_pair_poly) applied elementwise, so that tests can hold it against
// exp2 over its whole input range, -inf included.  It computes a quarter of
// the softmax exponentials in attn_prefill_pair_kernel / attn_prefill_tc_kernel.
#include "../../include/yoco.h"
#include "common.cuh"
#include "launch.h"
#include "tc.cuh"

namespace yoco {
namespace {

__global__ void exp2_poly_kernel(const float *x, float *y, int64_t n) {
    const int64_t i = 2 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float x0 = x[i];
    const float x1 = i + 1 < n ? x[i + 1] : 0.f;
    float e0, e1;
    tc::exp2_pair_poly(x0, x1, e0, e1);
    y[i] = e0;
    if (i + 1 < n) y[i + 1] = e1;
}

}  // namespace
}  // namespace yoco

extern "C" yoco_status yoco_debug_exp2_poly(const float *x, float *y, int64_t n, cudaStream_t stream) {
    if (n < 0) return YOCO_ERR_INVALID;
    if (n == 0) return YOCO_OK;
    if (!x || !y) return YOCO_ERR_INVALID;
    const int64_t pairs = (n + 1) / 2;
    const int64_t blocks = (pairs + 255) / 256;
    if (blocks > INT32_MAX) return YOCO_ERR_INVALID;
    yoco::note_launches(1);
    yoco::exp2_poly_kernel<<<(unsigned)blocks, 256, 0, stream>>>(x, y, n);
    return cudaGetLastError() == cudaSuccess ? YOCO_OK : YOCO_ERR_CUDA;
}
