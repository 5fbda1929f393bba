// Host-side launchers of the libyoco kernels (internal; the public ABI is
// include/yoco.h).  Every launcher assumes its arguments were validated by
// the API layer and returns the cudaError_t of its launches.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

struct CUtensorMap_st;  // cuda.h's TMA descriptor (CUtensorMap)

namespace yoco {

enum Dtype { kBF16 = 0, kFP32 = 1 };

inline size_t dtype_bytes(int dt) { return dt == kBF16 ? 2 : 4; }

// ------------------------------------------------------------ decode plan
// One decode "unit" is a contiguous token range of one sequence, streamed
// through shared memory by one CTA for every KV head.  Its partial softmax
// state (m, l, o) per query head and per consumer-warp subset goes to the
// workspace; a merge kernel combines them.
struct DecodePlan {
    int64_t stage_tokens;  // tokens per pipeline stage (128 / Hkv)
    int64_t split;         // tokens per unit (multiple of stage_tokens)
    int64_t n_split;       // units per sequence at max_len
    int sub;               // partial entries per unit per head (8 / Hkv)
    int stages;            // pipeline depth
    size_t smem_bytes;     // dynamic shared memory per CTA
    size_t ws_bytes;       // workspace bytes
};
bool make_decode_plan(int32_t B, int64_t max_len, int Hq, int Hkv, int D, int dtype,
                      DecodePlan *plan);

struct DecodeArgs {
    const void *q;        // [B, Hq, D]
    const void *k;        // cache [rows, Hkv, D]
    const void *v;
    const int64_t *seq_start;  // [B] (cross) or NULL (ring: b * window)
    const int32_t *seq_len;    // [B] (cross) or NULL (ring: window slots)
    const int32_t *slot_pos;   // ring only: [B, window]
    const int64_t *pos;        // ring only: [B]
    const void *k_new, *v_new; // ring only: the new token's K / V [B, Hkv, D], merged and written by the merge
    int32_t window;            // ring only
    int64_t cache_rows;        // rows of the K and V cache buffers (ring: B * window)
    int64_t max_len;           // longest allowed sequence (the plan's max_len; ring: window)
    int32_t B, Hq, Hkv, D, dtype;
    float scale;
    void *o;       // [B, Hq, D]
    float *lse;    // [B, Hq] or NULL
    void *ws;      // workspace
};
cudaError_t launch_decode(const DecodeArgs &a, const DecodePlan &plan, cudaStream_t s);
// Sliding-window decode step in one clustered launch (bf16, D 64 / 128, group
// size 1, 2, 4 or 8); cudaErrorNotSupported for any other shape.  compact: at
// most four CTAs per (sequence, KV head) instead of eight, each with two
// window chunks in flight (faster after launch_linear_few_reg).
cudaError_t launch_ring_decode(const DecodeArgs &a, cudaStream_t s, bool compact = false);

// Ring fill after a prefill of T tokens.
cudaError_t launch_ring_fill(const void *k, const void *v, int32_t B, int64_t T, int32_t window,
                             int Hkv, int D, int dtype, void *ring_k, void *ring_v,
                             int32_t *slot_pos, cudaStream_t s);

// ------------------------------------------------------------- prefill
struct PrefillArgs {
    const void *q;   // [B, Tq, Hq, D]
    const void *k;   // [B, Tkv, Hkv, D]
    const void *v;
    void *o;         // [B, Tq, Hq, D]
    float *lse;      // [B, Hq, Tq] or NULL
    int32_t B;
    int64_t Tq, Tkv, q_pos0;
    int32_t window;  // 0: causal only
    int32_t Hq, Hkv, D, dtype;
    float scale;
};
// CUDA-core path (any dtype; the fp32 path).
cudaError_t launch_prefill_simt(const PrefillArgs &a, cudaStream_t s);
// Tensor-core path (bf16): tcgen05 + TMEM + TMA.  Returns cudaErrorNotSupported
// when the shape is outside what it was built for.
cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t s);
// Tensor-core path for bf16 and an even group size: two query heads of one
// KV group per CTA.  cudaErrorNotSupported for other shapes.
cudaError_t launch_prefill_pair(const PrefillArgs &a, cudaStream_t s);

// ------------------------------------------------------------ projection
struct LinearArgs {
    const void *x;      // [n, d_in]
    const void *w;      // [d_out, d_in]
    int64_t n;
    int32_t d_in, d_out;
    int32_t apply_ln;
    float eps;
    int32_t split_col;  // columns < split_col -> out0/base0, the rest -> out1/base1
    void *out0, *out1;
    const void *base0, *base1;
    float w0, w1;
    const int64_t *dst_rows;  // optional row remap of the outputs
    int32_t dtype;
};
cudaError_t launch_linear_simt(const LinearArgs &a, cudaStream_t s);
// Few-token projection with the weight rows streamed through registers (bf16,
// 1 <= n <= 4, d_in a multiple of 256, d_out a multiple of 16).
// cudaErrorNotSupported otherwise.
cudaError_t launch_linear_few_reg(const LinearArgs &a, cudaStream_t s);
// Tensor-core path (bf16, >= 512 tokens, output width a multiple of 256):
// LayerNorm folded into the epilogue.  cudaErrorNotSupported otherwise.
cudaError_t launch_linear_tc(const LinearArgs &a, cudaStream_t s);

// ------------------------------------------------------- gated retention
struct GretArgs {
    const void *q, *k, *v;  // prefill [B, T, H, D], decode [B, H, D]
    const float *g;         // gate logits: prefill [B, T, H], decode [B, H]
    float *state;           // [B, H, D, D] fp32: prefill in/out or null, decode in/out
    void *o;                // like q
    int32_t B, H, D, dtype;
    int64_t T;              // prefill only
    float tau, scale;
    void *ws;               // prefill: scratch for the split over superchunks, or NULL (no split)
};
// Chunkwise prefill (bf16; cudaErrorNotSupported for other dtypes).
cudaError_t launch_gret_prefill(const GretArgs &a, cudaStream_t s);
// One recurrent decode step (bf16 or fp32).
cudaError_t launch_gret_decode(const GretArgs &a, cudaStream_t s);
// Chunkwise prefill on the tensor cores (bf16, D = 128; cudaErrorNotSupported otherwise).
cudaError_t launch_gret_prefill_tc(const GretArgs &a, cudaStream_t s);
// Superchunks per sequence of that kernel for B x H sequences of T tokens on
// `sms` SMs, and the scratch bytes a split needs (0: the kernel never splits).
int gret_superchunks(int32_t B, int32_t H, int64_t T, int sms);
size_t gret_workspace_bytes(int32_t B, int32_t H, int64_t T, int D);

// Test-only: a kernel whose bounded wait is never satisfied (see decode.cu).
cudaError_t launch_wait_timeout_probe(cudaStream_t s);

// Device status words of the translation units that hold bounded waits:
// bit 0 = a bounded wait gave up; bit 1 (decode only) = a decode sequence's
// seq_start / seq_len were out of range.
unsigned int read_and_clear_status_decode();
unsigned int read_and_clear_status_prefill_tc();
unsigned int read_and_clear_status_prefill_pair();
unsigned int read_and_clear_status_gret_tc();
unsigned int read_and_clear_status_project_tc();
unsigned int read_and_clear_status_linear();
unsigned int read_and_clear_status_ring();
unsigned int read_and_clear_status_step_proj();

int device_sm_count();

// A 4-D bf16 tensor map (innermost dimension first, strides of dimensions 1-3
// in bytes) with the 128-byte swizzle; false when the driver rejects it.
bool encode_bf16_map_4d(::CUtensorMap_st *m, const void *ptr, const uint64_t dims[4],
                        const uint64_t strides_bytes[3], const uint32_t box[4]);
// The same for bf16 or byte elements, with or without the 128-byte swizzle.
bool encode_map_4d(::CUtensorMap_st *m, const void *ptr, bool bytes, bool swizzle128, const uint64_t dims[4],
                   const uint64_t strides_bytes[3], const uint32_t box[4]);

// ------------------------------------------------------------- 8-bit cache
// One row of an 8-bit K or V cache: Hkv x D int8 codes, then the Hkv fp32
// scales, padded to a multiple of 16 bytes.
inline int64_t i8_scale_bytes(int Hkv) { return 16 * ((Hkv * 4 + 15) / 16); }
inline int64_t i8_row_bytes(int Hkv, int D) { return (int64_t)Hkv * D + i8_scale_bytes(Hkv); }
// Quantise n rows of K and V ([n, Hkv, D], bf16 or fp32) into 8-bit rows,
// row dst_rows[i] (or i) of kq / vq.
cudaError_t launch_kv_quantize_i8(const void *k, const void *v, int64_t n, int Hkv, int D, int dtype,
                                  const int64_t *dst_rows, void *kq, void *vq, cudaStream_t s);
// Split-KV decode over 8-bit caches (D = 128); a.k / a.v point at the 8-bit rows.
cudaError_t launch_decode_i8(const DecodeArgs &a, const DecodePlan &pl, cudaStream_t s);

// Host-side count of kernel launches (reported by yoco_launch_count()).
void note_launches(int n);

// Launch with programmatic stream serialization (see pdl_wait in common.cuh):
// the kernel may start before the previous kernel on the stream has finished,
// and must call pdl_wait() before reading anything.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace yoco
