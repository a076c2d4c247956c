// Internal declarations shared by the CUDA translation units of libq4kv.
// Nothing here is part of the C ABI (include/q4kv.h is).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "q4kv.h"

namespace q4kv {

constexpr int kBlockTokens = Q4KV_BLOCK_TOKENS;
constexpr int kGroup = Q4KV_GROUP;
constexpr int kMaskWords = Q4KV_MASK_WORDS;

// Everything a kernel needs about the pool, passed by value.
struct PoolView {
  int32_t head_dim;
  int32_t n_kv_heads;
  int32_t k_rotated;
  int32_t n_q4;
  int32_t n_q8;
  int32_t fp8;        // Q4KV_FORMAT_FP8: every block holds OCP E4M3 bytes, no params
  uint8_t* k_codes4;
  uint8_t* v_codes4;
  __half2* k_params4;
  __half2* v_params4;
  uint8_t* k_codes8;
  uint8_t* v_codes8;
  __half2* k_params8;
  __half2* v_params8;
  uint32_t* mask;
  uint32_t* error_word;
  int32_t n_q2;       // 2-bit blocks: unified ids [n_q4 + n_q8, n_q4 + n_q8 + n_q2)
  uint8_t* k_codes2;
  uint8_t* v_codes2;
  __half2* k_params2;
  __half2* v_params2;
  __host__ __device__ __forceinline__ int n_blocks() const { return n_q4 + n_q8 + n_q2; }
  // code bits of a valid unified block id
  __host__ __device__ __forceinline__ int bits_of(int blk) const {
    return blk < n_q4 ? 4 : (blk < n_q4 + n_q8 ? 8 : 2);
  }
};

inline PoolView view_of(const q4kv_pool& p) {
  PoolView v;
  v.head_dim = p.head_dim;
  v.n_kv_heads = p.n_kv_heads;
  v.k_rotated = p.k_rotated;
  v.n_q4 = p.n_q4_blocks;
  v.n_q8 = p.n_q8_blocks;
  v.fp8 = p.value_format == Q4KV_FORMAT_FP8;
  v.k_codes4 = p.k_codes4;
  v.v_codes4 = p.v_codes4;
  v.k_params4 = reinterpret_cast<__half2*>(p.k_params4);
  v.v_params4 = reinterpret_cast<__half2*>(p.v_params4);
  v.k_codes8 = p.k_codes8;
  v.v_codes8 = p.v_codes8;
  v.k_params8 = reinterpret_cast<__half2*>(p.k_params8);
  v.v_params8 = reinterpret_cast<__half2*>(p.v_params8);
  v.mask = p.remap_mask;
  v.error_word = p.error_word;
  v.n_q2 = p.n_q2_blocks;
  v.k_codes2 = p.k_codes2;
  v.v_codes2 = p.v_codes2;
  v.k_params2 = reinterpret_cast<__half2*>(p.k_params2);
  v.v_params2 = reinterpret_cast<__half2*>(p.v_params2);
  return v;
}

__device__ __forceinline__ void raise_error(uint32_t* word, uint32_t bit) {
  if (word != nullptr) atomicOr(word, bit);
}

// binary32 nearest to 1/sqrt(D) for the supported head sizes.
__host__ __device__ __forceinline__ float rotation_constant(int d) {
  return d == 256 ? 0.0625f : 0x1.6a09e6p-4f;   // 2^-4 and RN(2^-3.5)
}

// Load one element of an fp16/bf16 input as binary32 (exact).
template <typename T>
__device__ __forceinline__ float to_float(T x);
template <>
__device__ __forceinline__ float to_float<__half>(__half x) { return __half2float(x); }
template <>
__device__ __forceinline__ float to_float<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  The hot kernels (encoder, tensor-core
// decode, split merge) are launched so that they may start while the kernel
// before them in the stream drains, and each lets its own successor start
// early.  Such a kernel executes griddep_wait() before it touches any global
// memory: that returns once every earlier grid has completed and its writes
// are visible, so the stream order of results is unchanged.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------------------
// launchers (each returns cudaGetLastError() of its launch)
// ---------------------------------------------------------------------------
cudaError_t launch_quantize(const PoolView& pool, const void* k, const void* v, int in_dtype,
                            int64_t n_tokens, int64_t token_stride, const int32_t* block_ids,
                            cudaStream_t stream);
cudaError_t launch_append(const PoolView& pool, const void* k, const void* v, int in_dtype,
                          int32_t batch, int32_t max_new, const int32_t* n_new, int64_t seq_stride,
                          int64_t token_stride, const int32_t* tables, int32_t max_blocks,
                          const int32_t* seq_lens, cudaStream_t stream);
cudaError_t launch_selftest_wait(uint32_t* error_word, unsigned tries, cudaStream_t stream);
// Per-token mixed-width cards (quantize.cu).
int64_t card_max_bytes(int d, int hkv, int64_t n);
cudaError_t launch_card_encode(int d, int hkv, int k_rotated, const void* k, const void* v, int in_dtype,
                               int64_t n, int64_t stride, const uint8_t* widths, uint8_t* card,
                               uint32_t* error_word, cudaStream_t stream);
cudaError_t launch_card_decode(int d, int hkv, const uint8_t* card, int64_t card_bytes, int64_t n, void* k_out,
                               void* v_out, int out_dtype, uint32_t* error_word, cudaStream_t stream);
// Block images (paging.cu): stride of one image for this pool, and one
// launch moving n blocks' images between the pool and host memory.
int64_t image_stride_bytes(const PoolView& pool);
cudaError_t launch_page(const PoolView& pool, const int32_t* ids, int32_t n, void* host, bool to_host,
                        cudaStream_t stream);
// Copy-engine paging with host block ids (paging.cu): headers, then copies.
bool host_headers(const PoolView& pool, const int32_t* ids, int32_t n, uint8_t* host, bool write);
cudaError_t copy_pages(const PoolView& pool, const int32_t* ids, int32_t n, uint8_t* host, bool to_host,
                       cudaStream_t stream);
cudaError_t launch_dequantize(const PoolView& pool, const int32_t* block_ids, int32_t n_blocks,
                              void* k_out, void* v_out, int out_dtype, int unrotate_k,
                              cudaStream_t stream);
cudaError_t launch_invalidate(const PoolView& pool, const int64_t* slot_ids, int64_t n,
                              cudaStream_t stream);
cudaError_t launch_absmean(const void* k, int in_dtype, int64_t n_tokens, int64_t token_stride,
                           int n_kv_heads, int head_dim, double* out, cudaStream_t stream);
cudaError_t launch_mixed_ids(const double* absmean, int32_t n, int32_t n_q8, int32_t q4_first,
                             int32_t q8_first, int32_t* ids, cudaStream_t stream);

struct DecodeArgs {
  PoolView pool;
  q4kv_decode_plan plan;
  const void* q;
  int q_dtype;
  const int32_t* tables;
  const int32_t* seq_lens;
  // Sequence b is seq_lens[b] + (add_lens ? add_lens[b] : add_const) tokens
  // long (an append just before the decode adds the second term).
  const int32_t* add_lens;
  int add_const;
  // 1: the kernel before this one in the stream is an append whose writes
  // all land at positions >= seq_lens[b]; the tensor-core kernel then waits
  // for it only before it reads those blocks (programmatic dependent launch).
  int defer_wait;
  // Fused append (tensor-core kernel, pools of 4-, 8- and 2-bit blocks): when
  // app_k is set, the kernel itself encodes new row i < (add_lens ? add_lens[b]
  // : add_const) of sequence b -- element (b, i, h, c) at b * app_seq_stride +
  // i * app_token_stride + h * D + c of app_k and app_v, 16-bit app_dtype --
  // into the pool at position seq_lens[b] + i before it reads that block.
  const void* app_k;
  const void* app_v;
  int app_dtype;
  int64_t app_seq_stride, app_token_stride;
  float scale;
  void* out;
  int out_dtype;
  float* ws_o;   // [B][Hq][S][D]
  float* ws_ml;  // [B][Hq][S][2] (running max, running sum)
};
__device__ __forceinline__ int seq_len_of(const DecodeArgs& a, int b) {
  return a.seq_lens[b] + (a.add_lens != nullptr ? a.add_lens[b] : a.add_const);
}
// plan.kernel selects the decode kernel: 1 = tensor-core pipeline
// (decode_tc.cu), 0 = CUDA-core kernel (decode.cu); both share the merge.
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_tc(const DecodeArgs& a, int num_sms, cudaStream_t stream);
cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t stream);
int device_sm_count();

}  // namespace q4kv
