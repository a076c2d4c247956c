// Small pool operations: sentinel remapping of evicted slots, and the
// per-block statistics used to choose 8-bit blocks in a mixed cache.
//
// Remapping: IntentKV article (Qiita), "詰め直さずに「無効化」する" -- an
// evicted slot is pointed at a sentinel whose key is -1e4; nothing moves.
// Here the pointer is one bit per slot in a 256-bit mask per block.
//
// Mixed widths: QKVShare (arXiv 2605.03884 summary), "Méthodologie" -- bit
// widths per token from {2, 4, 8, FP16}.  This library chooses 8 bits per
// whole block for the blocks with the largest mean |K| and 4 bits elsewhere.
#include "async_copy.cuh"
#include "q4kv_internal.cuh"

namespace q4kv {
namespace {

__global__ void invalidate_kernel(PoolView pool, const int64_t* __restrict__ slot_ids, int64_t n) {
  const int64_t n_slots = static_cast<int64_t>(pool.n_blocks()) * kBlockTokens;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t s = slot_ids[i];
    if (s < 0 || s >= n_slots) {
      raise_error(pool.error_word, Q4KV_DEVERR_SLOT_ID);
      continue;
    }
    atomicOr(pool.mask + (s / kBlockTokens) * kMaskWords + (s % kBlockTokens) / 32,
             1u << (s % 32));
  }
}

// One CTA per 256-token chunk.  |x| of fp16/bf16 inputs converts exactly to
// double; sums stay exact while every partial sum is representable, so the
// result does not depend on the summation order for ordinary inputs.
template <typename T>
__global__ void __launch_bounds__(256) absmean_kernel(const T* __restrict__ k, int64_t n_tokens,
                                                      int64_t stride, int hkv, int d,
                                                      double* __restrict__ out) {
  const int64_t c = blockIdx.x;
  const int64_t t0 = c * kBlockTokens;
  const int64_t cnt = min(static_cast<int64_t>(kBlockTokens), n_tokens - t0);
  const int row = hkv * d;                  // elements per token
  const int vec_per_row = row / 8;          // 16-byte vectors per token
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < cnt * vec_per_row; i += blockDim.x) {
    const int64_t t = t0 + i / vec_per_row;
    const int e = static_cast<int>(i % vec_per_row) * 8;
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(k + t * stride + e));
    const T* x = reinterpret_cast<const T*>(&w);
#pragma unroll
    for (int q = 0; q < 8; ++q) acc += static_cast<double>(fabsf(to_float<T>(x[q])));
  }
  __shared__ double red[32];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    double a = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
    if (threadIdx.x == 0) out[c] = a / static_cast<double>(cnt * row);
  }
}

// Pass 1: flag[i] = 1 when chunk i ranks among the n_q8 largest (descending
// value, ties to the lower index), computed by counting the chunks that beat it.
__global__ void __launch_bounds__(256) mixed_rank_kernel(const double* __restrict__ a, int32_t n,
                                                         int32_t n_q8, int32_t* __restrict__ flag) {
  __shared__ double tile[1024];
  const int32_t i = blockIdx.x * blockDim.x + threadIdx.x;
  const double ai = i < n ? a[i] : 0.0;
  int32_t beats = 0;
  for (int32_t base = 0; base < n; base += 1024) {
    __syncthreads();
    for (int32_t q = threadIdx.x; q < 1024; q += blockDim.x)
      tile[q] = base + q < n ? a[base + q] : 0.0;
    __syncthreads();
    const int32_t lim = min(1024, n - base);
    for (int32_t q = 0; q < lim; ++q) {
      const double aj = tile[q];
      const int32_t jj = base + q;
      beats += (aj > ai) || (aj == ai && jj < i);
    }
  }
  if (i < n) flag[i] = beats < n_q8 ? 1 : 0;
}

// Pass 2 (one CTA): exclusive scan of the flags in chunk order -> ids.
__global__ void __launch_bounds__(1024) mixed_ids_kernel(int32_t n, int32_t q4_first,
                                                         int32_t q8_first, int32_t* __restrict__ ids) {
  __shared__ int32_t warp_sum[32];
  __shared__ int32_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  for (int32_t base = 0; base < n; base += 1024) {
    const int32_t i = base + threadIdx.x;
    const int32_t f = i < n ? ids[i] : 0;
    int32_t x = f;   // inclusive warp scan
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) warp_sum[wid] = x;
    __syncthreads();
    if (wid == 0) {
      int32_t s = warp_sum[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, s, off);
        if (lane >= off) s += y;
      }
      warp_sum[lane] = s;   // inclusive over warps
    }
    __syncthreads();
    const int32_t before = carry + (wid > 0 ? warp_sum[wid - 1] : 0) + x - f;  // exclusive
    if (i < n) ids[i] = f ? q8_first + before : q4_first + (i - before);
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_sum[31];
    __syncthreads();
  }
}

// One barrier that no thread ever arrives on: the bounded wait must give up.
__global__ void selftest_wait_kernel(uint32_t* error_word, unsigned tries) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (!mbar_wait(&bar, 0, tries)) raise_error(error_word, Q4KV_DEVERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_invalidate(const PoolView& pool, const int64_t* slot_ids, int64_t n,
                              cudaStream_t stream) {
  int64_t g = (n + 255) / 256;
  if (g > 4096) g = 4096;
  invalidate_kernel<<<static_cast<int>(g), 256, 0, stream>>>(pool, slot_ids, n);
  return cudaGetLastError();
}

cudaError_t launch_absmean(const void* k, int in_dtype, int64_t n_tokens, int64_t token_stride,
                           int n_kv_heads, int head_dim, double* out, cudaStream_t stream) {
  const int64_t chunks = (n_tokens + kBlockTokens - 1) / kBlockTokens;
  if (in_dtype == Q4KV_F16)
    absmean_kernel<__half><<<static_cast<unsigned>(chunks), 256, 0, stream>>>(
        static_cast<const __half*>(k), n_tokens, token_stride, n_kv_heads, head_dim, out);
  else
    absmean_kernel<__nv_bfloat16><<<static_cast<unsigned>(chunks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k), n_tokens, token_stride, n_kv_heads, head_dim, out);
  return cudaGetLastError();
}

cudaError_t launch_mixed_ids(const double* absmean, int32_t n, int32_t n_q8, int32_t q4_first,
                             int32_t q8_first, int32_t* ids, cudaStream_t stream) {
  mixed_rank_kernel<<<(n + 255) / 256, 256, 0, stream>>>(absmean, n, n_q8, ids);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  mixed_ids_kernel<<<1, 1024, 0, stream>>>(n, q4_first, q8_first, ids);
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(uint32_t* error_word, unsigned tries, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(error_word, tries);
  return cudaGetLastError();
}

}  // namespace q4kv
