// Host side of the C ABI declared in include/q4kv.h: argument checks, launch
// plans and dispatch to the kernels.  Every check happens before any CUDA
// call, so a rejected call touches no device.
#include <math.h>
#include <string.h>

#include "q4kv_internal.cuh"

using namespace q4kv;

namespace {

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

q4kv_status check_pool(const q4kv_pool* p) {
  if (p == nullptr) return Q4KV_ERR_INVALID_ARG;
  if ((p->value_format != Q4KV_FORMAT_INT && p->value_format != Q4KV_FORMAT_FP8) || p->n_kv_heads < 1 ||
      p->n_q4_blocks < 0 || p->n_q8_blocks < 0 || p->n_q2_blocks < 0 || p->reserved != 0 ||
      (p->k_rotated != 0 && p->k_rotated != 1))
    return Q4KV_ERR_INVALID_ARG;
  const bool fp8 = p->value_format == Q4KV_FORMAT_FP8;
  if (fp8 && (p->n_q4_blocks != 0 || p->n_q2_blocks != 0 || p->k_rotated != 0)) return Q4KV_ERR_INVALID_ARG;
  if (p->head_dim != 128 && p->head_dim != 256) return Q4KV_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(p->n_q4_blocks) + p->n_q8_blocks + p->n_q2_blocks > (int64_t{1} << 31) / kBlockTokens)
    return Q4KV_ERR_INVALID_ARG;
  if (p->n_q4_blocks > 0) {
    const void* a[4] = {p->k_codes4, p->v_codes4, p->k_params4, p->v_params4};
    for (const void* x : a)
      if (x == nullptr || !aligned(x, 16)) return Q4KV_ERR_INVALID_ARG;
  }
  if (p->n_q8_blocks > 0) {
    const void* a[4] = {p->k_codes8, p->v_codes8, p->k_params8, p->v_params8};
    for (int i = 0; i < (fp8 ? 2 : 4); ++i)   // an FP8 pool has no params
      if (a[i] == nullptr || !aligned(a[i], 16)) return Q4KV_ERR_INVALID_ARG;
  }
  if (p->n_q2_blocks > 0) {
    const void* a[4] = {p->k_codes2, p->v_codes2, p->k_params2, p->v_params2};
    for (const void* x : a)
      if (x == nullptr || !aligned(x, 16)) return Q4KV_ERR_INVALID_ARG;
  }
  if (p->n_q4_blocks + p->n_q8_blocks + p->n_q2_blocks > 0 &&
      (p->remap_mask == nullptr || !aligned(p->remap_mask, 16)))
    return Q4KV_ERR_INVALID_ARG;
  if (p->error_word != nullptr && !aligned(p->error_word, 4)) return Q4KV_ERR_INVALID_ARG;
  return Q4KV_OK;
}

q4kv_status check_input(const void* x, int32_t dtype, int64_t n_tokens, int64_t stride,
                        int32_t hkv, int32_t d) {
  if (dtype != Q4KV_F16 && dtype != Q4KV_BF16) return Q4KV_ERR_INVALID_ARG;
  if (n_tokens < 0 || stride < static_cast<int64_t>(hkv) * d) return Q4KV_ERR_INVALID_ARG;
  if ((stride * 2) % 16 != 0) return Q4KV_ERR_INVALID_ARG;
  if (n_tokens > 0 && (x == nullptr || !aligned(x, 16))) return Q4KV_ERR_INVALID_ARG;
  return Q4KV_OK;
}

// Host argument checks shared by export and import; *dev receives the
// device's address of the host buffer.
q4kv_status check_paging(const q4kv_pool* pool, const int32_t* ids, int32_t n, const void* host, void** dev) {
  q4kv_status st = check_pool(pool);
  if (st != Q4KV_OK) return st;
  if (n < 0) return Q4KV_ERR_INVALID_ARG;
  if (n == 0) return Q4KV_OK;
  if (ids == nullptr || !aligned(ids, 4) || host == nullptr || !aligned(host, 16)) return Q4KV_ERR_INVALID_ARG;
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, host) != cudaSuccess) {
    cudaGetLastError();
    return Q4KV_ERR_INVALID_ARG;
  }
  if (attr.type != cudaMemoryTypeHost || attr.devicePointer == nullptr) return Q4KV_ERR_INVALID_ARG;
  *dev = attr.devicePointer;
  return Q4KV_OK;
}

q4kv_status from_cuda(cudaError_t e) { return e == cudaSuccess ? Q4KV_OK : Q4KV_ERR_CUDA; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

extern "C" {

const char* q4kv_status_string(q4kv_status s) {
  switch (s) {
    case Q4KV_OK: return "ok";
    case Q4KV_ERR_INVALID_ARG: return "invalid argument";
    case Q4KV_ERR_UNSUPPORTED: return "unsupported shape";
    case Q4KV_ERR_CUDA: return "CUDA error";
    case Q4KV_ERR_WORKSPACE: return "workspace missing or too small";
    case Q4KV_ERR_DEVICE: return "device reported an error";
  }
  return "unknown status";
}

int32_t q4kv_abi_version(void) { return Q4KV_ABI_VERSION; }

q4kv_status q4kv_pool_array_bytes(int32_t head_dim, int32_t n_kv_heads, int64_t n_blocks,
                                  int32_t bits, size_t* codes_bytes, size_t* params_bytes) {
  if (codes_bytes == nullptr || params_bytes == nullptr || n_kv_heads < 1 || n_blocks < 0 ||
      (bits != 2 && bits != 4 && bits != 8))
    return Q4KV_ERR_INVALID_ARG;
  if (head_dim != 128 && head_dim != 256) return Q4KV_ERR_UNSUPPORTED;
  const size_t rows = static_cast<size_t>(n_blocks) * n_kv_heads * kBlockTokens;
  *codes_bytes = rows * head_dim * bits / 8;
  *params_bytes = rows * (head_dim / kGroup) * 4;
  return Q4KV_OK;
}

q4kv_status q4kv_quantize_blocks(const q4kv_pool* pool, const void* k, const void* v,
                                 int32_t in_dtype, int64_t n_tokens, int64_t token_stride,
                                 const int32_t* block_ids, void* stream) {
  q4kv_status st = check_pool(pool);
  if (st != Q4KV_OK) return st;
  st = check_input(k, in_dtype, n_tokens, token_stride, pool->n_kv_heads, pool->head_dim);
  if (st != Q4KV_OK) return st;
  st = check_input(v, in_dtype, n_tokens, token_stride, pool->n_kv_heads, pool->head_dim);
  if (st != Q4KV_OK) return st;
  if (n_tokens == 0) return Q4KV_OK;
  if (block_ids == nullptr || !aligned(block_ids, 4)) return Q4KV_ERR_INVALID_ARG;
  return from_cuda(launch_quantize(view_of(*pool), k, v, in_dtype, n_tokens, token_stride,
                                   block_ids, as_stream(stream)));
}

// Arguments of an append; *rows = 0 when it writes nothing.
static q4kv_status check_append(const q4kv_pool* pool, const void* k, const void* v, int32_t in_dtype,
                                int32_t batch, int32_t max_new, const int32_t* n_new, int64_t seq_stride,
                                int64_t token_stride, const int32_t* tables, int32_t max_blocks,
                                const int32_t* seq_lens, int64_t* rows) {
  q4kv_status st = check_pool(pool);
  if (st != Q4KV_OK) return st;
  if (batch < 0 || max_new < 0 || seq_stride < 0) return Q4KV_ERR_INVALID_ARG;
  *rows = batch > 0 && max_new > 0 ? 1 : 0;
  st = check_input(k, in_dtype, *rows, token_stride, pool->n_kv_heads, pool->head_dim);
  if (st != Q4KV_OK) return st;
  st = check_input(v, in_dtype, *rows, token_stride, pool->n_kv_heads, pool->head_dim);
  if (st != Q4KV_OK) return st;
  if ((seq_stride * 2) % 16 != 0) return Q4KV_ERR_INVALID_ARG;
  if (*rows == 0) return Q4KV_OK;
  if (tables == nullptr || !aligned(tables, 4) || max_blocks < 1 || seq_lens == nullptr ||
      !aligned(seq_lens, 4) || (n_new != nullptr && !aligned(n_new, 4)))
    return Q4KV_ERR_INVALID_ARG;
  return Q4KV_OK;
}

q4kv_status q4kv_append_tokens(const q4kv_pool* pool, const void* k, const void* v,
                               int32_t in_dtype, int32_t batch, int32_t max_new,
                               const int32_t* n_new, int64_t seq_stride, int64_t token_stride,
                               const int32_t* tables, int32_t max_blocks, const int32_t* seq_lens,
                               void* stream) {
  int64_t rows = 0;
  const q4kv_status st = check_append(pool, k, v, in_dtype, batch, max_new, n_new, seq_stride, token_stride,
                                      tables, max_blocks, seq_lens, &rows);
  if (st != Q4KV_OK || rows == 0) return st;
  return from_cuda(launch_append(view_of(*pool), k, v, in_dtype, batch, max_new, n_new, seq_stride,
                                 token_stride, tables, max_blocks, seq_lens, as_stream(stream)));
}

q4kv_status q4kv_block_image_stride(const q4kv_pool* pool, size_t* stride_bytes) {
  q4kv_status st = check_pool(pool);
  if (st != Q4KV_OK) return st;
  if (stride_bytes == nullptr) return Q4KV_ERR_INVALID_ARG;
  *stride_bytes = static_cast<size_t>(image_stride_bytes(view_of(*pool)));
  return Q4KV_OK;
}


q4kv_status q4kv_export_blocks(const q4kv_pool* pool, const int32_t* block_ids, int32_t n_blocks,
                               void* host_images, void* stream) {
  void* dev = nullptr;
  q4kv_status st = check_paging(pool, block_ids, n_blocks, host_images, &dev);
  if (st != Q4KV_OK || n_blocks == 0) return st;
  return from_cuda(launch_page(view_of(*pool), block_ids, n_blocks, dev, true, as_stream(stream)));
}

q4kv_status q4kv_import_blocks(const q4kv_pool* pool, const void* host_images, const int32_t* block_ids,
                               int32_t n_blocks, void* stream) {
  void* dev = nullptr;
  q4kv_status st = check_paging(pool, block_ids, n_blocks, host_images, &dev);
  if (st != Q4KV_OK || n_blocks == 0) return st;
  return from_cuda(launch_page(view_of(*pool), block_ids, n_blocks, dev, false, as_stream(stream)));
}

q4kv_status q4kv_export_blocks_host_ids(const q4kv_pool* pool, const int32_t* block_ids, int32_t n_blocks,
                                        void* host_images, void* stream) {
  void* dev = nullptr;
  q4kv_status st = check_paging(pool, block_ids, n_blocks, host_images, &dev);
  if (st != Q4KV_OK || n_blocks == 0) return st;
  const PoolView v = view_of(*pool);
  for (int32_t i = 0; i < n_blocks; ++i)
    if (block_ids[i] < 0 || block_ids[i] >= v.n_blocks()) return Q4KV_ERR_INVALID_ARG;
  host_headers(v, block_ids, n_blocks, static_cast<uint8_t*>(host_images), true);
  return from_cuda(copy_pages(v, block_ids, n_blocks, static_cast<uint8_t*>(host_images), true, as_stream(stream)));
}

q4kv_status q4kv_import_blocks_host_ids(const q4kv_pool* pool, const void* host_images, const int32_t* block_ids,
                                        int32_t n_blocks, void* stream) {
  void* dev = nullptr;
  q4kv_status st = check_paging(pool, block_ids, n_blocks, host_images, &dev);
  if (st != Q4KV_OK || n_blocks == 0) return st;
  const PoolView v = view_of(*pool);
  for (int32_t i = 0; i < n_blocks; ++i)
    if (block_ids[i] < 0 || block_ids[i] >= v.n_blocks()) return Q4KV_ERR_INVALID_ARG;
  uint8_t* img = static_cast<uint8_t*>(const_cast<void*>(host_images));
  if (!host_headers(v, block_ids, n_blocks, img, false)) return Q4KV_ERR_INVALID_ARG;
  return from_cuda(copy_pages(v, block_ids, n_blocks, img, false, as_stream(stream)));
}

q4kv_status q4kv_card_max_bytes(int32_t head_dim, int32_t n_kv_heads, int64_t n_tokens, size_t* bytes) {
  if (bytes == nullptr || n_kv_heads < 1 || n_tokens < 0 || n_tokens > (int64_t{1} << 31))
    return Q4KV_ERR_INVALID_ARG;
  if (head_dim != 128 && head_dim != 256) return Q4KV_ERR_UNSUPPORTED;
  *bytes = static_cast<size_t>(card_max_bytes(head_dim, n_kv_heads, n_tokens));
  return Q4KV_OK;
}

q4kv_status q4kv_card_encode(int32_t head_dim, int32_t n_kv_heads, int32_t k_rotated, const void* k,
                             const void* v, int32_t in_dtype, int64_t n_tokens, int64_t token_stride,
                             const uint8_t* widths, void* card, size_t card_bytes, uint32_t* error_word,
                             void* stream) {
  size_t need = 0;
  q4kv_status st = q4kv_card_max_bytes(head_dim, n_kv_heads, n_tokens, &need);
  if (st != Q4KV_OK) return st;
  if (k_rotated != 0 && k_rotated != 1) return Q4KV_ERR_INVALID_ARG;
  st = check_input(k, in_dtype, n_tokens, token_stride, n_kv_heads, head_dim);
  if (st != Q4KV_OK) return st;
  st = check_input(v, in_dtype, n_tokens, token_stride, n_kv_heads, head_dim);
  if (st != Q4KV_OK) return st;
  if ((n_tokens > 0 && widths == nullptr) || card == nullptr || !aligned(card, 16) || card_bytes < need ||
      (error_word != nullptr && !aligned(error_word, 4)))
    return Q4KV_ERR_INVALID_ARG;
  return from_cuda(launch_card_encode(head_dim, n_kv_heads, k_rotated, k, v, in_dtype, n_tokens, token_stride,
                                      widths, static_cast<uint8_t*>(card), error_word, as_stream(stream)));
}

q4kv_status q4kv_card_decode(const void* card, size_t card_bytes, int32_t head_dim, int32_t n_kv_heads,
                             int64_t n_tokens, void* k_out, void* v_out, int32_t out_dtype, uint32_t* error_word,
                             void* stream) {
  size_t least = 0;
  q4kv_status st = q4kv_card_max_bytes(head_dim, n_kv_heads, 0, &least);
  if (st != Q4KV_OK) return st;
  if (n_tokens < 0 || n_tokens > (int64_t{1} << 31)) return Q4KV_ERR_INVALID_ARG;
  if (out_dtype != Q4KV_F32 && out_dtype != Q4KV_F16) return Q4KV_ERR_INVALID_ARG;
  if (error_word != nullptr && !aligned(error_word, 4)) return Q4KV_ERR_INVALID_ARG;
  if (n_tokens == 0) return Q4KV_OK;
  const size_t tables = static_cast<size_t>((n_tokens + 15) / 16 * 16 + (8 * (n_tokens + 1) + 15) / 16 * 16);
  if (card == nullptr || !aligned(card, 16) || card_bytes < least + tables || k_out == nullptr ||
      v_out == nullptr || !aligned(k_out, 16) || !aligned(v_out, 16))
    return Q4KV_ERR_INVALID_ARG;
  return from_cuda(launch_card_decode(head_dim, n_kv_heads, static_cast<const uint8_t*>(card),
                                      static_cast<int64_t>(card_bytes), n_tokens, k_out, v_out, out_dtype,
                                      error_word, as_stream(stream)));
}

q4kv_status q4kv_selftest_bounded_wait(uint32_t* error_word, int32_t tries, void* stream) {
  if (error_word == nullptr || !aligned(error_word, 4) || tries < 1 || tries > (1 << 21))
    return Q4KV_ERR_INVALID_ARG;
  return from_cuda(launch_selftest_wait(error_word, static_cast<unsigned>(tries), as_stream(stream)));
}

q4kv_status q4kv_dequantize(const q4kv_pool* pool, const int32_t* block_ids, int32_t n_blocks,
                            void* k_out, void* v_out, int32_t out_dtype, int32_t unrotate_k,
                            void* stream) {
  q4kv_status st = check_pool(pool);
  if (st != Q4KV_OK) return st;
  if (n_blocks < 0 || (out_dtype != Q4KV_F32 && out_dtype != Q4KV_F16) ||
      (unrotate_k != 0 && unrotate_k != 1))
    return Q4KV_ERR_INVALID_ARG;
  if (n_blocks == 0) return Q4KV_OK;
  if (block_ids == nullptr || k_out == nullptr || v_out == nullptr || !aligned(block_ids, 4) ||
      !aligned(k_out, 16) || !aligned(v_out, 16))
    return Q4KV_ERR_INVALID_ARG;
  return from_cuda(launch_dequantize(view_of(*pool), block_ids, n_blocks, k_out, v_out,
                                     out_dtype, unrotate_k, as_stream(stream)));
}

q4kv_status q4kv_invalidate_slots(const q4kv_pool* pool, const int64_t* slot_ids, int64_t n_slots,
                                  void* stream) {
  q4kv_status st = check_pool(pool);
  if (st != Q4KV_OK) return st;
  if (n_slots < 0) return Q4KV_ERR_INVALID_ARG;
  if (n_slots == 0) return Q4KV_OK;
  if (slot_ids == nullptr || !aligned(slot_ids, 8)) return Q4KV_ERR_INVALID_ARG;
  return from_cuda(launch_invalidate(view_of(*pool), slot_ids, n_slots, as_stream(stream)));
}

q4kv_status q4kv_block_absmean(const void* k, int32_t in_dtype, int64_t n_tokens,
                               int64_t token_stride, int32_t n_kv_heads, int32_t head_dim,
                               double* out, void* stream) {
  if (n_kv_heads < 1 || head_dim < 1 || (static_cast<int64_t>(n_kv_heads) * head_dim) % 8 != 0)
    return Q4KV_ERR_INVALID_ARG;
  q4kv_status st = check_input(k, in_dtype, n_tokens, token_stride, n_kv_heads, head_dim);
  if (st != Q4KV_OK) return st;
  if (n_tokens == 0) return Q4KV_OK;
  if (out == nullptr || !aligned(out, 8)) return Q4KV_ERR_INVALID_ARG;
  if ((n_tokens + kBlockTokens - 1) / kBlockTokens > 0x7fffffff) return Q4KV_ERR_INVALID_ARG;
  return from_cuda(
      launch_absmean(k, in_dtype, n_tokens, token_stride, n_kv_heads, head_dim, out, as_stream(stream)));
}

q4kv_status q4kv_mixed_block_ids(const double* absmean, int32_t n_chunks, int32_t n_q8,
                                 int32_t q4_first, int32_t q8_first, int32_t* block_ids,
                                 void* stream) {
  if (n_chunks < 0 || n_chunks > 65536 || n_q8 < 0 || n_q8 > n_chunks || q4_first < 0 ||
      q8_first < 0)
    return Q4KV_ERR_INVALID_ARG;
  if (n_chunks == 0) return Q4KV_OK;
  if (absmean == nullptr || block_ids == nullptr || !aligned(absmean, 8) || !aligned(block_ids, 4))
    return Q4KV_ERR_INVALID_ARG;
  return from_cuda(launch_mixed_ids(absmean, n_chunks, n_q8, q4_first, q8_first, block_ids,
                                    as_stream(stream)));
}

// Longest work item the split model chooses, in 256-token blocks.
constexpr int64_t kMaxItemBlocks = 64;

q4kv_status q4kv_decode_plan_make(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                  int32_t head_dim, int32_t max_blocks_per_seq, int32_t n_splits,
                                  int32_t num_sms, q4kv_decode_plan* plan) {
  if (plan == nullptr || batch < 0 || n_q_heads < 1 || n_kv_heads < 1 ||
      max_blocks_per_seq < 1 || n_splits < 0 || num_sms < 0 || n_q_heads % n_kv_heads != 0)
    return Q4KV_ERR_INVALID_ARG;
  if (batch > 65535 || n_kv_heads > 65535) return Q4KV_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_blocks_per_seq) * kBlockTokens > 0x7fffffff)
    return Q4KV_ERR_INVALID_ARG;
  const int g = n_q_heads / n_kv_heads;
  if (head_dim != 128 && head_dim != 256) return Q4KV_ERR_UNSUPPORTED;
  if (g > 8 || g * head_dim / kGroup > 16) return Q4KV_ERR_UNSUPPORTED;
  if (num_sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return Q4KV_ERR_CUDA;
  }
  // kernel 1 (tensor-core pipeline) handles every shape accepted above; its
  // splits are whole 256-token blocks
  const int kernel = 1;
  const int64_t unit = kBlockTokens;
  const int64_t nb = max_blocks_per_seq;
  const int64_t ctx = nb * kBlockTokens;
  int64_t s = n_splits;
  if (s == 0) {
    // persistent CTAs (one per SM) take items (sequence, KV head, split) in
    // waves; cost = waves * (blocks per item + per-item cost).  The per-item
    // cost (what an item boundary costs the consumer warps: loading the next
    // item's query operands, handing the state to the aux warp that merges
    // it) is 0.9 block-time, fitted to decode times measured with forced
    // split counts on the Gemma-, Llama- and Qwen-shaped layers and the
    // batch/context sweep.
    //
    // Items are capped at kMaxItemBlocks blocks.  A warp's value sums are
    // accumulated by the tensor cores in fp32 over every tile of its item,
    // and the code-times-scale part nearly cancels the zero part, so their
    // rounding grows with the item's length: with one item per 131072-token
    // sequence the attention output was off by 2.2e-2 relative (L2), with
    // 32768 tokens per item by 2.7e-3.
    const int64_t pairs = static_cast<int64_t>(batch > 0 ? batch : 1) * n_kv_heads;
    const int64_t smin = (nb + kMaxItemBlocks - 1) / kMaxItemBlocks;
    double best = 1e300;
    s = smin;
    for (int64_t cand = smin; cand <= nb; ++cand) {
      const int64_t bps = (nb + cand - 1) / cand;
      if ((nb + bps - 1) / bps != cand) continue;         // each distinct split only once
      const int64_t items = pairs * cand;
      const int64_t waves = (items + num_sms - 1) / num_sms;
      const double cost = static_cast<double>(waves) * (static_cast<double>(bps) + 0.9);
      if (cost < best - 1e-9) {
        best = cost;
        s = cand;
      }
    }
  }
  if (s < 1) s = 1;
  if (s > nb) s = nb;
  if (s > 65535) s = 65535;
  int64_t tps = (ctx + s - 1) / s;
  tps = (tps + unit - 1) / unit * unit;
  s = (ctx + tps - 1) / tps;
  memset(plan, 0, sizeof(*plan));
  plan->batch = batch;
  plan->n_q_heads = n_q_heads;
  plan->n_kv_heads = n_kv_heads;
  plan->head_dim = head_dim;
  plan->max_blocks_per_seq = max_blocks_per_seq;
  plan->n_splits = static_cast<int32_t>(s);
  plan->tokens_per_split = static_cast<int32_t>(tps);
  plan->kernel = kernel;
  if (s > 1) {
    const size_t rows = static_cast<size_t>(batch) * n_q_heads * s;
    plan->workspace_bytes = round_up(rows * head_dim * sizeof(float), 256) + round_up(rows * 2 * sizeof(float), 256);
  }
  return Q4KV_OK;
}

// Arguments of a decode, filled into *a; *empty = 1 when there is nothing to do.
static q4kv_status prepare_decode(const q4kv_pool* pool, const q4kv_decode_plan* plan, const void* q,
                                  int32_t q_dtype, const int32_t* block_tables, const int32_t* seq_lens,
                                  float softmax_scale, void* out, int32_t out_dtype, void* workspace,
                                  size_t workspace_bytes, DecodeArgs* a, int* empty) {
  *empty = 1;
  q4kv_status st = check_pool(pool);
  if (st != Q4KV_OK) return st;
  if (plan == nullptr) return Q4KV_ERR_INVALID_ARG;
  // the plan must be one q4kv_decode_plan_make would produce for this pool
  q4kv_decode_plan ref;
  st = q4kv_decode_plan_make(plan->batch, plan->n_q_heads, plan->n_kv_heads, plan->head_dim,
                             plan->max_blocks_per_seq, plan->n_splits, 1, &ref);
  if (st != Q4KV_OK) return st;
  if (plan->head_dim != pool->head_dim || plan->n_kv_heads != pool->n_kv_heads ||
      ref.n_splits != plan->n_splits || ref.tokens_per_split != plan->tokens_per_split ||
      ref.workspace_bytes != plan->workspace_bytes || (plan->kernel != 0 && plan->kernel != 1))
    return Q4KV_ERR_INVALID_ARG;
  if ((q_dtype != Q4KV_F16 && q_dtype != Q4KV_BF16) ||
      (out_dtype != Q4KV_F32 && out_dtype != Q4KV_F16 && out_dtype != Q4KV_BF16) ||
      !isfinite(softmax_scale))
    return Q4KV_ERR_INVALID_ARG;
  if (plan->batch == 0) return Q4KV_OK;
  *empty = 0;
  if (q == nullptr || block_tables == nullptr || seq_lens == nullptr || out == nullptr ||
      !aligned(q, 16) || !aligned(block_tables, 16) || !aligned(seq_lens, 4) || !aligned(out, 16))
    return Q4KV_ERR_INVALID_ARG;
  if (pool->n_q4_blocks + pool->n_q8_blocks + pool->n_q2_blocks == 0) return Q4KV_ERR_INVALID_ARG;
  // the CUDA-core variant reads 4- and 8-bit blocks only
  if (plan->kernel == 0 && pool->n_q2_blocks > 0) return Q4KV_ERR_UNSUPPORTED;
  // TMA row coordinates are int32: (blocks of one width) x heads x 256 < 2^31
  int64_t widest = pool->n_q4_blocks > pool->n_q8_blocks ? pool->n_q4_blocks : pool->n_q8_blocks;
  if (pool->n_q2_blocks > widest) widest = pool->n_q2_blocks;
  const int64_t code_rows = widest * pool->n_kv_heads * kBlockTokens;
  if (code_rows >= (int64_t{1} << 31)) return Q4KV_ERR_UNSUPPORTED;
  // the FP8 comparison cache is read by the tensor-core kernel only
  if (pool->value_format == Q4KV_FORMAT_FP8 && plan->kernel != 1) return Q4KV_ERR_UNSUPPORTED;
  if (plan->workspace_bytes > 0 &&
      (workspace == nullptr || workspace_bytes < plan->workspace_bytes || !aligned(workspace, 256)))
    return Q4KV_ERR_WORKSPACE;
  a->pool = view_of(*pool);
  a->plan = *plan;
  a->q = q;
  a->q_dtype = q_dtype;
  a->tables = block_tables;
  a->seq_lens = seq_lens;
  a->add_lens = nullptr;
  a->add_const = 0;
  a->defer_wait = 0;
  a->app_k = nullptr;
  a->app_v = nullptr;
  a->app_dtype = 0;
  a->app_seq_stride = 0;
  a->app_token_stride = 0;
  a->scale = softmax_scale > 0.0f ? softmax_scale : 1.0f / sqrtf(static_cast<float>(plan->head_dim));
  a->out = out;
  a->out_dtype = out_dtype;
  const size_t rows = static_cast<size_t>(plan->batch) * plan->n_q_heads * plan->n_splits;
  a->ws_o = static_cast<float*>(workspace);
  a->ws_ml = plan->workspace_bytes > 0
                 ? reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                            round_up(rows * plan->head_dim * sizeof(float), 256))
                 : nullptr;
  return Q4KV_OK;
}

q4kv_status q4kv_decode_attention(const q4kv_pool* pool, const q4kv_decode_plan* plan,
                                  const void* q, int32_t q_dtype, const int32_t* block_tables,
                                  const int32_t* seq_lens, float softmax_scale, void* out,
                                  int32_t out_dtype, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  DecodeArgs a;
  int empty = 1;
  const q4kv_status st = prepare_decode(pool, plan, q, q_dtype, block_tables, seq_lens, softmax_scale, out,
                                        out_dtype, workspace, workspace_bytes, &a, &empty);
  if (st != Q4KV_OK || empty) return st;
  return from_cuda(launch_decode(a, as_stream(stream)));
}

q4kv_status q4kv_append_decode(const q4kv_pool* pool, const q4kv_decode_plan* plan, const void* k_new,
                               const void* v_new, int32_t in_dtype, int32_t max_new, const int32_t* n_new,
                               int64_t seq_stride, int64_t token_stride, const void* q, int32_t q_dtype,
                               const int32_t* block_tables, const int32_t* seq_lens, float softmax_scale,
                               void* out, int32_t out_dtype, void* workspace, size_t workspace_bytes,
                               void* stream) {
  if (plan == nullptr) return Q4KV_ERR_INVALID_ARG;
  int64_t rows = 0;
  q4kv_status st = check_append(pool, k_new, v_new, in_dtype, plan->batch, max_new, n_new, seq_stride,
                                token_stride, block_tables, plan->max_blocks_per_seq, seq_lens, &rows);
  if (st != Q4KV_OK) return st;
  DecodeArgs a;
  int empty = 1;
  st = prepare_decode(pool, plan, q, q_dtype, block_tables, seq_lens, softmax_scale, out, out_dtype,
                      workspace, workspace_bytes, &a, &empty);
  if (st != Q4KV_OK || empty) return st;
  cudaStream_t s = as_stream(stream);
  if (rows > 0) {
    a.add_lens = n_new;
    a.add_const = max_new;
    if (!a.pool.fp8 && plan->kernel == 1) {
      // one launch: the tensor-core kernel encodes the new rows itself
      a.app_k = k_new;
      a.app_v = v_new;
      a.app_dtype = in_dtype;
      a.app_seq_stride = seq_stride;
      a.app_token_stride = token_stride;
    } else {
      const cudaError_t e = launch_append(view_of(*pool), k_new, v_new, in_dtype, plan->batch, max_new, n_new,
                                          seq_stride, token_stride, block_tables, plan->max_blocks_per_seq,
                                          seq_lens, s);
      if (e != cudaSuccess) return from_cuda(e);
      a.defer_wait = 1;
    }
  }
  return from_cuda(launch_decode(a, s));
}

q4kv_status q4kv_read_device_error(const q4kv_pool* pool, uint32_t* bits, int32_t clear,
                                   void* stream) {
  if (pool == nullptr || bits == nullptr) return Q4KV_ERR_INVALID_ARG;
  *bits = 0;
  if (pool->error_word == nullptr) return Q4KV_OK;
  cudaStream_t s = as_stream(stream);
  uint32_t host = 0;
  if (cudaMemcpyAsync(&host, pool->error_word, sizeof(host), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return Q4KV_ERR_CUDA;
  if (clear && host != 0) {
    if (cudaMemsetAsync(pool->error_word, 0, sizeof(uint32_t), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return Q4KV_ERR_CUDA;
  }
  *bits = host;
  return host != 0 ? Q4KV_ERR_DEVICE : Q4KV_OK;
}

}  // extern "C"
