// Allocation-free decode entry point: the split partials of
// q4kv_decode_attention live in a file-scope device array instead of a
// caller-provided workspace, for callers that cannot allocate device memory.
#include "q4kv_internal.cuh"

namespace {

constexpr size_t kScratchBytes = Q4KV_STATIC_SCRATCH_BYTES;

// One copy per device that loads this library, held until process exit.
__device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

// In host code `g_decode_scratch` names a host-side stand-in, not device
// memory.  The device address is looked up on every call for the device and
// context current at that moment: a cached address would dangle after a
// cudaDeviceReset or under another context that loaded the module anew.
// The lookup allocates nothing; the first one on a device loads the module.
q4kv_status scratch_address(void** addr) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess || p == nullptr) return Q4KV_ERR_CUDA;
  *addr = p;
  return Q4KV_OK;
}

}  // namespace

extern "C" q4kv_status q4kv_decode_attention_static_scratch(
    const q4kv_pool* pool, const q4kv_decode_plan* plan, const void* q, int32_t q_dtype,
    const int32_t* block_tables, const int32_t* seq_lens, float softmax_scale, void* out,
    int32_t out_dtype, void* stream) {
  if (plan == nullptr) return Q4KV_ERR_INVALID_ARG;
  if (plan->workspace_bytes > kScratchBytes) return Q4KV_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (plan->workspace_bytes > 0 && plan->batch > 0) {
    const q4kv_status st = scratch_address(&scratch);
    if (st != Q4KV_OK) return st;
  }
  return q4kv_decode_attention(pool, plan, q, q_dtype, block_tables, seq_lens, softmax_scale, out,
                               out_dtype, scratch, scratch ? kScratchBytes : 0, stream);
}
