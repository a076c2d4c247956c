// Paging blocks between the device pool and host memory.
//
// "Agent Memory Below the Prompt" (gist.science summary of arXiv 2603.04428),
// section 2.1 item 1: the cache lives in 256-token blocks that page between
// fast memory and storage; item 3: one agent's cache is brought in while
// another agent decodes; section 5: storage acts as the cache's swap space.
// Here the fast memory is HBM and the other side is pinned host memory (the
// storage tier behind it is the caller's).  A block travels as an image: a
// 16-byte header and then the block's sections byte for byte as the pool
// holds them -- K codes, V codes, K params, V params (not for FP8 pools), the
// 32-byte remap mask; its class tag is the block's code width (2, 4 or 8) or
// 0x108 for an FP8 block.
//
// Two ways to move them.  With the block ids on the device, one kernel moves
// any number of blocks in either direction, reading or writing the host side
// directly over the bus (no staging copy, no per-block copy call); it is a
// small persistent grid with no shared memory, so it shares SMs with the
// kernels beside it.  With the ids on the host, the copy engines do the
// moving (strided 2-D copies per run of consecutive ids) and no SM is used,
// which is the way to page blocks in while decode runs.
#include "q4kv_internal.cuh"

namespace q4kv {
namespace {

constexpr uint32_t kImageMagic = 0x424B3451u;   // bytes 'Q', '4', 'K', 'B'
constexpr int kPageThreads = 256;
constexpr int kPageUnroll = 4;                  // 16-byte words in flight per thread
// At most this many CTAs: 64 x 256 threads x 4 words = 1 MiB in flight, far
// more than the bus needs to stay busy (bandwidth x latency is ~100 KB), while
// the rest of every SM stays free for the kernels it runs beside.
constexpr int kPageCtas = 64;

// 16-byte word counts of one image's sections for the block class.
struct ImageWords {
  int64_t codes;    // per tensor
  int64_t params;   // per tensor (0 for FP8)
  __host__ __device__ int64_t total() const { return 1 + 2 * codes + 2 * params + 2; }
};

// bits: the block's code width (2, 4 or 8; FP8 blocks are 8 bits wide)
__host__ __device__ inline ImageWords image_words(int d, int hkv, int bits, bool fp8) {
  ImageWords w;
  w.codes = static_cast<int64_t>(hkv) * kBlockTokens * (d * bits / 8) / 16;
  w.params = fp8 ? 0 : static_cast<int64_t>(hkv) * kBlockTokens * (d / kGroup) * 4 / 16;
  return w;
}

__host__ __device__ inline uint32_t class_tag(int bits, bool fp8) { return fp8 ? 0x108u : static_cast<uint32_t>(bits); }

// The arrays and array index of a block of the pool's class `bits`.
struct ClassArrays {
  uint8_t *kc, *vc;
  void *kp, *vp;
  int64_t phys;
};
__host__ __device__ inline ClassArrays class_arrays(const PoolView& p, int32_t blk, int bits) {
  if (bits == 4) return {p.k_codes4, p.v_codes4, p.k_params4, p.v_params4, blk};
  if (bits == 8) return {p.k_codes8, p.v_codes8, p.k_params8, p.v_params8, static_cast<int64_t>(blk) - p.n_q4};
  return {p.k_codes2, p.v_codes2, p.k_params2, p.v_params2, static_cast<int64_t>(blk) - p.n_q4 - p.n_q8};
}

// Word w (1 <= w < total) of block blk's image, as a pointer into the pool.
__device__ __forceinline__ uint4* pool_word(const PoolView& p, int32_t blk, int bits, const ImageWords& iw,
                                            int64_t w) {
  const ClassArrays a = class_arrays(p, blk, bits);
  w -= 1;
  if (w < iw.codes) return reinterpret_cast<uint4*>(a.kc) + a.phys * iw.codes + w;
  w -= iw.codes;
  if (w < iw.codes) return reinterpret_cast<uint4*>(a.vc) + a.phys * iw.codes + w;
  w -= iw.codes;
  if (w < iw.params) return reinterpret_cast<uint4*>(a.kp) + a.phys * iw.params + w;
  w -= iw.params;
  if (w < iw.params) return reinterpret_cast<uint4*>(a.vp) + a.phys * iw.params + w;
  w -= iw.params;
  return reinterpret_cast<uint4*>(p.mask + static_cast<int64_t>(blk) * kMaskWords) + w;
}

// EXPORT: pool -> host images.  IMPORT: host images -> pool, after checking
// each image's header against its target block.  A small persistent grid
// walks the chunks (image i, words [c * 1024, c * 1024 + 1024)) with a grid
// stride; every thread keeps kPageUnroll loads in flight before it stores.
template <bool EXPORT>
__global__ void __launch_bounds__(kPageThreads) page_kernel(const __grid_constant__ PoolView pool,
                                                            const int32_t* __restrict__ ids, int32_t n,
                                                            uint4* host, int64_t stride_words,
                                                            int32_t chunks_per_image) {
  const int d = pool.head_dim, hkv = pool.n_kv_heads;
  const bool fp8 = pool.fp8 != 0;
  constexpr int kChunk = kPageThreads * kPageUnroll;
  const int64_t n_chunks = static_cast<int64_t>(n) * chunks_per_image;
  for (int64_t ch = blockIdx.x; ch < n_chunks; ch += gridDim.x) {
    const int64_t i = ch / chunks_per_image;
    const int64_t w0 = (ch - i * chunks_per_image) * kChunk + threadIdx.x;
    const int32_t blk = __ldg(ids + i);
    if (blk < 0 || blk >= pool.n_blocks()) {
      if (w0 == 0) raise_error(pool.error_word, Q4KV_DEVERR_BLOCK_ID);
      continue;
    }
    const int bits = pool.bits_of(blk);
    const ImageWords iw = image_words(d, hkv, bits, fp8);
    const int64_t total = iw.total();
    uint4* img = host + i * stride_words;
    const uint4 hdr = make_uint4(kImageMagic, class_tag(bits, fp8) | static_cast<uint32_t>(d) << 16,
                                 static_cast<uint32_t>(hkv), static_cast<uint32_t>(blk));
    uint4 val[kPageUnroll];
    if constexpr (EXPORT) {
#pragma unroll
      for (int u = 0; u < kPageUnroll; ++u) {
        const int64_t w = w0 + u * kPageThreads;
        if (w > 0 && w < total) val[u] = __ldg(pool_word(pool, blk, bits, iw, w));
      }
#pragma unroll
      for (int u = 0; u < kPageUnroll; ++u) {
        const int64_t w = w0 + u * kPageThreads;
        if (w < total) img[w] = w == 0 ? hdr : val[u];
      }
    } else {
      const uint4 got = img[0];   // the header, loaded beside the data
#pragma unroll
      for (int u = 0; u < kPageUnroll; ++u) {
        const int64_t w = w0 + u * kPageThreads;
        if (w > 0 && w < total) val[u] = img[w];
      }
      // magic, class, head_dim and Hkv must fit the block; the source id is informational
      if (got.x != hdr.x || got.y != hdr.y || got.z != hdr.z) {
        if (w0 == 0) raise_error(pool.error_word, Q4KV_DEVERR_IMAGE);
        continue;
      }
#pragma unroll
      for (int u = 0; u < kPageUnroll; ++u) {
        const int64_t w = w0 + u * kPageThreads;
        if (w > 0 && w < total) *pool_word(pool, blk, bits, iw, w) = val[u];
      }
    }
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// Copy-engine path (block ids known on the host): no kernel and no SM time.
// The CPU writes (export) or checks (import) each image's header in the
// pinned buffer, and each run of consecutive ids of one class whose images
// are consecutive moves as one strided 2-D copy per section: rows of one
// section's bytes, the pool side dense, the host side at the image stride.
// ---------------------------------------------------------------------------
namespace {

struct HostClass {
  int bits;
  ImageWords iw;
};

HostClass host_class(const PoolView& p, int32_t blk) {
  HostClass c;
  c.bits = p.bits_of(blk);
  c.iw = image_words(p.head_dim, p.n_kv_heads, c.bits, p.fp8 != 0);
  return c;
}

void host_header(const PoolView& p, int32_t blk, const HostClass& c, uint32_t out[4]) {
  out[0] = kImageMagic;
  out[1] = class_tag(c.bits, p.fp8 != 0) | static_cast<uint32_t>(p.head_dim) << 16;
  out[2] = static_cast<uint32_t>(p.n_kv_heads);
  out[3] = static_cast<uint32_t>(blk);
}

}  // namespace

cudaError_t copy_pages(const PoolView& p, const int32_t* ids, int32_t n, uint8_t* host, bool to_host,
                       cudaStream_t stream) {
  const int64_t stride = image_stride_bytes(p);
  int32_t i = 0;
  while (i < n) {
    const HostClass c = host_class(p, ids[i]);
    int32_t len = 1;   // the run: ids[i] + r for r < len, all of the same class
    while (i + len < n && ids[i + len] == ids[i] + len && host_class(p, ids[i + len]).bits == c.bits) ++len;
    const int64_t cb = c.iw.codes * 16, pb = c.iw.params * 16;
    const ClassArrays a = class_arrays(p, ids[i], c.bits);
    struct Sec {
      void* pool;
      int64_t bytes, image_off;
    } secs[5] = {
        {a.kc + a.phys * cb, cb, 16},
        {a.vc + a.phys * cb, cb, 16 + cb},
        {static_cast<uint8_t*>(a.kp) + a.phys * pb, pb, 16 + 2 * cb},
        {static_cast<uint8_t*>(a.vp) + a.phys * pb, pb, 16 + 2 * cb + pb},
        {p.mask + static_cast<int64_t>(ids[i]) * kMaskWords, kMaskWords * 4, 16 + 2 * cb + 2 * pb},
    };
    for (const Sec& sec : secs) {
      if (sec.bytes == 0) continue;   // FP8 blocks have no params
      uint8_t* img = host + static_cast<int64_t>(i) * stride + sec.image_off;
      const cudaError_t e =
          to_host ? cudaMemcpy2DAsync(img, stride, sec.pool, sec.bytes, sec.bytes, len, cudaMemcpyDeviceToHost, stream)
                  : cudaMemcpy2DAsync(sec.pool, sec.bytes, img, stride, sec.bytes, len, cudaMemcpyHostToDevice, stream);
      if (e != cudaSuccess) return e;
    }
    i += len;
  }
  return cudaSuccess;
}

// Host side of the copy-engine path: headers written (export) or checked
// (import) by the CPU before any copy is enqueued.  Returns false when an
// import header does not fit its target block.
bool host_headers(const PoolView& p, const int32_t* ids, int32_t n, uint8_t* host, bool write) {
  const int64_t stride = image_stride_bytes(p);
  for (int32_t i = 0; i < n; ++i) {
    uint32_t h[4];
    host_header(p, ids[i], host_class(p, ids[i]), h);
    uint32_t* img = reinterpret_cast<uint32_t*>(host + static_cast<int64_t>(i) * stride);
    if (write) {
      for (int w = 0; w < 4; ++w) img[w] = h[w];
    } else if (img[0] != h[0] || img[1] != h[1] || img[2] != h[2]) {
      return false;
    }
  }
  return true;
}

int64_t image_stride_bytes(const PoolView& pool) {
  const bool fp8 = pool.fp8 != 0;
  // the widest class present (a pool with no blocks: as if 4-bit)
  const int bits = (fp8 || pool.n_q8 > 0) ? 8 : (pool.n_q4 > 0 || pool.n_q2 == 0 ? 4 : 2);
  return image_words(pool.head_dim, pool.n_kv_heads, bits, fp8).total() * 16;
}

cudaError_t launch_page(const PoolView& pool, const int32_t* ids, int32_t n, void* host, bool to_host,
                        cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int64_t stride_words = image_stride_bytes(pool) / 16;
  const int64_t per_cta = static_cast<int64_t>(kPageThreads) * kPageUnroll;
  const int32_t chunks = static_cast<int32_t>((stride_words + per_cta - 1) / per_cta);
  const int64_t all = static_cast<int64_t>(n) * chunks;
  const dim3 grid(static_cast<unsigned>(all < kPageCtas ? all : kPageCtas));
  if (to_host)
    page_kernel<true><<<grid, kPageThreads, 0, stream>>>(pool, ids, n, static_cast<uint4*>(host), stride_words,
                                                         chunks);
  else
    page_kernel<false><<<grid, kPageThreads, 0, stream>>>(pool, ids, n, static_cast<uint4*>(host), stride_words,
                                                          chunks);
  return cudaGetLastError();
}

}  // namespace q4kv
