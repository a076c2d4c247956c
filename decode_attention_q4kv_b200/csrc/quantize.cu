// Encoder and decoder of the paged 4/8-bit KV format.
//
// Format: "Agent Memory Below the Prompt" (arXiv 2603.04428 summary), sec. 2.1
// item 2 -- codes packed into uint32 words, one 16-bit scale and one 16-bit
// bias per group; keys rotated by a Walsh-Hadamard transform before coding,
// values not (UltraQuant news item, arXiv 2606.20474, "技術/ビジネス面").
//
// Work mapping: a warp takes one KV head of 4 consecutive tokens (D = 128) or
// 2 consecutive tokens (D = 256).  Each lane holds 16 consecutive channels of
// one (token, head) vector, so the rotation runs as 4 butterfly stages inside
// the lane followed by 3 (or 4) stages across lanes with warp shuffles, and a
// 64-value group spans 4 lanes.  The warp's code rows are contiguous in the
// pool (consecutive slots of one block and head), so its stores form one
// 256-byte (Q4, D = 128) run.
//
// Bit-exactness: every arithmetic step is one IEEE binary32 operation written
// with an _rn intrinsic (no contraction, no reassociation): butterflies in
// ascending stride order, one multiply by c, exact min/max, subtraction and
// division for the scale, fp16 round-to-nearest-even for scale and zero,
// subtraction and division for each code, round-half-even to an integer,
// clamp.  Dequantisation is fma(code, s, z), equal to code*s + z because the
// product is exact.
#include "async_copy.cuh"
#include "encode.cuh"
#include "q4kv_internal.cuh"

namespace q4kv {
namespace {

// ---------------------------------------------------------------------------
// Encoder kernel.  Persistent CTAs (one per SM): one producer warp streams
// the K and V rows of a unit -- T consecutive tokens x a run of H' heads,
// 16 KB of input per tensor -- into a 4-deep ring of shared-memory stages
// with bulk copies (one copy per token row, or one per tensor when the run
// is contiguous in memory); 23 consumer warps encode its warp items: VPW
// tokens of one head, a lane holding 16 channels.  T and H'
// are chosen so that every full unit holds exactly 16 warp items.
// ---------------------------------------------------------------------------
constexpr int kQConsumers = 23;                 // consumer warps (6 warps per scheduler)
constexpr int kQItems = 16;                     // warp items in a full unit
constexpr int kQThreads = (kQConsumers + 1) * 32;
constexpr int kQStages = 4;
constexpr int kQFull = 2 * kQStages;            // full barriers: two per stage, by unit mod 8
constexpr int kQHalf = 16384;                 // input bytes of one tensor per stage
constexpr int kQStageBytes = 2 * kQHalf;
static_assert((kQStages & (kQStages - 1)) == 0, "stage index is a mask");

struct EncodeGeometry {
  uint32_t n_tokens;
  int64_t stride;        // elements between consecutive tokens
  int32_t unit_tokens;   // T
  int32_t unit_heads;    // H'
  int32_t head_chunks;   // ceil(Hkv / H')
  uint32_t n_chunks;     // ceil(n_tokens / T)
  int32_t items_per_head_log2;   // log2(T / VPW)
};

template <int D, typename InT, bool ROT, bool MIXED, bool FP8 = false>
__global__ void __launch_bounds__(kQThreads, 1)
    quantize_kernel(const __grid_constant__ PoolView pool, const InT* __restrict__ k,
                    const InT* __restrict__ v, const __grid_constant__ EncodeGeometry geo,
                    const int32_t* __restrict__ block_ids) {
  using S = Shape<D>;
  extern __shared__ __align__(128) uint8_t qsmem[];
  uint8_t* stages = qsmem;
  uint64_t* full = reinterpret_cast<uint64_t*>(qsmem + kQStages * kQStageBytes);   // [kQFull]
  uint64_t* empty = full + kQFull;                                                 // [kQStages]
  __shared__ int s_timeout;

  griddep_wait();   // the inputs may come from the kernel before in the stream
  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hkv = pool.n_kv_heads;
  const int T = geo.unit_tokens, HP = geo.unit_heads, HC = geo.head_chunks;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kQFull; ++i) mbar_init(&full[i], 1);
    for (int i = 0; i < kQStages; ++i) mbar_init(&empty[i], kQItems);
    s_timeout = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kQConsumers) {
    // ---------------- producer ----------------
    if (lane != 0) return;
    uint32_t it = 0;
    bool stop = false;
    for (uint32_t c = blockIdx.x; c < geo.n_chunks && !stop; c += gridDim.x) {
      const uint32_t t0 = c * T;
      const int nvalid = static_cast<int>(umin(static_cast<uint32_t>(T), geo.n_tokens - t0));
      for (int hc = 0; hc < HC; ++hc, ++it) {
        const int s = it % kQStages;
        uint64_t* fb = &full[it % kQFull];
        if (!mbar_wait(&empty[s], ((it / kQStages) & 1) ^ 1)) {
          // production ends; an arrival here could fall in a phase still in
          // flight, so the consumers find out through their own bounded waits
          s_timeout = 1;
          stop = true;
          break;
        }
        const int h0 = hc * HP, nh = min(HP, hkv - h0);
        const uint32_t row = static_cast<uint32_t>(nh) * D * sizeof(InT);   // bytes per token
        uint8_t* dst = stages + s * kQStageBytes;
        mbar_arrive_tx(fb, 2u * nvalid * row);
        const InT* ks = k + static_cast<int64_t>(t0) * geo.stride + h0 * D;
        const InT* vs = v + static_cast<int64_t>(t0) * geo.stride + h0 * D;
        if (nh == hkv && geo.stride == static_cast<int64_t>(hkv) * D) {
          bulk_g2s(dst, ks, nvalid * row, fb);
          bulk_g2s(dst + kQHalf, vs, nvalid * row, fb);
        } else {
          for (int t = 0; t < nvalid; ++t) {
            bulk_g2s(dst + t * row, ks + t * geo.stride, row, fb);
            bulk_g2s(dst + kQHalf + t * row, vs + t * geo.stride, row, fb);
          }
        }
      }
    }
    // no copy may still be landing when the CTA exits
    for (uint32_t q = (it > kQStages ? it - kQStages : 0); q < it; ++q)
      if (!mbar_wait(&full[q % kQFull], (q / kQFull) & 1)) break;
    return;
  }

  // ---------------- consumers ----------------
  // The CTA's units come in the producer's order; their warp items (16 per
  // unit, item w = head w / tpi of the unit's run, tokens (w % tpi) * VPW ..
  // + VPW - 1 of its T) form one stream that warp w walks with stride 23.
  // A stage is released after its 16 items have arrived.  The position
  // (chunk c, head chunk hc, unit ul, item w16) advances without division.
  //
  // A parity wait tells only two phases of a barrier apart.  With stride 23 a
  // warp has no item in some units (never two in a row), so with one full
  // barrier per stage it could wait for unit u without having seen unit u - 4
  // (same stage) complete, and a copy of u - 4 landing after later units'
  // copies would let that wait return on the earlier phase: the warp would
  // read the wrong data and arrive on the wrong phase of the empty barrier,
  // after which the producer can arrive twice on one full phase.  Unit u
  // therefore completes full barrier u mod 8 (two per stage), whose previous
  // phase is unit u - 8.  A warp that waits for u has seen its previous item's
  // unit (u - 1 or u - 2) land, so the producer had issued u - 4, which it
  // does only once the items of u - 8 are released, i.e. after u - 8 landed;
  // and the barrier cannot be past u while this warp's item in u is held.
  const int r = lane / S::LPV;       // token of the warp item
  const int j = lane % S::LPV;       // 16-channel run of the lane
  const int tpi_log = geo.items_per_head_log2;   // tpi = T / VPW, a power of two
  struct Pos {
    uint32_t c, ul;
    int hc, w16;
  };
  auto advance = [&](Pos& p, int by) {
    p.w16 += by;
    while (p.w16 >= kQItems) {
      p.w16 -= kQItems;
      ++p.ul;
      if (++p.hc == HC) {
        p.hc = 0;
        p.c += gridDim.x;
      }
    }
  };
  Pos pos = {blockIdx.x, 0u, 0, 0};
  advance(pos, warp);
  int32_t blk = pos.c < geo.n_chunks ? __ldg(block_ids + (pos.c * T) / kBlockTokens) : 0;
  while (pos.c < geo.n_chunks) {
    Pos nxt = pos;
    advance(nxt, kQConsumers);
    const int32_t blk_next = nxt.c < geo.n_chunks ? __ldg(block_ids + (nxt.c * T) / kBlockTokens) : 0;
    const int s = pos.ul & (kQStages - 1);
    if (!mbar_wait(&full[pos.ul % kQFull], (pos.ul / kQFull) & 1) || s_timeout) {
      if (lane == 0) raise_error(pool.error_word, Q4KV_DEVERR_TIMEOUT);
      break;
    }
    const uint32_t t0 = pos.c * T;
    const int h0 = pos.hc * HP, nh = min(HP, hkv - h0);
    const int hh = pos.w16 >> tpi_log;
    const int ti = (pos.w16 & ((1 << tpi_log) - 1)) * S::VPW;   // first token of the item in the unit
    const int tt = ti + r;
    if (hh < nh) {
      const uint32_t t = t0 + tt;
      const bool valid = t < geo.n_tokens;
      const uint8_t* src = stages + s * kQStageBytes + ((tt * nh + hh) * D + j * kEPL) * sizeof(InT);
      const uint4 k0 = lds16(src), k1 = lds16(src + 16);
      const uint4 v0 = lds16(src + kQHalf), v1 = lds16(src + kQHalf + 16);
      const int h = h0 + hh;
      if (blk < 0 || blk >= pool.n_blocks()) {
        if (lane == 0) raise_error(pool.error_word, Q4KV_DEVERR_BLOCK_ID);
      } else {
        const int slot = static_cast<int>(t % kBlockTokens);
        // a pool with only 4-bit blocks drops the other widths' paths
        const int bits = MIXED ? pool.bits_of(blk) : 4;
        const bool is8 = bits == 8;
        const int64_t phys = bits == 4 ? blk : (is8 ? blk - pool.n_q4 : blk - pool.n_q4 - pool.n_q8);
        const int64_t row = (phys * hkv + h) * kBlockTokens + slot;   // (block, head, slot)
        float2 xk[8], xv[8];
        unpack16<InT>(k0, k1, xk);
        unpack16<InT>(v0, v1, xv);
        if constexpr (FP8) {
          if (valid) {
            store_fp8(xk, pool.k_codes8 + row * D + j * kEPL);
            store_fp8(xv, pool.v_codes8 + row * D + j * kEPL);
          }
        } else {
          if (ROT) rotate_pairs<D>(xk, j);   // keys are coded rotated, values as they are
          constexpr float ks = ROT ? kRotScale<D> : 1.0f;
          if (is8)
            encode_kv<8>(xk, ks, xv, j, valid, pool.k_codes8 + row * D, pool.k_params8 + row * S::NG,
                         pool.v_codes8 + row * D, pool.v_params8 + row * S::NG);
          else if (MIXED && bits == 2)
            encode_kv<2>(xk, ks, xv, j, valid, pool.k_codes2 + row * (D / 4), pool.k_params2 + row * S::NG,
                         pool.v_codes2 + row * (D / 4), pool.v_params2 + row * S::NG);
          else
            encode_kv<4>(xk, ks, xv, j, valid, pool.k_codes4 + row * (D / 2), pool.k_params4 + row * S::NG,
                         pool.v_codes4 + row * (D / 2), pool.v_params4 + row * S::NG);
        }
        // freshly written slots are live: one word update for the item's tokens
        const uint32_t tf = t0 + ti;
        if (h == 0) {
          const bool doit = lane == 0 && tf < geo.n_tokens;
          const int nv = doit ? static_cast<int>(umin(static_cast<uint32_t>(S::VPW), geo.n_tokens - tf)) : 0;
          const int sf = static_cast<int>(tf % kBlockTokens);
          red_and_if(doit, pool.mask + static_cast<int64_t>(blk) * kMaskWords + sf / 32,
                     ~(((1u << nv) - 1u) << (sf % 32)));
        }
      }
    }
    __syncwarp();
    arrive_if(lane == 0, &empty[s]);
    pos = nxt;
    blk = blk_next;
  }
}

// Scalar butterflies for the decoder's optional un-rotation (channels 16j ..
// 16j+15 of the lane in order); same stage order and operations as above.
// ---------------------------------------------------------------------------
// Append kernel: new tokens of many sequences, each at its own position.  A
// warp item is one (sequence, new token) and VPW consecutive KV heads (a lane
// holds 16 channels of one head, as in the bulk encoder, so the rotation and
// the group statistics are the same warp code); items are walked with a grid
// stride.  The data are small (a few tokens per sequence), so rows are read
// with plain 16-byte loads.
// ---------------------------------------------------------------------------
template <int D, typename InT, bool ROT>
__global__ void __launch_bounds__(256) append_kernel(const __grid_constant__ PoolView pool,
                                                     const InT* __restrict__ k, const InT* __restrict__ v,
                                                     int32_t batch, int32_t max_new,
                                                     const int32_t* __restrict__ n_new, int64_t seq_stride,
                                                     int64_t token_stride, const int32_t* __restrict__ tables,
                                                     int32_t max_blocks, const int32_t* __restrict__ seq_lens) {
  using S = Shape<D>;
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int r = lane / S::LPV, j = lane % S::LPV;
  const int hkv = pool.n_kv_heads;
  const int hgroups = (hkv + S::VPW - 1) / S::VPW;
  const int64_t n_items = static_cast<int64_t>(batch) * max_new * hgroups;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t item = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; item < n_items;
       item += n_warps) {
    const int hg = static_cast<int>(item % hgroups);
    const int64_t bi = item / hgroups;
    const int i = static_cast<int>(bi % max_new);
    const int b = static_cast<int>(bi / max_new);
    if (n_new != nullptr && i >= __ldg(n_new + b)) continue;    // warp-uniform
    const int len = __ldg(seq_lens + b);
    const int64_t p = static_cast<int64_t>(len) + i;
    if (len < 0 || p >= static_cast<int64_t>(max_blocks) * kBlockTokens) {
      if (lane == 0 && hg == 0) raise_error(pool.error_word, Q4KV_DEVERR_SEQ_LEN);
      continue;
    }
    const int32_t blk = __ldg(tables + static_cast<int64_t>(b) * max_blocks + p / kBlockTokens);
    if (blk < 0 || blk >= pool.n_blocks()) {
      if (lane == 0 && hg == 0) raise_error(pool.error_word, Q4KV_DEVERR_BLOCK_ID);
      continue;
    }
    const int slot = static_cast<int>(p % kBlockTokens);
    const int h = hg * S::VPW + r;
    const bool valid = h < hkv;
    const int hs = valid ? h : hkv - 1;   // lanes past the last head read a real row, store nothing
    const int64_t src = static_cast<int64_t>(b) * seq_stride + static_cast<int64_t>(i) * token_stride +
                        static_cast<int64_t>(hs) * D + j * kEPL;
    const uint4 k0 = __ldg(reinterpret_cast<const uint4*>(k + src));
    const uint4 k1 = __ldg(reinterpret_cast<const uint4*>(k + src) + 1);
    const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(v + src));
    const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(v + src) + 1);
    const int bits = pool.bits_of(blk);
    const bool is8 = bits == 8;
    const int64_t phys = bits == 4 ? blk : (is8 ? blk - pool.n_q4 : blk - pool.n_q4 - pool.n_q8);
    const int64_t row = (phys * hkv + hs) * kBlockTokens + slot;   // (block, head, slot)
    float2 xk[8], xv[8];
    unpack16<InT>(k0, k1, xk);
    unpack16<InT>(v0, v1, xv);
    if (pool.fp8) {   // FP8 comparison cache
      if (valid) {
        store_fp8(xk, pool.k_codes8 + row * D + j * kEPL);
        store_fp8(xv, pool.v_codes8 + row * D + j * kEPL);
      }
      if (lane == 0 && hg == 0)
        atomicAnd(pool.mask + static_cast<int64_t>(blk) * kMaskWords + slot / 32, ~(1u << (slot % 32)));
      continue;
    }
    if (ROT) rotate_pairs<D>(xk, j);
    constexpr float ks = ROT ? kRotScale<D> : 1.0f;
    if (is8)
      encode_kv<8>(xk, ks, xv, j, valid, pool.k_codes8 + row * D, pool.k_params8 + row * S::NG,
                   pool.v_codes8 + row * D, pool.v_params8 + row * S::NG);
    else if (bits == 2)
      encode_kv<2>(xk, ks, xv, j, valid, pool.k_codes2 + row * (D / 4), pool.k_params2 + row * S::NG,
                   pool.v_codes2 + row * (D / 4), pool.v_params2 + row * S::NG);
    else
      encode_kv<4>(xk, ks, xv, j, valid, pool.k_codes4 + row * (D / 2), pool.k_params4 + row * S::NG,
                   pool.v_codes4 + row * (D / 2), pool.v_params4 + row * S::NG);
    if (lane == 0 && hg == 0)
      atomicAnd(pool.mask + static_cast<int64_t>(blk) * kMaskWords + slot / 32, ~(1u << (slot % 32)));
  }
}

template <int D>
__device__ __forceinline__ void fwht_vector(float (&x)[kEPL], int j) {
#pragma unroll
  for (int h = 1; h < kEPL; h <<= 1) {
#pragma unroll
    for (int i = 0; i < kEPL; ++i) {
      if ((i & h) == 0) {
        const float a = x[i], b = x[i + h];
        x[i] = __fadd_rn(a, b);
        x[i + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int h = kEPL; h < D; h <<= 1) {
    const int lane_bit = h / kEPL;
    const bool upper = (j & lane_bit) != 0;
#pragma unroll
    for (int i = 0; i < kEPL; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, x[i], lane_bit);
      x[i] = upper ? __fsub_rn(other, x[i]) : __fadd_rn(x[i], other);
    }
  }
}

template <int D>
__device__ __forceinline__ void rotate_vector(float (&x)[kEPL], int j) {
  fwht_vector<D>(x, j);
  const float c = rotation_constant(D);
#pragma unroll
  for (int i = 0; i < kEPL; ++i) x[i] = __fmul_rn(x[i], c);
}

// ---------------------------------------------------------------------------
// dequantisation
// ---------------------------------------------------------------------------

template <int BITS>
__device__ __forceinline__ void decode_lane(const uint8_t* __restrict__ codes,
                                            const __half2* __restrict__ params, int j,
                                            float (&x)[kEPL]) {
  const __half2 p = params[j >> 2];
  const float s = __low2float(p);
  const float z = __high2float(p);
  uint32_t w[4];
  if (BITS == 2) {
    w[0] = *reinterpret_cast<const uint32_t*>(codes + j * 4);
#pragma unroll
    for (int i = 0; i < kEPL; ++i) x[i] = __fmaf_rn(static_cast<float>((w[0] >> (2 * i)) & 3u), s, z);
  } else if (BITS == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(codes + j * 8);
    w[0] = u.x;
    w[1] = u.y;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      x[i] = __fmaf_rn(static_cast<float>((w[0] >> (4 * i)) & 15u), s, z);
      x[8 + i] = __fmaf_rn(static_cast<float>((w[1] >> (4 * i)) & 15u), s, z);
    }
  } else {
    const uint4 u = *reinterpret_cast<const uint4*>(codes + j * 16);
    w[0] = u.x;
    w[1] = u.y;
    w[2] = u.z;
    w[3] = u.w;
#pragma unroll
    for (int i = 0; i < kEPL; ++i)
      x[i] = __fmaf_rn(static_cast<float>((w[i / 4] >> (8 * (i % 4))) & 255u), s, z);
  }
}

// The lane's 16 E4M3 bytes as binary32 (every E4M3 value is exact in fp16).
__device__ __forceinline__ void decode_fp8_lane(const uint8_t* __restrict__ codes, int j, float (&x)[kEPL]) {
  const uint4 u = *reinterpret_cast<const uint4*>(codes + j * kEPL);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
        static_cast<__nv_fp8x2_storage_t>(w[i / 2] >> (16 * (i % 2))), __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}

template <typename OutT>
__device__ __forceinline__ void store16(OutT* dst, const float (&x)[kEPL]);
template <>
__device__ __forceinline__ void store16<float>(float* dst, const float (&x)[kEPL]) {
  float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) d[i] = make_float4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3]);
}
template <>
__device__ __forceinline__ void store16<__half>(__half* dst, const float (&x)[kEPL]) {
  __align__(16) __half h[kEPL];
#pragma unroll
  for (int i = 0; i < kEPL; ++i) h[i] = __float2half_rn(x[i]);
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = reinterpret_cast<const uint4*>(h)[0];
  d[1] = reinterpret_cast<const uint4*>(h)[1];
}

template <int D, typename OutT>
__global__ void __launch_bounds__(256) dequantize_kernel(PoolView pool,
                                                         const int32_t* __restrict__ block_ids,
                                                         OutT* __restrict__ k_out,
                                                         OutT* __restrict__ v_out, int unrotate_k,
                                                         int64_t n_items) {
  using S = Shape<D>;
  const int lane = threadIdx.x & 31;
  const int r = lane / S::LPV;
  const int j = lane % S::LPV;
  const int hkv = pool.n_kv_heads;
  constexpr int kQuads = kBlockTokens / S::VPW;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;

  for (int64_t item = warp0; item < n_items; item += n_warps) {
    // item = ((list index * Hkv) + head) * kQuads + quad
    const int quad = static_cast<int>(item % kQuads);
    const int64_t bh = item / kQuads;
    const int h = static_cast<int>(bh % hkv);
    const int64_t li = bh / hkv;
    const int slot = quad * S::VPW + r;
    const int64_t out_row = (li * hkv + h) * kBlockTokens + slot;
    OutT* kd = k_out + out_row * D + j * kEPL;
    OutT* vd = v_out + out_row * D + j * kEPL;
    const int32_t blk = __ldg(block_ids + li);
    float x[kEPL];
    if (blk < 0 || blk >= pool.n_blocks()) {
      if (lane == 0) raise_error(pool.error_word, Q4KV_DEVERR_BLOCK_ID);
#pragma unroll
      for (int i = 0; i < kEPL; ++i) x[i] = 0.0f;
      store16<OutT>(kd, x);
      store16<OutT>(vd, x);
      continue;
    }
    const int bits = pool.bits_of(blk);
    const bool is8 = bits == 8, is2 = bits == 2;
    const int64_t phys = bits == 4 ? blk : (is8 ? blk - pool.n_q4 : blk - pool.n_q4 - pool.n_q8);
    const int64_t row = (phys * hkv + h) * kBlockTokens + slot;
    const bool masked =
        (pool.mask[static_cast<int64_t>(blk) * kMaskWords + slot / 32] >> (slot % 32)) & 1u;

    if (pool.fp8)
      decode_fp8_lane(pool.k_codes8 + row * D, j, x);
    else if (is8)
      decode_lane<8>(pool.k_codes8 + row * D, pool.k_params8 + row * S::NG, j, x);
    else if (is2)
      decode_lane<2>(pool.k_codes2 + row * (D / 4), pool.k_params2 + row * S::NG, j, x);
    else
      decode_lane<4>(pool.k_codes4 + row * (D / 2), pool.k_params4 + row * S::NG, j, x);
    if (unrotate_k && pool.k_rotated) rotate_vector<D>(x, j);
    if (masked) {
#pragma unroll
      for (int i = 0; i < kEPL; ++i) x[i] = Q4KV_SENTINEL_LOGIT;
    }
    store16<OutT>(kd, x);

    if (pool.fp8)
      decode_fp8_lane(pool.v_codes8 + row * D, j, x);
    else if (is8)
      decode_lane<8>(pool.v_codes8 + row * D, pool.v_params8 + row * S::NG, j, x);
    else if (is2)
      decode_lane<2>(pool.v_codes2 + row * (D / 4), pool.v_params2 + row * S::NG, j, x);
    else
      decode_lane<4>(pool.v_codes4 + row * (D / 2), pool.v_params4 + row * S::NG, j, x);
    if (masked) {
#pragma unroll
      for (int i = 0; i < kEPL; ++i) x[i] = 0.0f;
    }
    store16<OutT>(vd, x);
  }
}

// ---------------------------------------------------------------------------
// Per-token widths {2, 4, 8, FP16} in one cache: the card.  QKVShare
// (gist.science summary of arXiv 2605.03884), "Méthodologie": every token
// gets a width from {2, 4, 8, FP16}; the cache travels as a compact artifact
// of quantised groups, per-token widths and metadata, and the receiver
// rebuilds FP16 keys and values from it.  Layout (bytes): a 64-byte header,
// the widths (one byte per token, padded to 16), the int64 offset of every
// token's record from the payload start plus the total (padded to 16), then
// the records.  Record of (token, KV head h) at width w: K codes (D w / 8
// bytes), V codes, K (s, z) pairs, V (s, z) pairs -- the pool's group coding
// with L = 2^w - 1 -- or, at w = 16, the raw K row and V row.
// ---------------------------------------------------------------------------
constexpr uint32_t kCardMagic = 0x43564B51u;   // bytes 'Q', 'K', 'V', 'C'
constexpr int kCardHeader = 64;

__host__ __device__ inline int64_t card_record_bytes(int d, int w) {
  if (w == 16) return 4 * d;
  if (w == 2 || w == 4 || w == 8) return 2 * (d * w / 8 + (d / kGroup) * 4);
  return 0;
}
__host__ __device__ inline int64_t round16(int64_t x) { return (x + 15) / 16 * 16; }

__host__ __device__ inline int64_t card_payload_at(int64_t n) {
  return kCardHeader + round16(n) + round16(8 * (n + 1));
}

// The record offsets are an exclusive scan of Hkv * record bytes over the
// tokens, done in three launches with no waiting between CTAs: per-chunk
// sums (4096 tokens per CTA), one CTA scanning the chunk sums (which also
// writes the header and the table's last entry and zeroes the padding),
// then per-chunk scans from those bases, staged in shared memory so the
// table is written with coalesced stores.  The chunk sums live in the card's
// payload, which the encoder overwrites afterwards.  A width outside
// {2, 4, 8, 16} takes no bytes and raises Q4KV_DEVERR_WIDTH.
constexpr int kScanThreads = 256;
constexpr int kScanPer = 16;                              // tokens per thread
constexpr int kScanChunk = kScanThreads * kScanPer;       // tokens per CTA

__device__ __forceinline__ int64_t block_exclusive_scan(int64_t x, int64_t* warp_sums, int64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int64_t w = lane < static_cast<int>(blockDim.x >> 5) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;   // inclusive over warps
  }
  __syncthreads();
  const int64_t ex = (warp > 0 ? warp_sums[warp - 1] : 0) + incl - x;
  if (total != nullptr) *total = warp_sums[(blockDim.x >> 5) - 1];
  __syncthreads();   // warp_sums may be reused right after
  return ex;
}

__device__ __forceinline__ int64_t token_bytes(int w, int d, int hkv, uint32_t* error_word) {
  const int64_t b = hkv * card_record_bytes(d, w);
  if (b == 0) raise_error(error_word, Q4KV_DEVERR_WIDTH);
  return b;
}

__global__ void __launch_bounds__(kScanThreads) card_chunk_sums_kernel(const uint8_t* __restrict__ widths, int64_t n,
                                                                       int d, int hkv, int64_t* sums,
                                                                       uint32_t* error_word) {
  __shared__ int64_t warp_sums[32];
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kScanChunk + threadIdx.x * kScanPer;
  int64_t sum = 0;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i)
    if (t0 + i < n) sum += token_bytes(widths[t0 + i], d, hkv, error_word);
  int64_t total;
  block_exclusive_scan(sum, warp_sums, &total);
  if (threadIdx.x == 0) sums[blockIdx.x] = total;
}

// One CTA: chunk sums -> exclusive chunk bases (in place), then the header,
// the table's last entry (the payload size) and the zero padding.
__global__ void __launch_bounds__(1024) card_chunk_scan_kernel(int64_t* sums, int64_t n_chunks, int64_t n, int d,
                                                               int hkv, int k_rotated, int raw_dtype, uint8_t* card) {
  __shared__ int64_t warp_sums[32];
  __shared__ int64_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int64_t base = 0; base < n_chunks; base += blockDim.x) {
    const int64_t c = base + threadIdx.x;
    const int64_t x = c < n_chunks ? sums[c] : 0;
    int64_t total;
    const int64_t ex = block_exclusive_scan(x, warp_sums, &total);
    if (c < n_chunks) sums[c] = carry + ex;
    __syncthreads();
    if (threadIdx.x == 0) carry += total;
    __syncthreads();
  }
  uint8_t* wdst = card + kCardHeader;
  uint8_t* otab = card + kCardHeader + round16(n);
  // padding after the widths and after the offsets is zero, so a card's bytes
  // depend on its contents only
  if (threadIdx.x < 16 && n + threadIdx.x < round16(n)) wdst[n + threadIdx.x] = 0;
  if (threadIdx.x < 16 && 8 * (n + 1) + threadIdx.x < round16(8 * (n + 1))) otab[8 * (n + 1) + threadIdx.x] = 0;
  if (threadIdx.x == 0) {
    reinterpret_cast<int64_t*>(otab)[n] = carry;
    uint32_t* h = reinterpret_cast<uint32_t*>(card);
    h[0] = kCardMagic;
    h[1] = 1;   // version
    h[2] = static_cast<uint32_t>(d);
    h[3] = static_cast<uint32_t>(hkv);
    h[4] = static_cast<uint32_t>(n & 0xFFFFFFFF);
    h[5] = static_cast<uint32_t>(n >> 32);
    h[6] = static_cast<uint32_t>(k_rotated);
    h[7] = static_cast<uint32_t>(raw_dtype);
    *reinterpret_cast<int64_t*>(card + 32) = carry;
    for (int i = 40; i < kCardHeader; i += 4) *reinterpret_cast<uint32_t*>(card + i) = 0;
  }
}

// Per chunk: the widths copied into the card and the record offsets, from
// the chunk's base.
__global__ void __launch_bounds__(kScanThreads) card_offsets_kernel(const uint8_t* __restrict__ widths, int64_t n,
                                                                    int d, int hkv, const int64_t* bases,
                                                                    uint8_t* card) {
  __shared__ int64_t warp_sums[32];
  __shared__ int64_t stage[kScanChunk];
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kScanChunk;
  const int64_t t0 = c0 + threadIdx.x * kScanPer;
  int w[kScanPer];
  int64_t sum = 0;
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    w[i] = t0 + i < n ? widths[t0 + i] : 0;
    sum += hkv * card_record_bytes(d, w[i]);
  }
  int64_t run = bases[blockIdx.x] + block_exclusive_scan(sum, warp_sums, nullptr);
#pragma unroll
  for (int i = 0; i < kScanPer; ++i) {
    stage[threadIdx.x * kScanPer + i] = run;
    run += hkv * card_record_bytes(d, w[i]);
  }
  uint8_t* wdst = card + kCardHeader;
  if (t0 + kScanPer <= n) {   // 16 widths as one aligned 16-byte store
    uint32_t q[4] = {0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < kScanPer; ++i) q[i / 4] |= static_cast<uint32_t>(w[i]) << (8 * (i % 4));
    *reinterpret_cast<uint4*>(wdst + t0) = make_uint4(q[0], q[1], q[2], q[3]);
  } else {
    for (int i = 0; i < kScanPer && t0 + i < n; ++i) wdst[t0 + i] = static_cast<uint8_t>(w[i]);
  }
  __syncthreads();
  int64_t* otab = reinterpret_cast<int64_t*>(card + kCardHeader + round16(n));
  const int64_t cnt = min(static_cast<int64_t>(kScanChunk), n - c0);
  for (int64_t i = threadIdx.x; i < cnt; i += kScanThreads) otab[c0 + i] = stage[i];
}


// Warp item = (token, VPW KV heads): every lane of a warp works on one token,
// so its width is warp-uniform; the lane layout, rotation and coding are the
// append kernel's.
template <int D, typename InT>
__global__ void __launch_bounds__(256) card_encode_kernel(const InT* __restrict__ k, const InT* __restrict__ v,
                                                          int64_t n, int64_t stride, int hkv, int k_rotated,
                                                          uint8_t* card) {
  using S = Shape<D>;
  const int lane = threadIdx.x & 31;
  const int r = lane / S::LPV, j = lane % S::LPV;
  const int hgroups = (hkv + S::VPW - 1) / S::VPW;
  const int64_t* offs = reinterpret_cast<const int64_t*>(card + kCardHeader + round16(n));
  uint8_t* payload = card + card_payload_at(n);
  const int64_t n_items = n * hgroups;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t item = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; item < n_items;
       item += n_warps) {
    const int64_t t = item / hgroups;
    const int hg = static_cast<int>(item % hgroups);
    const int w = card[kCardHeader + t];
    const int64_t rec = card_record_bytes(D, w);
    if (rec == 0) continue;   // warp-uniform; reported by the layout kernel
    const int h = hg * S::VPW + r;
    const bool valid = h < hkv;
    const int hs = valid ? h : hkv - 1;   // lanes past the last head read a real row, store nothing
    const int64_t src = t * stride + static_cast<int64_t>(hs) * D + j * kEPL;
    const uint4 k0 = __ldg(reinterpret_cast<const uint4*>(k + src));
    const uint4 k1 = __ldg(reinterpret_cast<const uint4*>(k + src) + 1);
    const uint4 v0 = __ldg(reinterpret_cast<const uint4*>(v + src));
    const uint4 v1 = __ldg(reinterpret_cast<const uint4*>(v + src) + 1);
    uint8_t* dst = payload + offs[t] + static_cast<int64_t>(hs) * rec;
    if (w == 16) {   // raw 16-bit rows
      if (valid) {
        uint4* kd = reinterpret_cast<uint4*>(dst + j * 32);
        uint4* vd = reinterpret_cast<uint4*>(dst + 2 * D + j * 32);
        kd[0] = k0;
        kd[1] = k1;
        vd[0] = v0;
        vd[1] = v1;
      }
      continue;
    }
    float2 xk[8], xv[8];
    unpack16<InT>(k0, k1, xk);
    unpack16<InT>(v0, v1, xv);
    float ks = 1.0f;
    if (k_rotated) {   // warp-uniform
      rotate_pairs<D>(xk, j);
      ks = kRotScale<D>;
    }
    const int64_t cb = D * w / 8;
    __half2* kp = reinterpret_cast<__half2*>(dst + 2 * cb);
    __half2* vp = kp + S::NG;
    if (w == 2) encode_kv<2>(xk, ks, xv, j, valid, dst, kp, dst + cb, vp);
    else if (w == 4) encode_kv<4>(xk, ks, xv, j, valid, dst, kp, dst + cb, vp);
    else encode_kv<8>(xk, ks, xv, j, valid, dst, kp, dst + cb, vp);
  }
}

// Card -> K_hat, V_hat [n][Hkv][D]: x_hat = fl(code s + z), K un-rotated when
// the card stores it rotated; FP16 tokens convert exactly; a token of an
// invalid width reads 0.  The header must describe (D, Hkv, n) and every
// record must lie inside the card's `card_bytes`, else the rows read 0 and
// Q4KV_DEVERR_IMAGE is raised: a damaged card is never read out of bounds.
__device__ __forceinline__ float raw16_to_float(uint16_t b, bool bf16) {
  return bf16 ? __uint_as_float(static_cast<uint32_t>(b) << 16) : __half2float(__ushort_as_half(b));
}

template <int D, typename OutT>
__global__ void __launch_bounds__(256) card_decode_kernel(const uint8_t* card, int64_t card_bytes, int64_t n,
                                                          int hkv, OutT* __restrict__ k_out,
                                                          OutT* __restrict__ v_out, uint32_t* error_word) {
  using S = Shape<D>;
  const int lane = threadIdx.x & 31;
  const int r = lane / S::LPV, j = lane % S::LPV;
  const int hgroups = (hkv + S::VPW - 1) / S::VPW;
  const uint32_t* hdr = reinterpret_cast<const uint32_t*>(card);
  const bool header_ok = hdr[0] == kCardMagic && hdr[1] == 1u && hdr[2] == static_cast<uint32_t>(D) &&
                         hdr[3] == static_cast<uint32_t>(hkv) &&
                         (static_cast<int64_t>(hdr[5]) << 32 | hdr[4]) == n;
  const bool k_rotated = hdr[6] != 0, raw_bf16 = hdr[7] != 0;
  const uint8_t* widths = card + kCardHeader;
  const int64_t* offs = reinterpret_cast<const int64_t*>(card + kCardHeader + round16(n));
  const uint8_t* payload = card + card_payload_at(n);
  const int64_t room = card_bytes - card_payload_at(n);
  const int64_t n_items = n * hgroups;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t item = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; item < n_items;
       item += n_warps) {
    const int64_t t = item / hgroups;
    const int hg = static_cast<int>(item % hgroups);
    const int h = hg * S::VPW + r;
    const bool valid = h < hkv;
    const int hs = valid ? h : hkv - 1;
    OutT* kd = k_out + (t * hkv + hs) * D + j * kEPL;
    OutT* vd = v_out + (t * hkv + hs) * D + j * kEPL;
    int w = 0;
    int64_t rec = 0, off = 0;
    if (header_ok) {
      w = widths[t];
      rec = card_record_bytes(D, w);
      off = offs[t];
      if (rec != 0 && (off < 0 || off + hkv * rec > room)) {   // warp-uniform
        if (lane == 0) raise_error(error_word, Q4KV_DEVERR_IMAGE);
        rec = 0;
      }
    } else if (item == 0 && lane == 0) {
      raise_error(error_word, Q4KV_DEVERR_IMAGE);
    }
    const uint8_t* src = payload + off + static_cast<int64_t>(hs) * rec;
    float xk[kEPL], xv[kEPL];
    if (rec == 0) {
#pragma unroll
      for (int i = 0; i < kEPL; ++i) xk[i] = xv[i] = 0.0f;
    } else if (w == 16) {
      const uint4* rk = reinterpret_cast<const uint4*>(src + j * 32);
      const uint4* rv = reinterpret_cast<const uint4*>(src + 2 * D + j * 32);
      const uint4 a[2] = {rk[0], rk[1]}, b[2] = {rv[0], rv[1]};
      const uint16_t* ka = reinterpret_cast<const uint16_t*>(a);
      const uint16_t* vb = reinterpret_cast<const uint16_t*>(b);
#pragma unroll
      for (int i = 0; i < kEPL; ++i) {
        xk[i] = raw16_to_float(ka[i], raw_bf16);
        xv[i] = raw16_to_float(vb[i], raw_bf16);
      }
    } else {
      const int64_t cb = D * w / 8;
      const __half2* kp = reinterpret_cast<const __half2*>(src + 2 * cb);
      const __half2* vp = kp + S::NG;
      if (w == 2) {
        decode_lane<2>(src, kp, j, xk);
        decode_lane<2>(src + cb, vp, j, xv);
      } else if (w == 4) {
        decode_lane<4>(src, kp, j, xk);
        decode_lane<4>(src + cb, vp, j, xv);
      } else {
        decode_lane<8>(src, kp, j, xk);
        decode_lane<8>(src + cb, vp, j, xv);
      }
      if (k_rotated) rotate_vector<D>(xk, j);   // warp-uniform
    }
    if (valid) {
      store16<OutT>(kd, xk);
      store16<OutT>(vd, xv);
    }
  }
}

inline int grid_for(int64_t n_items) {
  const int64_t warps_per_cta = 8;
  int64_t g = (n_items + warps_per_cta - 1) / warps_per_cta;
  if (g > (1 << 30)) g = 1 << 30;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_quantize(const PoolView& pool, const void* k, const void* v, int in_dtype,
                            int64_t n_tokens, int64_t token_stride, const int32_t* block_ids,
                            cudaStream_t stream) {
  const int d = pool.head_dim, hkv = pool.n_kv_heads;
  if (n_tokens >= (int64_t{1} << 31)) return cudaErrorInvalidValue;
  // a unit holds T tokens x H' heads with T * H' * D = 8192 elements (16 KB of
  // 16-bit input per tensor): H' the largest power of two <= Hkv that leaves
  // T >= VPW, so a full unit is 16 warp items
  const int vpw = d == 128 ? Shape<128>::VPW : Shape<256>::VPW;
  const int per_unit = 8192 / d;   // T * H'
  int hp = 1;
  while (hp * 2 <= hkv && per_unit / (hp * 2) >= vpw) hp *= 2;
  EncodeGeometry geo;
  geo.n_tokens = static_cast<uint32_t>(n_tokens);
  geo.stride = token_stride;
  geo.unit_tokens = per_unit / hp;
  geo.unit_heads = hp;
  geo.head_chunks = (hkv + hp - 1) / hp;
  geo.items_per_head_log2 = 0;
  while ((vpw << (geo.items_per_head_log2 + 1)) <= geo.unit_tokens) ++geo.items_per_head_log2;
  const int64_t n_chunks = (n_tokens + geo.unit_tokens - 1) / geo.unit_tokens;
  geo.n_chunks = static_cast<uint32_t>(n_chunks);
  const int sms = device_sm_count() > 0 ? device_sm_count() : 148;
  const int64_t grid = n_chunks < sms ? n_chunks : sms;
  const size_t smem = kQStages * kQStageBytes + (kQFull + kQStages) * sizeof(uint64_t);
  cudaError_t e = cudaSuccess;
#define Q4KV_LAUNCH_Q(DD, T, R, M, ...)                                                              \
  do {                                                                                                 \
    e = cudaFuncSetAttribute(quantize_kernel<DD, T, R, M, ##__VA_ARGS__>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             static_cast<int>(smem));                                                  \
    if (e == cudaSuccess)                                                                              \
      e = launch_pdl(quantize_kernel<DD, T, R, M, ##__VA_ARGS__>, dim3(static_cast<unsigned>(grid)), dim3(kQThreads),  \
                     smem, stream, pool, static_cast<const T*>(k), static_cast<const T*>(v), geo,        \
                     block_ids);                                                                       \
  } while (0)
#define Q4KV_LAUNCH_QR(DD, T)                                   \
  do {                                                          \
    const bool mixed = pool.n_q8 > 0 || pool.n_q2 > 0;          \
    if (pool.k_rotated && mixed) Q4KV_LAUNCH_Q(DD, T, true, true);        \
    else if (pool.k_rotated) Q4KV_LAUNCH_Q(DD, T, true, false);           \
    else if (mixed) Q4KV_LAUNCH_Q(DD, T, false, true);                    \
    else Q4KV_LAUNCH_Q(DD, T, false, false);                              \
  } while (0)
  if (n_chunks == 0) return cudaSuccess;
  if (pool.fp8) {   // FP8 pools: raw keys, every block 8-bit
    if (d == 128 && in_dtype == Q4KV_F16) Q4KV_LAUNCH_Q(128, __half, false, true, true);
    else if (d == 128) Q4KV_LAUNCH_Q(128, __nv_bfloat16, false, true, true);
    else if (in_dtype == Q4KV_F16) Q4KV_LAUNCH_Q(256, __half, false, true, true);
    else Q4KV_LAUNCH_Q(256, __nv_bfloat16, false, true, true);
    return e;
  }
  if (d == 128 && in_dtype == Q4KV_F16) Q4KV_LAUNCH_QR(128, __half);
  else if (d == 128) Q4KV_LAUNCH_QR(128, __nv_bfloat16);
  else if (in_dtype == Q4KV_F16) Q4KV_LAUNCH_QR(256, __half);
  else Q4KV_LAUNCH_QR(256, __nv_bfloat16);
#undef Q4KV_LAUNCH_QR
#undef Q4KV_LAUNCH_Q
  return e;
}

cudaError_t launch_append(const PoolView& pool, const void* k, const void* v, int in_dtype,
                          int32_t batch, int32_t max_new, const int32_t* n_new, int64_t seq_stride,
                          int64_t token_stride, const int32_t* tables, int32_t max_blocks,
                          const int32_t* seq_lens, cudaStream_t stream) {
  const int d = pool.head_dim;
  const int vpw = d == 128 ? Shape<128>::VPW : Shape<256>::VPW;
  const int64_t items = static_cast<int64_t>(batch) * max_new * ((pool.n_kv_heads + vpw - 1) / vpw);
  if (items == 0) return cudaSuccess;
  const int sms = device_sm_count() > 0 ? device_sm_count() : 148;
  int64_t g = (items + 7) / 8;                   // 8 warps per CTA
  if (g > static_cast<int64_t>(sms) * 8) g = static_cast<int64_t>(sms) * 8;
  const dim3 grid(static_cast<unsigned>(g)), block(256);
#define Q4KV_LAUNCH_A(DD, T, R)                                                                     \
  return launch_pdl(append_kernel<DD, T, R>, grid, block, 0, stream, pool, static_cast<const T*>(k), \
                    static_cast<const T*>(v), batch, max_new, n_new, seq_stride, token_stride,        \
                    tables, max_blocks, seq_lens)
#define Q4KV_LAUNCH_AR(DD, T)       \
  if (pool.k_rotated) {             \
    Q4KV_LAUNCH_A(DD, T, true);     \
  } else {                          \
    Q4KV_LAUNCH_A(DD, T, false);    \
  }
  if (d == 128 && in_dtype == Q4KV_F16) { Q4KV_LAUNCH_AR(128, __half) }
  if (d == 128) { Q4KV_LAUNCH_AR(128, __nv_bfloat16) }
  if (in_dtype == Q4KV_F16) { Q4KV_LAUNCH_AR(256, __half) }
  Q4KV_LAUNCH_AR(256, __nv_bfloat16)
#undef Q4KV_LAUNCH_AR
#undef Q4KV_LAUNCH_A
}

int64_t card_max_bytes(int d, int hkv, int64_t n) { return card_payload_at(n) + n * hkv * 4 * d; }

cudaError_t launch_card_encode(int d, int hkv, int k_rotated, const void* k, const void* v, int in_dtype,
                               int64_t n, int64_t stride, const uint8_t* widths, uint8_t* card,
                               uint32_t* error_word, cudaStream_t stream) {
  // record offsets: chunk sums, their scan (with the header), then the table
  const int64_t n_chunks = (n + kScanChunk - 1) / kScanChunk;
  int64_t* sums = reinterpret_cast<int64_t*>(card + card_payload_at(n));   // scratch in the payload
  if (n_chunks > 0)
    card_chunk_sums_kernel<<<static_cast<unsigned>(n_chunks), kScanThreads, 0, stream>>>(widths, n, d, hkv, sums,
                                                                                          error_word);
  card_chunk_scan_kernel<<<1, 1024, 0, stream>>>(sums, n_chunks, n, d, hkv, k_rotated, in_dtype == Q4KV_BF16, card);
  if (n_chunks > 0)
    card_offsets_kernel<<<static_cast<unsigned>(n_chunks), kScanThreads, 0, stream>>>(widths, n, d, hkv, sums, card);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || n == 0) return e;
  const int vpw = d == 128 ? Shape<128>::VPW : Shape<256>::VPW;
  const int64_t items = n * ((hkv + vpw - 1) / vpw);
  const int sms = device_sm_count() > 0 ? device_sm_count() : 148;
  int64_t g = (items + 7) / 8;
  if (g > static_cast<int64_t>(sms) * 8) g = static_cast<int64_t>(sms) * 8;
#define Q4KV_CARD_E(DD, T)                                                                            \
  card_encode_kernel<DD, T><<<static_cast<unsigned>(g), 256, 0, stream>>>(                          \
      static_cast<const T*>(k), static_cast<const T*>(v), n, stride, hkv, k_rotated, card)
  if (d == 128 && in_dtype == Q4KV_F16) Q4KV_CARD_E(128, __half);
  else if (d == 128) Q4KV_CARD_E(128, __nv_bfloat16);
  else if (in_dtype == Q4KV_F16) Q4KV_CARD_E(256, __half);
  else Q4KV_CARD_E(256, __nv_bfloat16);
#undef Q4KV_CARD_E
  return cudaGetLastError();
}

cudaError_t launch_card_decode(int d, int hkv, const uint8_t* card, int64_t card_bytes, int64_t n, void* k_out,
                               void* v_out, int out_dtype, uint32_t* error_word, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int vpw = d == 128 ? Shape<128>::VPW : Shape<256>::VPW;
  const dim3 grid(grid_for(n * ((hkv + vpw - 1) / vpw))), block(256);
#define Q4KV_CARD_D(DD, T)                                                                            \
  card_decode_kernel<DD, T><<<grid, block, 0, stream>>>(card, card_bytes, n, hkv, static_cast<T*>(k_out), \
                                                        static_cast<T*>(v_out), error_word)
  if (d == 128 && out_dtype == Q4KV_F32) Q4KV_CARD_D(128, float);
  else if (d == 128) Q4KV_CARD_D(128, __half);
  else if (out_dtype == Q4KV_F32) Q4KV_CARD_D(256, float);
  else Q4KV_CARD_D(256, __half);
#undef Q4KV_CARD_D
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const PoolView& pool, const int32_t* block_ids, int32_t n_blocks,
                              void* k_out, void* v_out, int out_dtype, int unrotate_k,
                              cudaStream_t stream) {
  const int d = pool.head_dim;
  const int vpw = d == 128 ? Shape<128>::VPW : Shape<256>::VPW;
  const int64_t n_items = static_cast<int64_t>(n_blocks) * pool.n_kv_heads * (kBlockTokens / vpw);
  const dim3 grid(grid_for(n_items)), block(256);
#define Q4KV_LAUNCH_D(DD, T)                                                            \
  dequantize_kernel<DD, T><<<grid, block, 0, stream>>>(pool, block_ids, static_cast<T*>(k_out), \
                                                       static_cast<T*>(v_out), unrotate_k, n_items)
  if (d == 128 && out_dtype == Q4KV_F32) Q4KV_LAUNCH_D(128, float);
  else if (d == 128) Q4KV_LAUNCH_D(128, __half);
  else if (out_dtype == Q4KV_F32) Q4KV_LAUNCH_D(256, float);
  else Q4KV_LAUNCH_D(256, __half);
#undef Q4KV_LAUNCH_D
  return cudaGetLastError();
}

}  // namespace q4kv
