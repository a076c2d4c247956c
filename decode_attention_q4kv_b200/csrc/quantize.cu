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
#include "q4kv_internal.cuh"

namespace q4kv {
namespace {

constexpr int kEPL = 16;  // channels held by one lane

template <int D>
struct Shape {
  static constexpr int LPV = D / kEPL;        // lanes per vector
  static constexpr int VPW = 32 / LPV;        // vectors (tokens) per warp
  static constexpr int NG = D / kGroup;       // groups per vector
};

// ---------------------------------------------------------------------------
// Encoder.  A lane holds its 16 channels as 8 packed pairs: pair p = channels
// (p, p + 8) of the lane's run, so the butterflies of strides 1, 2 and 4 pair
// whole registers and run as packed f32x2 operations; stride 8 works inside a
// pair.  Every packed operation is two independent binary32 operations with
// round-to-nearest-even, identical to the scalar ones.
// ---------------------------------------------------------------------------

__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {   // a - b
  return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}

template <int D>
__device__ __forceinline__ void fwht_pairs(float2 (&x)[8], int j) {
  // stride 1, 2, 4: register pairs p and p + h (bit h of p clear)
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      if ((p & h) == 0) {
        const float2 a = x[p], b = x[p + h];
        x[p] = add2(a, b);
        x[p + h] = sub2(a, b);
      }
    }
  }
  // stride 8: channels p and p + 8 share a register pair
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const float a = x[p].x, b = x[p].y;
    x[p].x = __fadd_rn(a, b);
    x[p].y = __fsub_rn(a, b);
  }
  // strides 16 .. D/2: across lanes; fma(own, +-1, other) = other +- own exactly
#pragma unroll
  for (int h = kEPL; h < D; h <<= 1) {
    const int lane_bit = h / kEPL;
    const float sg = (j & lane_bit) ? -1.0f : 1.0f;
    const float2 sgn = make_float2(sg, sg);
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      float2 o;
      o.x = __shfl_xor_sync(0xffffffffu, x[p].x, lane_bit);
      o.y = __shfl_xor_sync(0xffffffffu, x[p].y, lane_bit);
      x[p] = __ffma2_rn(x[p], sgn, o);
    }
  }
}

template <int D>
__device__ __forceinline__ void rotate_pairs(float2 (&x)[8], int j) {
  fwht_pairs<D>(x, j);
  const float c = rotation_constant(D);
#pragma unroll
  for (int p = 0; p < 8; ++p) x[p] = __fmul2_rn(x[p], make_float2(c, c));
}

template <typename T>
__device__ __forceinline__ void unpack16(const uint4& w0, const uint4& w1, float2 (&x)[8]) {
  static_assert(sizeof(T) == 2, "16-bit inputs");
  const T* e0 = reinterpret_cast<const T*>(&w0);
  const T* e1 = reinterpret_cast<const T*>(&w1);
#pragma unroll
  for (int p = 0; p < 8; ++p) x[p] = make_float2(to_float<T>(e0[p]), to_float<T>(e1[p]));
}

__device__ __forceinline__ float min3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 1.5 * 2^23: adding it rounds |y| < 2^22 to an integer (ties to even) held in
// the low mantissa bits.
constexpr float kRoundMagic = 12582912.0f;

// Encode the lane's 16 values (one quarter of a 64-value group) and store its
// codes and, from the group's first lane, the group's (scale, zero).
//
// Codes are defined as clamp(rne(fl(fl(x - z) / s)), 0, L).  Fast path:
// y = fl(x * r + (-z * r)) with r = fl(1/s), then k = rne(y).  With
// |y - fl(fl(x - z)/s)| <= B = (4 (L + 1) + |z r|) 2^-24, k is the defined
// code whenever y lies more than 2B away from a half-integer.  The fast path
// is taken for a group only when |z r| <= 2^10 (so B < 2^-13) and every
// value's quotient stays inside [-0.49, L + 0.49] (so no clamp is needed);
// a lane whose values come within 2^-13 (4-bit) or 2^-12 (8-bit) of a
// half-integer recomputes its codes with IEEE division.  Either way the codes
// equal the definition.
template <int BITS>
__device__ __forceinline__ void encode_store(const float2 (&x)[8], int j, bool valid,
                                             uint8_t* __restrict__ code_dst,
                                             __half2* __restrict__ param_dst) {
  constexpr int L = (1 << BITS) - 1;
  float mn = min3(min3(min3(x[0].x, x[0].y, x[1].x), min3(x[1].y, x[2].x, x[2].y),
                       min3(x[3].x, x[3].y, x[4].x)),
                  min3(x[4].y, x[5].x, x[5].y), min3(x[6].x, x[6].y, min(x[7].x, x[7].y)));
  float mx = max3(max3(max3(x[0].x, x[0].y, x[1].x), max3(x[1].y, x[2].x, x[2].y),
                       max3(x[3].x, x[3].y, x[4].x)),
                  max3(x[4].y, x[5].x, x[5].y), max3(x[6].x, x[6].y, max(x[7].x, x[7].y)));
  // the 4 lanes of a group are j = 4k .. 4k+3
  mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 2));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  mn = __fadd_rn(mn, 0.0f);  // -0 -> +0
  mx = __fadd_rn(mx, 0.0f);
  const float s = __fdiv_rn(__fsub_rn(mx, mn), static_cast<float>(L));
  const __half sh = __float2half_rn(s);
  const __half zh = __float2half_rn(mn);
  const float sf = __half2float(sh);
  const float zf = __half2float(zh);

  uint32_t q[kEPL];   // code e in the low bits of q[e]; lane element e = pair e%8, half e/8
  bool exact = true;
  if (sf != 0.0f) {
    const float r = __frcp_rn(sf);
    const float nzr = __fmul_rn(-zf, r);
    const float t_lo = __fmaf_rn(mn, r, nzr), t_hi = __fmaf_rn(mx, r, nzr);
    exact = fabsf(nzr) > 1024.0f || t_lo < -0.49f || t_hi > L + 0.49f;
    if (!exact) {
      constexpr float thr = 0.5f - (BITS == 4 ? 0x1p-13f : 0x1p-12f);
      const float2 r2 = make_float2(r, r), n2 = make_float2(nzr, nzr);
      const float2 m2 = make_float2(kRoundMagic, kRoundMagic);
      const float2 mm2 = make_float2(-kRoundMagic, -kRoundMagic);
      const float2 t2 = make_float2(-thr * thr, -thr * thr);
      uint32_t all_neg = 0xffffffffu;
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const float2 y = __ffma2_rn(x[p], r2, n2);
        const float2 yk = __fadd2_rn(y, m2);        // integer in the low bits
        const float2 k = __fadd2_rn(yk, mm2);       // that integer as a float
        const float2 d = sub2(y, k);                // distance to it, |d| <= 0.5
        const float2 e = __ffma2_rn(d, d, t2);      // < 0 iff |d| < thr
        all_neg &= __float_as_uint(e.x) & __float_as_uint(e.y);
        q[p] = __float_as_uint(yk.x);
        q[p + 8] = __float_as_uint(yk.y);
      }
      exact = (all_neg >> 31) == 0;
    }
    if (exact) {
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        int r0 = __float2int_rn(__fdiv_rn(__fsub_rn(x[p].x, zf), sf));
        int r1 = __float2int_rn(__fdiv_rn(__fsub_rn(x[p].y, zf), sf));
        q[p] = static_cast<uint32_t>(min(max(r0, 0), L));
        q[p + 8] = static_cast<uint32_t>(min(max(r1, 0), L));
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < kEPL; ++e) q[e] = 0;
  }
  if (!valid) return;
  if (BITS == 4) {
    // byte b holds elements 2b (low nibble) and 2b+1 (high nibble)
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) b[i] = (q[2 * i] & 15u) | ((q[2 * i + 1] & 15u) << 4);
    const uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
    *reinterpret_cast<uint2*>(code_dst + j * 8) = make_uint2(lo, hi);
  } else {
    uint4 w;
    w.x = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
    w.y = __byte_perm(__byte_perm(q[4], q[5], 0x0040), __byte_perm(q[6], q[7], 0x0040), 0x5410);
    w.z = __byte_perm(__byte_perm(q[8], q[9], 0x0040), __byte_perm(q[10], q[11], 0x0040), 0x5410);
    w.w = __byte_perm(__byte_perm(q[12], q[13], 0x0040), __byte_perm(q[14], q[15], 0x0040), 0x5410);
    *reinterpret_cast<uint4*>(code_dst + j * 16) = w;
  }
  if ((j & 3) == 0) param_dst[j >> 2] = __halves2half2(sh, zh);
}

// One warp item = (group of VPW consecutive tokens, KV head).  Items are
// walked with a grid stride; the next item's K/V rows are loaded before the
// current one is encoded, so every warp keeps two items of loads in flight.
template <typename InT>
struct ItemLoad {
  uint4 k0, k1, v0, v1;
  int32_t blk;
};

template <int D, typename InT>
__device__ __forceinline__ void load_item(uint32_t item, uint32_t hkv, int r, int j, uint32_t n_tokens,
                                          int64_t stride, const InT* __restrict__ k,
                                          const InT* __restrict__ v,
                                          const int32_t* __restrict__ block_ids, ItemLoad<InT>& L) {
  using S = Shape<D>;
  const uint32_t grp = item / hkv, h = item - grp * hkv;
  const uint32_t t0 = grp * S::VPW, t = t0 + r;
  L.blk = __ldg(block_ids + t0 / kBlockTokens);
  L.k0 = L.k1 = L.v0 = L.v1 = make_uint4(0, 0, 0, 0);
  if (t < n_tokens) {
    const int64_t src = static_cast<int64_t>(t) * stride + h * D + j * kEPL;
    L.k0 = __ldg(reinterpret_cast<const uint4*>(k + src));
    L.k1 = __ldg(reinterpret_cast<const uint4*>(k + src) + 1);
    L.v0 = __ldg(reinterpret_cast<const uint4*>(v + src));
    L.v1 = __ldg(reinterpret_cast<const uint4*>(v + src) + 1);
  }
}

template <int D, typename InT>
__global__ void __launch_bounds__(256, 2) quantize_kernel(PoolView pool, const InT* __restrict__ k,
                                                          const InT* __restrict__ v,
                                                          uint32_t n_tokens, int64_t stride,
                                                          const int32_t* __restrict__ block_ids,
                                                          uint32_t n_items) {
  using S = Shape<D>;
  const int lane = threadIdx.x & 31;
  const int r = lane / S::LPV;
  const int j = lane % S::LPV;
  const uint32_t hkv = pool.n_kv_heads;
  const uint32_t n_warps = (gridDim.x * blockDim.x) >> 5;
  uint32_t item = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  griddep_wait();   // the inputs may come from the kernel before in the stream
  griddep_launch_dependents();
  if (item >= n_items) return;

  ItemLoad<InT> cur, nxt;
  load_item<D, InT>(item, hkv, r, j, n_tokens, stride, k, v, block_ids, cur);
  for (; item < n_items; item += n_warps) {
    const uint32_t next = item + n_warps;
    if (next < n_items) load_item<D, InT>(next, hkv, r, j, n_tokens, stride, k, v, block_ids, nxt);

    const uint32_t grp = item / hkv, h = item - grp * hkv;
    const uint32_t t0 = grp * S::VPW, t = t0 + r;
    const bool valid = t < n_tokens;
    const int32_t blk = cur.blk;
    if (blk < 0 || blk >= pool.n_q4 + pool.n_q8) {
      if (lane == 0) raise_error(pool.error_word, Q4KV_DEVERR_BLOCK_ID);
    } else {
      const int slot = static_cast<int>(t % kBlockTokens);
      const bool is8 = blk >= pool.n_q4;
      const int64_t phys = is8 ? blk - pool.n_q4 : blk;
      const int64_t row = (phys * hkv + h) * kBlockTokens + slot;   // (block, head, slot)
      float2 x[8];
      // keys: rotate, then code
      unpack16<InT>(cur.k0, cur.k1, x);
      if (pool.k_rotated) rotate_pairs<D>(x, j);
      if (is8)
        encode_store<8>(x, j, valid, pool.k_codes8 + row * D, pool.k_params8 + row * S::NG);
      else
        encode_store<4>(x, j, valid, pool.k_codes4 + row * (D / 2), pool.k_params4 + row * S::NG);
      // values: code unrotated
      unpack16<InT>(cur.v0, cur.v1, x);
      if (is8)
        encode_store<8>(x, j, valid, pool.v_codes8 + row * D, pool.v_params8 + row * S::NG);
      else
        encode_store<4>(x, j, valid, pool.v_codes4 + row * (D / 2), pool.v_params4 + row * S::NG);
      // a freshly written slot is live
      if (valid && h == 0 && j == 0)
        atomicAnd(pool.mask + static_cast<int64_t>(blk) * kMaskWords + slot / 32,
                  ~(1u << (slot % 32)));
    }
    cur = nxt;
  }
}

// Scalar butterflies for the decoder's optional un-rotation (channels 16j ..
// 16j+15 of the lane in order); same stage order and operations as above.
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
  if (BITS == 4) {
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
    if (blk < 0 || blk >= pool.n_q4 + pool.n_q8) {
      if (lane == 0) raise_error(pool.error_word, Q4KV_DEVERR_BLOCK_ID);
#pragma unroll
      for (int i = 0; i < kEPL; ++i) x[i] = 0.0f;
      store16<OutT>(kd, x);
      store16<OutT>(vd, x);
      continue;
    }
    const bool is8 = blk >= pool.n_q4;
    const int64_t phys = is8 ? blk - pool.n_q4 : blk;
    const int64_t row = (phys * hkv + h) * kBlockTokens + slot;
    const bool masked =
        (pool.mask[static_cast<int64_t>(blk) * kMaskWords + slot / 32] >> (slot % 32)) & 1u;

    if (is8)
      decode_lane<8>(pool.k_codes8 + row * D, pool.k_params8 + row * S::NG, j, x);
    else
      decode_lane<4>(pool.k_codes4 + row * (D / 2), pool.k_params4 + row * S::NG, j, x);
    if (unrotate_k && pool.k_rotated) rotate_vector<D>(x, j);
    if (masked) {
#pragma unroll
      for (int i = 0; i < kEPL; ++i) x[i] = Q4KV_SENTINEL_LOGIT;
    }
    store16<OutT>(kd, x);

    if (is8)
      decode_lane<8>(pool.v_codes8 + row * D, pool.v_params8 + row * S::NG, j, x);
    else
      decode_lane<4>(pool.v_codes4 + row * (D / 2), pool.v_params4 + row * S::NG, j, x);
    if (masked) {
#pragma unroll
      for (int i = 0; i < kEPL; ++i) x[i] = 0.0f;
    }
    store16<OutT>(vd, x);
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
  const int d = pool.head_dim;
  const int vpw = d == 128 ? Shape<128>::VPW : Shape<256>::VPW;
  const int64_t n_items = ((n_tokens + vpw - 1) / vpw) * pool.n_kv_heads;
  if (n_items >= (int64_t{1} << 32) || n_tokens >= (int64_t{1} << 32)) return cudaErrorInvalidValue;
  // two CTAs of 8 warps per SM, each warp with two items of loads in flight
  const int sms = device_sm_count();
  int64_t g = (n_items + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sms > 0 ? sms : 148) * 2;
  if (g > cap) g = cap;
  const dim3 grid(static_cast<unsigned>(g < 1 ? 1 : g)), block(256);
  const uint32_t nt = static_cast<uint32_t>(n_tokens), ni = static_cast<uint32_t>(n_items);
#define Q4KV_LAUNCH_Q(DD, T)                                                                 \
  launch_pdl(quantize_kernel<DD, T>, grid, block, 0, stream, pool, static_cast<const T*>(k), \
             static_cast<const T*>(v), nt, token_stride, block_ids, ni)
  if (d == 128 && in_dtype == Q4KV_F16) return Q4KV_LAUNCH_Q(128, __half);
  if (d == 128) return Q4KV_LAUNCH_Q(128, __nv_bfloat16);
  if (in_dtype == Q4KV_F16) return Q4KV_LAUNCH_Q(256, __half);
  return Q4KV_LAUNCH_Q(256, __nv_bfloat16);
#undef Q4KV_LAUNCH_Q
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
