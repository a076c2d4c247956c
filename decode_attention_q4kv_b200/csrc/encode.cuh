// Encoding of one (token, head) row of the paged format, shared by the
// encoder and append kernels (quantize.cu) and the decode kernel's fused
// append (decode_tc.cu).  A lane holds 16 consecutive channels of one (token,
// head) vector; the rotation runs as butterfly stages inside the lane, then
// across lanes with warp shuffles, and a 64-value group spans 4 lanes.  Every
// arithmetic step is one IEEE binary32 operation with an _rn intrinsic, in the
// defined order (see quantize.cu).
#pragma once
#include "q4kv_internal.cuh"

namespace q4kv {
namespace {

// Single-lane operations without a divergent branch: the instruction is
// predicated on the lane.
__device__ __forceinline__ void red_and_if(bool p, uint32_t* addr, uint32_t v) {
  asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %0, 0;\n @q red.global.and.b32 [%1], %2;\n}"
               :: "r"(static_cast<uint32_t>(p)), "l"(addr), "r"(v) : "memory");
}

// Stores predicated on p (one instruction each, no branch around them).
__device__ __forceinline__ void st_if(bool p, void* a, uint32_t x) {
  asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %0, 0;\n @q st.global.u32 [%1], %2;\n}"
               :: "r"(static_cast<uint32_t>(p)), "l"(a), "r"(x) : "memory");
}
__device__ __forceinline__ void st_if(bool p, void* a, uint2 x) {
  asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %0, 0;\n @q st.global.v2.u32 [%1], {%2, %3};\n}"
               :: "r"(static_cast<uint32_t>(p)), "l"(a), "r"(x.x), "r"(x.y) : "memory");
}
__device__ __forceinline__ void st_if(bool p, void* a, uint4 x) {
  asm volatile("{\n .reg .pred q;\n setp.ne.u32 q, %0, 0;\n @q st.global.v4.u32 [%1], {%2, %3, %4, %5};\n}"
               :: "r"(static_cast<uint32_t>(p)), "l"(a), "r"(x.x), "r"(x.y), "r"(x.z), "r"(x.w) : "memory");
}
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

// c * H x.  At D = 256 the constant c = 2^-4 is exact, so the multiply is
// left to the encoder (kRotScale), which folds it into its first operations
// without changing any rounding; at D = 128 it is applied here.
template <int D>
constexpr float kRotScale = D == 256 ? 0.0625f : 1.0f;

template <int D>
__device__ __forceinline__ void rotate_pairs(float2 (&x)[8], int j) {
  fwht_pairs<D>(x, j);
  if (D != 256) {
    const float c = rotation_constant(D);
#pragma unroll
    for (int p = 0; p < 8; ++p) x[p] = __fmul2_rn(x[p], make_float2(c, c));
  }
}

__device__ __forceinline__ uint4 lds16(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

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

// Correctly rounded quotient RN(u / s) for a divisor s whose significand
// has at most 11 bits (every fp16 value, and the constants 3, 15 and 255), from
// r = RN(1/s): q0 = RN(u r), the residual u - q0 s is exact under an FMA, and
// one correction q1 = RN(q0 + (u - q0 s) r) gives RN(u / s).  This is
// Markstein's correction step (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990); the quotient is checked exhaustively for every 11-bit divisor
// significand against every binary32 dividend significand (the steps scale
// exactly with the exponents), and the codes it produces are checked
// bit-exact against the oracle's IEEE division.
__device__ __forceinline__ float quot(float u, float s, float r) {
  const float q0 = __fmul_rn(u, r);
  return __fmaf_rn(__fmaf_rn(-q0, s, u), r, q0);
}

// Encoding of one lane's 16 values (a quarter of a 64-value group).
//
// Codes are defined as clamp(rne(fl(fl(x - z) / s)), 0, L): u = fl(x - z),
// then the correctly rounded quotient above, then round-half-even to an
// integer by adding 1.5 * 2^23.  The quotient is monotone in x, so when the
// group's extremes give quotients inside [-0.49, L + 0.49] (tested with the
// uncorrected product (x - z) r, off by a few ulp) no code needs the clamp;
// other groups (a zero far outside the fp16 grid of the values) are
// recomputed with IEEE division and an integer clamp.  s = 0 (a constant
// group) is handled by r = 0, which makes every quotient 0.
//
// The steps are split so that the K and V encodings of a warp item form one
// branch-free stretch of code the compiler can interleave: group statistics,
// codes, then the rare clamp path and the stores.
struct GroupParams {
  __half sh, zh;   // stored scale and zero
  float s, z, r;   // the same as binary32, and RN(1/s) (0 when s = 0)
  bool fast;       // every code of the group is rne(quotient) without a clamp
};

// x holds the values divided by xs (a power of two): every use multiplies
// by xs first, which is exact.
template <int BITS>
__device__ __forceinline__ GroupParams group_params(const float2 (&x)[8], float xs) {
  constexpr int L = (1 << BITS) - 1;
  // RN(1/L); 3, 15 and 255 have significands of at most 11 bits
  constexpr float kRecipL = BITS == 2 ? 0x1.555556p-2f : BITS == 4 ? 0x1.111112p-4f : 0x1.010102p-8f;
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
  mn = __fmaf_rn(mn, xs, 0.0f);  // exact scaling, and -0 + 0 = +0
  mx = __fmaf_rn(mx, xs, 0.0f);
  GroupParams g;
  g.sh = __float2half_rn(quot(__fsub_rn(mx, mn), static_cast<float>(L), kRecipL));
  g.zh = __float2half_rn(mn);
  g.s = __half2float(g.sh);
  g.z = __half2float(g.zh);
  g.r = g.s != 0.0f ? __frcp_rn(g.s) : 0.0f;
  // fl(x r + fl(-z r)) differs from the defined quotient by at most
  // (4 (L + 1) + |z r|) 2^-24 < 0.005 when |z r| <= 2^16, so the 0.01 margin
  // keeps the test conservative; a group it rejects just takes the exact path
  const float nzr = __fmul_rn(-g.z, g.r);
  const float q_lo = __fmaf_rn(mn, g.r, nzr), q_hi = __fmaf_rn(mx, g.r, nzr);
  g.fast = fabsf(nzr) <= 65536.0f && q_lo >= -0.49f && q_hi <= L + 0.49f;
  return g;
}

// Codes as floats.  4-bit: c[i] = code of register pair 2i plus 1.5 * 2^23
// (i < 4) and c[4 + i] = code of pair 2i + 1, so c[4 + i] * 16 + c[i] holds
// the byte of channels (2i, 2i + 1) (.x) and (2i + 8, 2i + 9) (.y) in its low
// bits.  8-bit: c[p] = code of pair p plus 1.5 * 2^23.
template <int BITS>
__device__ __forceinline__ void fast_codes(const float2 (&x)[8], float xs, const GroupParams& g, float2 (&c)[8]) {
  const float2 m2 = make_float2(kRoundMagic, kRoundMagic);
  const float2 mm2 = make_float2(-kRoundMagic, -kRoundMagic);
  const float2 r2 = make_float2(g.r, g.r), ns2 = make_float2(-g.s, -g.s), nz2 = make_float2(-g.z, -g.z);
  const float2 xs2 = make_float2(xs, xs);
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const float2 u = __ffma2_rn(x[p], xs2, nz2);                         // fl(x xs - z), x xs exact
    const float2 q0 = __fmul2_rn(u, r2);
    const float2 q1 = __ffma2_rn(__ffma2_rn(q0, ns2, u), r2, q0);        // fl(u / s)
    const float2 yk = __fadd2_rn(q1, m2);                                // rne(q1) in the low bits
    if (BITS == 4) {
      if (p % 2 == 0) c[p / 2] = yk;
      else c[4 + p / 2] = __fadd2_rn(yk, mm2);
    } else {
      c[p] = yk;
    }
  }
}

template <int BITS>
__device__ __forceinline__ void clamped_codes(const float2 (&x)[8], float xs, const GroupParams& g, float2 (&c)[8]) {
  constexpr int L = (1 << BITS) - 1;
  const float2 m2 = make_float2(kRoundMagic, kRoundMagic);
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    // s = 0 (a constant group) codes 0, as on the fast path
    const int r0 = g.s == 0.0f ? 0 : min(max(__float2int_rn(__fdiv_rn(__fsub_rn(__fmul_rn(x[p].x, xs), g.z), g.s)), 0), L);
    const int r1 = g.s == 0.0f ? 0 : min(max(__float2int_rn(__fdiv_rn(__fsub_rn(__fmul_rn(x[p].y, xs), g.z), g.s)), 0), L);
    const float2 k = make_float2(static_cast<float>(r0), static_cast<float>(r1));
    if (BITS == 4) {
      if (p % 2 == 0) c[p / 2] = __fadd2_rn(k, m2);
      else c[4 + p / 2] = k;
    } else {
      c[p] = __fadd2_rn(k, m2);
    }
  }
}

template <int BITS>
__device__ __forceinline__ void store_codes(const float2 (&c)[8], const GroupParams& g, int j,
                                            uint8_t* __restrict__ code_dst,
                                            __half2* __restrict__ param_dst, bool valid) {
  if (BITS == 2) {
    // element e (pair e % 8, half e / 8) at bits 2e of the lane's word: four
    // codes per byte, element 4i + m at bits 2m of byte i
    uint32_t w = 0;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      w |= (__float_as_uint(c[p].x) & 3u) << (2 * p);
      w |= (__float_as_uint(c[p].y) & 3u) << (2 * (p + 8));
    }
    st_if(valid, code_dst + j * 4, w);
  } else if (BITS == 4) {
    // byte b holds elements 2b (low nibble) and 2b+1 (high nibble); the sums
    // are exact (integers below 2^24)
    uint32_t b[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 w = __ffma2_rn(c[4 + i], make_float2(16.0f, 16.0f), c[i]);
      b[i] = __float_as_uint(w.x);
      b[i + 4] = __float_as_uint(w.y);
    }
    const uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
    st_if(valid, code_dst + j * 8, make_uint2(lo, hi));
  } else {
    // element e: pair e % 8, half e / 8
    uint32_t q[kEPL];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      q[p] = __float_as_uint(c[p].x);
      q[p + 8] = __float_as_uint(c[p].y);
    }
    uint4 w;
    w.x = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
    w.y = __byte_perm(__byte_perm(q[4], q[5], 0x0040), __byte_perm(q[6], q[7], 0x0040), 0x5410);
    w.z = __byte_perm(__byte_perm(q[8], q[9], 0x0040), __byte_perm(q[10], q[11], 0x0040), 0x5410);
    w.w = __byte_perm(__byte_perm(q[12], q[13], 0x0040), __byte_perm(q[14], q[15], 0x0040), 0x5410);
    st_if(valid, code_dst + j * 16, w);
  }
  // the four lanes of a group hold the same parameters and all store them:
  // one branch fewer, and the stores merge in the same sector
  const __half2 pv = __halves2half2(g.sh, g.zh);
  st_if(valid, param_dst + (j >> 2), *reinterpret_cast<const uint32_t*>(&pv));
}

// FP8 comparison cache: the lane's 16 values as OCP E4M3 bytes (round to
// nearest even, saturated to +-448), channel order, one 16-byte store.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {   // lo -> low byte
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ void store_fp8(const float2 (&x)[8], uint8_t* __restrict__ dst) {
  // pair p holds channels p (.x) and p + 8 (.y)
  uint4 w;
  w.x = e4m3x2(x[0].x, x[1].x) | e4m3x2(x[2].x, x[3].x) << 16;
  w.y = e4m3x2(x[4].x, x[5].x) | e4m3x2(x[6].x, x[7].x) << 16;
  w.z = e4m3x2(x[0].y, x[1].y) | e4m3x2(x[2].y, x[3].y) << 16;
  w.w = e4m3x2(x[4].y, x[5].y) | e4m3x2(x[6].y, x[7].y) << 16;
  *reinterpret_cast<uint4*>(dst) = w;
}

// K (already rotated when the pool stores rotated keys; its values are the
// rotated ones divided by ks) and V of one warp item.
template <int BITS>
__device__ __forceinline__ void encode_kv(const float2 (&xk)[8], float ks, const float2 (&xv)[8], int j,
                                          bool valid, uint8_t* __restrict__ kc, __half2* __restrict__ kp,
                                          uint8_t* __restrict__ vc, __half2* __restrict__ vp) {
  const GroupParams gk = group_params<BITS>(xk, ks);
  const GroupParams gv = group_params<BITS>(xv, 1.0f);
  float2 ck[8], cv[8];
  fast_codes<BITS>(xk, ks, gk, ck);
  fast_codes<BITS>(xv, 1.0f, gv, cv);
  if (!gk.fast) clamped_codes<BITS>(xk, ks, gk, ck);
  if (!gv.fast) clamped_codes<BITS>(xv, 1.0f, gv, cv);
  store_codes<BITS>(ck, gk, j, kc, kp, valid);
  store_codes<BITS>(cv, gv, j, vc, vp, valid);
}

}  // namespace
}  // namespace q4kv
