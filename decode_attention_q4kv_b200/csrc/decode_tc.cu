// Split-K paged GQA decode attention on the tensor cores.
//
// "Agent Memory Below the Prompt" (arXiv 2603.04428 summary), sec. 2.1 items
// 2-3 and sec. 2.2: batched GQA attention read straight from the packed
// 4-bit cache.  IntentKV article (Qiita), "詰め直さずに「無効化」する":
// remapped slots get logit -1e4 and value 0.  UltraQuant news item
// (arXiv 2606.20474), "技術/ビジネス面": keys are stored Walsh-Hadamard
// rotated, so the query is rotated by the same transform.
//
// Why tensor cores: per (token, KV head) the g query heads of a GQA group do
// g*D multiply-adds against the keys and g*D against the values, over 144
// bytes of packed data (D = 128).  At HBM speed that is more fp32 FMA issue
// than the SM has, so both contractions run as mma.sync.m16n8k16 (fp16 in,
// fp32 accumulate) with the codes (exact small integers in fp16) as one
// operand.  tcgen05 would need the unpacked codes in shared memory or TMEM
// (4x the packed bytes of shared-memory traffic, N <= 16 columns), so the
// register-fed mma.sync is the better fit for this N.
//
//   keys:   S^T[16 tokens][8 cols] += Kcodes[16 tokens][16 ch] x Qm[16 ch][8 cols]
//           A column of Qm is one (query head h, group gr) pair: q_rot[h] on
//           the 64 channels of group gr and 0 elsewhere, so each thread gets
//           the per-group partial dots and applies that token's (s, z) in
//           registers: logit = sum_gr s_gr S_gr + z_gr sum(q_rot over gr).
//           q_rot is split into fp16 hi + lo parts (two MMAs), so it is
//           carried to ~22 bits.
//   values: O^T[16 ch][8 cols] += Vcodes^T[16 ch][16 tokens] x W[16 tokens][8 cols]
//           with W[t][(h, gr)] = p_t,h * s_t,gr (the value scale folded into
//           the weight) and the zero term sum_t p_t,h z_t,gr added at the end;
//           a channel keeps only the column of its own group.  The softmax
//           weights come out of the key MMA in the accumulator layout; one
//           movmatrix.trans per 8x8 turns them into the B operand.
//
// Data movement: a producer warp streams each (block, KV head) run of codes,
// scales/zeros and the block's remap mask with 1-D TMA bulk copies
// (cp.async.bulk, no multicast) into a 4-deep ring of shared-memory stages
// guarded by mbarriers; 8 consumer warps each take 16-token tiles of a stage.
// Every mbarrier wait is bounded: on time-out the kernel raises
// Q4KV_DEVERR_TIMEOUT, poisons the affected rows and returns.
//
// Scheduling: persistent CTAs (one per SM) walk the work items
// (sequence, KV head, split) with a static stride; the producer runs ahead
// across item boundaries.  Each item ends with a cross-warp log-sum-exp merge
// in shared memory and writes either the final row (one split) or a partial.
#include <math.h>

#include "q4kv_internal.cuh"

namespace q4kv {
namespace {

constexpr int kCW = 8;                      // consumer warps
constexpr int kThreadsTC = (kCW + 1) * 32;  // + one producer warp
constexpr int kNS = 4;                      // pipeline stages
constexpr int kCodeBytes = 16384;           // codes of one tensor per stage
constexpr int kParamBytes = 2048;           // scale/zero of one tensor per stage
constexpr int kOffV = kCodeBytes;
constexpr int kOffKP = 2 * kCodeBytes;
constexpr int kOffVP = kOffKP + kParamBytes;
constexpr int kOffMask = kOffVP + kParamBytes;
constexpr int kOffMeta = kOffMask + 32;
constexpr int kStageBytes = kOffMeta + 32;  // 36928, a multiple of 16
constexpr float kLog2e = 1.4426950408889634f;
constexpr unsigned kSpinLimit = 1u << 26;   // bounded mbarrier waits

struct StageMeta {
  int32_t blk;      // unified block id, -1 if none / invalid
  int32_t tok0;     // first token of the stage within the sequence
  int16_t slot0;    // first slot within the block
  int16_t ntok;     // tokens of the stage that belong to the range
  uint8_t is8;
  uint8_t last;     // last stage of its work item
  uint8_t poison;   // the item touched a bad block id or a bad length
  uint8_t timeout;  // the producer gave up waiting
};

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; false when the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (unsigned i = 0; i < kSpinLimit; ++i) {
    if (mbar_test(bar, parity)) return true;
    if (i > 64) __nanosleep(32);
  }
  return false;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kCW * 32) : "memory");
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movtrans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t lop_or(uint32_t x, uint32_t mask, uint32_t bits) {
  return (x & mask) | bits;
}
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// 0x6400 is fp16 1024: (nibble | 0x6400) = 1024 + nibble, (nibble << 4 | 0x6400) = 1024 + 16 nibble.
__device__ __forceinline__ uint32_t lo_nib(uint32_t x) {   // nibbles at bits 0-3, 16-19 -> exact codes
  return h2u(__hsub2(u2h(lop_or(x, 0x000F000Fu, 0x64006400u)), u2h(0x64006400u)));
}
__device__ __forceinline__ uint32_t hi_nib(uint32_t x) {   // nibbles at bits 4-7, 20-23 -> exact codes
  return h2u(__hfma2(u2h(lop_or(x, 0x00F000F0u, 0x64006400u)), u2h(0x2C002C00u) /*1/16*/,
                     u2h(0xD400D400u) /*-64*/));
}
__device__ __forceinline__ uint32_t byte_pair(uint32_t x) {  // bytes at 0, 2 -> exact codes
  return h2u(__hsub2(u2h(lop_or(x, 0x00FF00FFu, 0x64006400u)), u2h(0x64006400u)));
}

template <typename T>
__device__ __forceinline__ T lds(const void* p) { return *reinterpret_cast<const T*>(p); }

// ---------------------------------------------------------------------------
// geometry
// ---------------------------------------------------------------------------
template <int D, bool Q8>
struct Geo {
  static constexpr int NG = D / kGroup;
  static constexpr int RB = Q8 ? D : D / 2;             // code bytes per token row
  static constexpr int TS = kCodeBytes / RB;            // tokens per stage
  static constexpr int PB = NG * 4;                     // param bytes per token row
  static constexpr int MTILES = TS / 16;                // 16-token tiles per stage
  static constexpr int KB = Q8 ? D / 4 : D / 8;         // key bytes a thread owns per row
  static constexpr int VB = Q8 ? D / 8 : D / 16;        // value bytes a thread owns per row
  static_assert(TS * PB <= kParamBytes, "stage params");
};

// Key A operand of k-step s for the thread's two rows (from their key bytes).
// Thread t owns channels 128c + 32t + [0, 32) of each row (c < D/128); k-step
// s uses chunk c = s/8, 8-channel word w = (s%8)/2, pairs p0 = 2 (s%2) and
// p0 + 1, where pair p of a word = channels (p, p + 4) of it.
template <int D, bool Q8>
__device__ __forceinline__ void key_a(const uint32_t* rg, const uint32_t* rg8, int s, uint32_t (&a)[4]) {
  const int c = s / 8, w = (s % 8) / 2, p0 = 2 * (s % 2);
  if (!Q8) {
    // 16 bytes per chunk = 4 words of 8 nibbles; word index c*4 + w
    const uint32_t x0 = rg[c * 4 + w], x1 = rg8[c * 4 + w];
    if (p0 == 0) {   // pairs 0 (lo nibbles of bytes 0, 2) and 1 (hi nibbles of bytes 0, 2)
      a[0] = lo_nib(x0); a[1] = lo_nib(x1); a[2] = hi_nib(x0); a[3] = hi_nib(x1);
    } else {         // pairs 2, 3: the same for bytes 1, 3
      a[0] = lo_nib(x0 >> 8); a[1] = lo_nib(x1 >> 8); a[2] = hi_nib(x0 >> 8); a[3] = hi_nib(x1 >> 8);
    }
  } else {
    // 32 bytes per chunk = 8 words of 4 codes; channels 8w + e are in words 2w (e < 4), 2w+1
    const uint32_t l0 = rg[c * 8 + 2 * w], h0 = rg[c * 8 + 2 * w + 1];
    const uint32_t l1 = rg8[c * 8 + 2 * w], h1 = rg8[c * 8 + 2 * w + 1];
    const uint32_t s0 = p0 | (p0 << 8) + 0x400u;          // [lo.p0, -, hi.p0, -]
    const uint32_t s1 = (p0 + 1) | ((p0 + 1) << 8) + 0x400u;
    a[0] = byte_pair(__byte_perm(l0, h0, s0));
    a[1] = byte_pair(__byte_perm(l1, h1, s0));
    a[2] = byte_pair(__byte_perm(l0, h0, s1));
    a[3] = byte_pair(__byte_perm(l1, h1, s1));
  }
}

// Value A operands for one 16-token tile: tokens T = 2t, 2t+1, 2t+8, 2t+9 of
// the tile, thread g's channels cb + [0, D/8).  Tile mv (channels) uses rows
// g -> cb + 2 mv and g + 8 -> cb + 2 mv + 1.
template <int D, bool Q8>
__device__ __forceinline__ void value_a(const uint32_t* v0, const uint32_t* v1, const uint32_t* v8,
                                        const uint32_t* v9, int mv, uint32_t (&a)[4]) {
  if (!Q8) {
    // byte mv of the thread's run: low nibble = channel cb + 2mv, high = cb + 2mv + 1
    const int wi = mv / 4, bp = mv % 4;
    const uint32_t sel = bp | ((bp + 4) << 8);             // [T1.b, -, T2.b, -]
    const uint32_t x01 = __byte_perm(v0[wi], v1[wi], sel);
    const uint32_t x89 = __byte_perm(v8[wi], v9[wi], sel);
    a[0] = lo_nib(x01); a[1] = hi_nib(x01); a[2] = lo_nib(x89); a[3] = hi_nib(x89);
  } else {
    const int wi = (2 * mv) / 4, bp = (2 * mv) % 4;
    const uint32_t sa = bp | ((bp + 4) << 8), sb = (bp + 1) | ((bp + 5) << 8);
    a[0] = byte_pair(__byte_perm(v0[wi], v1[wi], sa));
    a[1] = byte_pair(__byte_perm(v0[wi], v1[wi], sb));
    a[2] = byte_pair(__byte_perm(v8[wi], v9[wi], sa));
    a[3] = byte_pair(__byte_perm(v8[wi], v9[wi], sb));
  }
}

__device__ __forceinline__ void store_out(void* p, int dtype, int64_t i, float x) {
  if (dtype == Q4KV_F32) static_cast<float*>(p)[i] = x;
  else if (dtype == Q4KV_F16) static_cast<__half*>(p)[i] = __float2half_rn(x);
  else static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
}

// ---------------------------------------------------------------------------
// per-consumer-warp running state of one work item
// ---------------------------------------------------------------------------
template <int D, int NT>
struct WarpState {
  float o[D / 16][NT][4];   // value accumulators (channels x (head, group) columns)
  float m[NT];              // running max, log2 units
  float l[NT];              // this thread's share of the running sum
  float z[NT][2];           // sum p * zero for the thread's two columns
};

template <int D, int NT>
__device__ __forceinline__ void reset(WarpState<D, NT>& st) {
#pragma unroll
  for (int mv = 0; mv < D / 16; ++mv)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) st.o[mv][j][e] = 0.0f;
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    st.m[j] = -INFINITY;
    st.l[j] = 0.0f;
    st.z[j][0] = st.z[j][1] = 0.0f;
  }
}

// One 16-token tile of a stage: keys, softmax update, values.
template <int D, int NT, bool Q8>
__device__ __forceinline__ void tile(WarpState<D, NT>& st, const uint8_t* stage, int row0, int nvalid,
                                     const uint32_t (&bq)[D / 16][NT][4], const float (&qs)[NT][2],
                                     float sc2, int lane) {
  using G = Geo<D, Q8>;
  const int g = lane >> 2, t = lane & 3;
  // ---- keys: two rows per thread (tile rows g and g + 8) ----
  uint32_t rg[G::KB / 4], rg8[G::KB / 4];
  {
    const uint8_t* kc = stage + (row0 + g) * G::RB;
    const uint8_t* kc8 = stage + (row0 + g + 8) * G::RB;
#pragma unroll
    for (int c = 0; c < D / 128; ++c) {
#pragma unroll
      for (int q = 0; q < G::KB / (D / 128) / 16; ++q) {
        const int off = c * (G::RB / (D / 128)) + t * (G::KB / (D / 128)) + q * 16;
        const uint4 u = lds<uint4>(kc + off), u8 = lds<uint4>(kc8 + off);
        const int wi = c * (G::KB / (D / 128) / 4) + q * 4;
        rg[wi] = u.x; rg[wi + 1] = u.y; rg[wi + 2] = u.z; rg[wi + 3] = u.w;
        rg8[wi] = u8.x; rg8[wi + 1] = u8.y; rg8[wi + 2] = u8.z; rg8[wi + 3] = u8.w;
      }
    }
  }
  float sacc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.0f;
#pragma unroll
  for (int s = 0; s < D / 16; ++s) {
    uint32_t a[4];
    key_a<D, Q8>(rg, rg8, s, a);
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      mma16816(sacc[j], a, bq[s][j][0], bq[s][j][1]);   // q hi
      mma16816(sacc[j], a, bq[s][j][2], bq[s][j][3]);   // q lo
    }
  }
  // ---- per-token parameters for the thread's two columns' groups ----
  // D = 128: columns (h, 0), (h, 1); D = 256: (h, 2 (t%2)), (h, 2 (t%2) + 1).
  const int gbase = (G::NG == 2) ? 0 : 2 * (t & 1);
  const uint8_t* kp = stage + kOffKP;
  const uint8_t* vp = stage + kOffVP;
  const uint32_t* mask = reinterpret_cast<const uint32_t*>(stage + kOffMask);
  const StageMeta& meta = *reinterpret_cast<const StageMeta*>(stage + kOffMeta);
  float logit[NT][2];
  float ws[2][2], wz[2][2];   // [row][e]: value scale, zero
  bool live[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int row = row0 + g + 8 * r;
    const bool valid = row < nvalid;
    const int slot = meta.slot0 + row;
    const bool masked = valid && ((mask[slot >> 5] >> (slot & 31)) & 1u);
    live[r] = valid && !masked;
    const uint2 kpw = lds<uint2>(kp + row * G::PB + gbase * 4);
    const uint2 vpw = lds<uint2>(vp + row * G::PB + gbase * 4);
    const float2 k0 = __half22float2(u2h(kpw.x)), k1 = __half22float2(u2h(kpw.y));
    const float2 v0 = __half22float2(u2h(vpw.x)), v1 = __half22float2(u2h(vpw.y));
    // rows outside the range or remapped may hold any bytes (even NaN
    // parameters): select, never multiply, them away
    ws[r][0] = live[r] ? v0.x : 0.0f;
    wz[r][0] = live[r] ? v0.y : 0.0f;
    ws[r][1] = live[r] ? v1.x : 0.0f;
    wz[r][1] = live[r] ? v1.y : 0.0f;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      float part = __fmaf_rn(k0.x, sacc[j][2 * r], k1.x * sacc[j][2 * r + 1]) * sc2 +
                   (k0.y * qs[j][0] + k1.y * qs[j][1]);
      if (G::NG == 4) part += __shfl_xor_sync(0xffffffffu, part, 1);
      logit[j][r] = !valid ? -INFINITY : (masked ? Q4KV_SENTINEL_LOGIT * kLog2e : part);
    }
  }
  // ---- online softmax over the tile (16 tokens), per column head ----
  uint32_t wb[NT][2];   // W pairs for rows g, g + 8 (accumulator layout)
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    float mx = fmaxf(logit[j][0], logit[j][1]);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    const float m_new = fmaxf(st.m[j], mx);
    float alpha = 1.0f, p0 = 0.0f, p1 = 0.0f;
    if (m_new != -INFINITY) {
      alpha = ex2(st.m[j] - m_new);   // 0 when the old max is -inf
      p0 = ex2(logit[j][0] - m_new);
      p1 = ex2(logit[j][1] - m_new);
    }
    st.m[j] = m_new;
    st.l[j] = __fmaf_rn(st.l[j], alpha, p0 + p1);
    const float q0 = live[0] ? p0 : 0.0f, q1 = live[1] ? p1 : 0.0f;
    st.z[j][0] = __fmaf_rn(st.z[j][0], alpha, __fmaf_rn(q0, wz[0][0], q1 * wz[1][0]));
    st.z[j][1] = __fmaf_rn(st.z[j][1], alpha, __fmaf_rn(q0, wz[0][1], q1 * wz[1][1]));
#pragma unroll
    for (int mv = 0; mv < D / 16; ++mv)
#pragma unroll
      for (int e = 0; e < 4; ++e) st.o[mv][j][e] *= alpha;
    wb[j][0] = h2u(__floats2half2_rn(q0 * ws[0][0], q0 * ws[0][1]));
    wb[j][1] = h2u(__floats2half2_rn(q1 * ws[1][0], q1 * ws[1][1]));
  }
  // ---- values ----
  uint32_t bw[NT][2];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    bw[j][0] = movtrans(wb[j][0]);   // tokens 2t, 2t+1 of rows 0-7
    bw[j][1] = movtrans(wb[j][1]);   // tokens 8 + 2t, 9 + 2t
  }
  constexpr int VW = G::VB / 4;   // words of value codes per token row
  uint32_t v0[VW], v1[VW], v8[VW], v9[VW];
  {
    const uint8_t* vc = stage + kOffV + g * G::VB;
#pragma unroll
    for (int q = 0; q < VW; q += 2) {
      const uint2 a0 = lds<uint2>(vc + (row0 + 2 * t) * G::RB + 4 * q);
      const uint2 a1 = lds<uint2>(vc + (row0 + 2 * t + 1) * G::RB + 4 * q);
      const uint2 a8 = lds<uint2>(vc + (row0 + 2 * t + 8) * G::RB + 4 * q);
      const uint2 a9 = lds<uint2>(vc + (row0 + 2 * t + 9) * G::RB + 4 * q);
      v0[q] = a0.x; v0[q + 1] = a0.y; v1[q] = a1.x; v1[q + 1] = a1.y;
      v8[q] = a8.x; v8[q + 1] = a8.y; v9[q] = a9.x; v9[q + 1] = a9.y;
    }
  }
#pragma unroll
  for (int mv = 0; mv < D / 16; ++mv) {
    uint32_t a[4];
    value_a<D, Q8>(v0, v1, v8, v9, mv, a);
#pragma unroll
    for (int j = 0; j < NT; ++j) mma16816(st.o[mv][j], a, bw[j][0], bw[j][1]);
  }
}

template <int D, int NT>
__global__ void __launch_bounds__(kThreadsTC, 1) decode_tc_kernel(const DecodeArgs a, int n_items) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kNS * kStageBytes);
  uint64_t* empty = full + kNS;
  float* qrot = reinterpret_cast<float*>(empty + kNS);                 // [G][D]
  float* qsum = qrot + 8 * D;                                          // [8][4]
  float* mrg_ml = qsum + 32;                                           // [kCW][8][2]
  float* mrg_o = mrg_ml + kCW * 16;                                    // [kCW][G][D]
  __shared__ int s_flags[2];                                            // poison, timeout

  const PoolView& P = a.pool;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hkv = P.n_kv_heads, hq = a.plan.n_q_heads, G = hq / hkv;
  const int S = a.plan.n_splits, tps = a.plan.tokens_per_split, mb = a.plan.max_blocks_per_seq;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kCW);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // -------------------------------------------------------------------------
  // producer warp
  // -------------------------------------------------------------------------
  if (warp == kCW) {
    if (lane != 0) return;
    uint32_t it = 0;
    bool gave_up = false;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const int split = item % S;
      const int kvh = (item / S) % hkv;
      const int b = item / (S * hkv);
      const int seq = a.seq_lens[b];
      const bool bad_seq = seq < 0 || seq > mb * kBlockTokens;
      if (bad_seq && split == 0 && kvh == 0) raise_error(P.error_word, Q4KV_DEVERR_SEQ_LEN);
      const int t0 = split * tps;
      const int t1 = bad_seq ? t0 : min(t0 + tps, seq);
      int tok = t0;
      do {
        const int s = it % kNS;
        if (!gave_up && !mbar_wait(&empty[s], ((it / kNS) & 1) ^ 1)) gave_up = true;
        uint8_t* stg = stages + s * kStageBytes;
        StageMeta meta;
        meta.tok0 = tok;
        meta.poison = bad_seq;
        meta.timeout = gave_up;
        meta.blk = -1;
        meta.is8 = 0;
        meta.slot0 = static_cast<int16_t>(tok % kBlockTokens);
        int step = Geo<D, false>::TS;
        if (tok < t1) {
          // a stage never crosses a block boundary, whatever the split length
          const int32_t blk = a.tables[static_cast<int64_t>(b) * mb + tok / kBlockTokens];
          if (blk < 0 || blk >= P.n_q4 + P.n_q8) {
            raise_error(P.error_word, Q4KV_DEVERR_BLOCK_ID);
            meta.poison = 1;
          } else {
            meta.blk = blk;
            meta.is8 = blk >= P.n_q4;
            if (meta.is8) step = Geo<D, true>::TS;
          }
          step = min(step, kBlockTokens - tok % kBlockTokens);
        }
        meta.ntok = static_cast<int16_t>(max(0, min(step, t1 - tok)));
        meta.last = (tok + step >= t1) ? 1 : 0;
        *reinterpret_cast<StageMeta*>(stg + kOffMeta) = meta;
        if (meta.blk >= 0 && !gave_up) {
          const int rows = (meta.ntok + 15) & ~15;   // whole 16-token tiles, inside the block
          const bool is8 = meta.is8;
          const int64_t phys = is8 ? meta.blk - P.n_q4 : meta.blk;
          const int64_t row = (phys * hkv + kvh) * kBlockTokens + meta.slot0;
          const int rb = is8 ? D : D / 2, pb = (D / kGroup) * 4;
          const uint8_t* kc = (is8 ? P.k_codes8 : P.k_codes4) + row * rb;
          const uint8_t* vc = (is8 ? P.v_codes8 : P.v_codes4) + row * rb;
          const uint8_t* kpp = reinterpret_cast<const uint8_t*>(is8 ? P.k_params8 : P.k_params4) + row * pb;
          const uint8_t* vpp = reinterpret_cast<const uint8_t*>(is8 ? P.v_params8 : P.v_params4) + row * pb;
          const uint32_t cb = rows * rb, prb = rows * pb;
          mbar_arrive_tx(&full[s], 2 * cb + 2 * prb + 32);
          bulk_g2s(stg, kc, cb, &full[s]);
          bulk_g2s(stg + kOffV, vc, cb, &full[s]);
          bulk_g2s(stg + kOffKP, kpp, prb, &full[s]);
          bulk_g2s(stg + kOffVP, vpp, prb, &full[s]);
          bulk_g2s(stg + kOffMask, P.mask + static_cast<int64_t>(meta.blk) * kMaskWords, 32, &full[s]);
        } else {
          mbar_arrive(&full[s]);
        }
        ++it;
        tok += step;
      } while (tok < t1);
    }
    // no copy may still be landing when the CTA exits: wait (bounded) for the
    // last stages issued to complete
    for (uint32_t k = (it > kNS ? it - kNS : 0); k < it; ++k)
      if (!mbar_wait(&full[k % kNS], (k / kNS) & 1)) break;
    return;
  }

  // -------------------------------------------------------------------------
  // consumer warps
  // -------------------------------------------------------------------------
  const int g = lane >> 2, t = lane & 3;
  constexpr int NG = D / kGroup;
  const float sc2 = a.scale * kLog2e;
  WarpState<D, NT> st;
  uint32_t bq[D / 16][NT][4];
  float qs[NT][2];
  uint32_t it = 0;
  bool dead = false;

  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int split = item % S;
    const int kvh = (item / S) % hkv;
    const int b = item / (S * hkv);
    // ---- rotated query of the item's G heads -> B fragments ----
    for (int i = threadIdx.x; i < G * D; i += kCW * 32) {
      const int64_t qi = (static_cast<int64_t>(b) * hq + kvh * G) * D + i;
      qrot[i] = a.q_dtype == Q4KV_F16 ? __half2float(static_cast<const __half*>(a.q)[qi])
                                      : __bfloat162float(static_cast<const __nv_bfloat16*>(a.q)[qi]);
    }
    consumer_sync();
    if (P.k_rotated) {
      for (int hs = 1; hs < D; hs <<= 1) {
        for (int i = threadIdx.x; i < G * (D / 2); i += kCW * 32) {
          const int h = i / (D / 2), p = i % (D / 2);
          const int lo = h * D + (p / hs) * 2 * hs + (p % hs), hi = lo + hs;
          const float x = qrot[lo], y = qrot[hi];
          qrot[lo] = x + y;
          qrot[hi] = x - y;
        }
        consumer_sync();
      }
      const float c = rotation_constant(D);
      for (int i = threadIdx.x; i < G * D; i += kCW * 32) qrot[i] *= c;
      consumer_sync();
    }
    if (threadIdx.x < G * NG) {   // group sums of the rotated query
      const int h = threadIdx.x / NG, gr = threadIdx.x % NG;
      float acc = 0.0f;
      for (int c = 0; c < kGroup; ++c) acc += qrot[h * D + gr * kGroup + c];
      qsum[h * 4 + gr] = acc;
    }
    consumer_sync();
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int col = 8 * j + g;                // this thread's B column
      const int h = col / NG, gr = col % NG;
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const int c = s / 8, w = (s % 8) / 2, p0 = 2 * (s % 2);
        const int base = 128 * c + 32 * t + 8 * w;
        float v[4];
        const int chs[4] = {base + p0, base + p0 + 4, base + p0 + 1, base + p0 + 5};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          v[e] = (h < G && chs[e] / kGroup == gr) ? qrot[h * D + chs[e]] : 0.0f;
        const __half2 h01 = __floats2half2_rn(v[0], v[1]), h23 = __floats2half2_rn(v[2], v[3]);
        const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
        bq[s][j][0] = h2u(h01);
        bq[s][j][1] = h2u(h23);
        bq[s][j][2] = h2u(__floats2half2_rn(v[0] - f01.x, v[1] - f01.y));
        bq[s][j][3] = h2u(__floats2half2_rn(v[2] - f23.x, v[3] - f23.y));
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {   // the thread's accumulator columns 8j + 2t + e
        const int c2 = 8 * j + 2 * t + e;
        const int h2 = c2 / NG, g2 = c2 % NG;
        qs[j][e] = h2 < G ? qsum[h2 * 4 + g2] * sc2 : 0.0f;
      }
    }
    reset(st);
    bool poison = false, timeout = false;

    // ---- the item's stages ----
    for (;;) {
      const int s = it % kNS;
      if (!dead && !mbar_wait(&full[s], (it / kNS) & 1)) dead = true;
      const uint8_t* stg = stages + s * kStageBytes;
      const StageMeta meta = *reinterpret_cast<const StageMeta*>(stg + kOffMeta);
      const bool last = dead ? true : meta.last;
      timeout |= dead || meta.timeout;
      poison |= meta.poison;
      if (!dead && !meta.timeout && meta.blk >= 0) {
        if (!meta.is8) {
          for (int mt = warp; mt < Geo<D, false>::MTILES; mt += kCW)
            if (mt * 16 < meta.ntok) tile<D, NT, false>(st, stg, mt * 16, meta.ntok, bq, qs, sc2, lane);
        } else {
          for (int mt = warp; mt < Geo<D, true>::MTILES; mt += kCW)
            if (mt * 16 < meta.ntok) tile<D, NT, true>(st, stg, mt * 16, meta.ntok, bq, qs, sc2, lane);
        }
      }
      __syncwarp();
      if (lane == 0 && !dead) mbar_arrive(&empty[s]);
      ++it;
      if (last) break;
    }
    if (timeout && threadIdx.x == 0) raise_error(P.error_word, Q4KV_DEVERR_TIMEOUT);

    // ---- cross-warp merge of the item ----
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      float lt = st.l[j], z0 = st.z[j][0], z1 = st.z[j][1];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        lt += __shfl_xor_sync(0xffffffffu, lt, off);
        z0 += __shfl_xor_sync(0xffffffffu, z0, off);
        z1 += __shfl_xor_sync(0xffffffffu, z1, off);
      }
      const int c0 = 8 * j + 2 * t;
      const int h = c0 / NG;
      if (g == 0 && h < G && (NG == 2 || (t & 1) == 0)) {
        mrg_ml[(warp * 8 + h) * 2] = st.m[j];
        mrg_ml[(warp * 8 + h) * 2 + 1] = lt;
      }
      const float zz[2] = {z0, z1};
#pragma unroll
      for (int mv = 0; mv < D / 16; ++mv) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int ch = (D / 8) * g + 2 * mv + (e >> 1);
          const int col = c0 + (e & 1);
          const int hh = col / NG, gr = col % NG;
          if (hh < G && gr == ch / kGroup)
            mrg_o[(warp * G + hh) * D + ch] = st.o[mv][j][e] + zz[e & 1];
        }
      }
    }
    if (threadIdx.x == 0) {
      s_flags[0] = poison || timeout;
    }
    consumer_sync();
    const bool bad = s_flags[0] != 0;
    for (int i = threadIdx.x; i < G * D; i += kCW * 32) {
      const int h = i / D, ch = i % D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kCW; ++w) M = fmaxf(M, mrg_ml[(w * 8 + h) * 2]);
      float num = 0.0f, den = 0.0f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kCW; ++w) {
          const float f = ex2(mrg_ml[(w * 8 + h) * 2] - M);
          den = __fmaf_rn(mrg_ml[(w * 8 + h) * 2 + 1], f, den);
          num = __fmaf_rn(mrg_o[(w * G + h) * D + ch], f, num);
        }
      }
      const int64_t qrow = static_cast<int64_t>(b) * hq + kvh * G + h;
      if (S == 1) {
        store_out(a.out, a.out_dtype, qrow * D + ch, (!bad && den > 0.0f) ? num / den : 0.0f);
      } else {
        a.ws_o[(qrow * S + split) * D + ch] = num;
        if (ch == 0) {
          a.ws_ml[(qrow * S + split) * 2] = M == -INFINITY ? -INFINITY : M / kLog2e;
          a.ws_ml[(qrow * S + split) * 2 + 1] = bad ? -1.0f : den;
        }
      }
    }
    consumer_sync();   // the merge area and the query buffers are reused by the next item
  }
}

}  // namespace

size_t decode_tc_smem_bytes(int head_dim) {
  return static_cast<size_t>(kNS) * kStageBytes + 2 * kNS * sizeof(uint64_t) +
         (8 * head_dim + 32 + kCW * 16) * sizeof(float) + static_cast<size_t>(kCW) * 1024 * sizeof(float);
}

cudaError_t launch_decode_tc(const DecodeArgs& a, int num_sms, cudaStream_t stream) {
  const q4kv_decode_plan& p = a.plan;
  const int n_items = p.batch * p.n_kv_heads * p.n_splits;
  const int grid = min(n_items, num_sms);
  const int g = p.n_q_heads / p.n_kv_heads;
  const int nt = (g * (p.head_dim / kGroup) + 7) / 8;
  const size_t smem = decode_tc_smem_bytes(p.head_dim);
  cudaError_t e = cudaSuccess;
#define Q4KV_TC(DD, NN)                                                                           \
  do {                                                                                            \
    e = cudaFuncSetAttribute(decode_tc_kernel<DD, NN>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             static_cast<int>(smem));                                             \
    if (e == cudaSuccess) decode_tc_kernel<DD, NN><<<grid, kThreadsTC, smem, stream>>>(a, n_items); \
  } while (0)
  if (p.head_dim == 128 && nt == 1) Q4KV_TC(128, 1);
  else if (p.head_dim == 128) Q4KV_TC(128, 2);
  else if (nt == 1) Q4KV_TC(256, 1);
  else Q4KV_TC(256, 2);
#undef Q4KV_TC
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace q4kv
