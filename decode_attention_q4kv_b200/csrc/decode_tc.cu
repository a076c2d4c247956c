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
// than the SM has, so both contractions run on the tensor cores with the
// codes as one operand, unpacked in registers.  tcgen05 would need the
// unpacked codes in shared memory or TMEM (2-4x the packed bytes of
// shared-memory traffic, N <= 16 columns), so the register-fed mma.sync is
// the better fit for this N.
//
//   keys:   S^T[16 tokens][8 cols] += Kcodes[16 tokens][32 ch] x Qm[32 ch][8 cols]
//           (mma.sync.m16n8k32, u8 codes x s8 query digits, exact int32).
//           A column of Qm is one (query head h, group gr) pair: q_rot[h] on
//           the 64 channels of group gr and 0 elsewhere, so each thread gets
//           the per-group partial dots and applies that token's (s, z) in
//           registers: logit = sum_gr s_gr S_gr + z_gr sum(q_rot over gr).
//           q_rot is scaled to 16-bit fixed point and split into two int8
//           digits (two MMAs), exact up to the rounding of the scaled query.
//   values: O^T[16 ch][8 cols] += Vcodes^T[16 ch][16 tokens] x W[16 tokens][8 cols]
//           (mma.sync.m16n8k16, fp16 in, fp32 accumulate) with
//           W[t][(h, gr)] = p_t,h * s_t,gr (the value scale folded into the
//           weight) and the zero term sum_t p_t,h z_t,gr added at the end;
//           a channel keeps only the column of its own group.  The softmax
//           weights come out of the key MMA in the accumulator layout; one
//           movmatrix.trans per 8x8 turns them into the B operand.
//
// Data movement: a producer warp streams each (block, KV head) run of codes
// with 2-D TMA tensor copies (cp.async.bulk.tensor, no multicast) that swizzle
// 16-byte chunks across banks (64B pattern for 64-byte rows, 128B for 128-byte
// rows), and the run's scales/zeros and the block's remap mask with 1-D bulk
// copies, into a 4-deep ring of shared-memory stages guarded by mbarriers; 8
// consumer warps each take 16-token tiles of a stage.
// Every mbarrier wait is bounded: on time-out the kernel raises
// Q4KV_DEVERR_TIMEOUT, poisons the affected rows and returns.
//
// Scheduling: persistent CTAs (one per SM) walk the work items
// (sequence, KV head, split) with a static stride; the producer runs ahead
// across item boundaries.  Each item ends with a cross-warp log-sum-exp merge
// in shared memory and writes either the final row (one split) or a partial.
#include <cuda.h>   // CUtensorMap and its enums; the encoder is reached through the runtime
#include <math.h>
#include <string.h>

#include <mutex>

#include "async_copy.cuh"
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
constexpr int kStageBytes = 37 * 1024;      // 1024-byte aligned stages (128B swizzle atoms)
static_assert(kOffMeta + 32 <= kStageBytes, "stage layout");
constexpr float kLog2e = 1.4426950408889634f;

struct StageMeta {
  int32_t blk;      // unified block id, -1 if none / invalid
  int32_t tok0;     // first token of the stage within the sequence
  int16_t slot0;    // first slot within the block
  int16_t ntok;     // tokens of the stage that belong to the range
  uint8_t is8;
  uint8_t last;     // last stage of its work item
  uint8_t poison;   // the item touched a bad block id or a bad length
  uint8_t pad;
};

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_rows(void* dst, const CUtensorMap* map, int row, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(row), "r"(smem_u32(bar))
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
// keys: u8 codes x s8 query digits, exact int32 accumulation
__device__ __forceinline__ void mma_u8s8(int (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
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

// Value codes enter the fp16 MMA as exact fp16 numbers with no offset: a
// nibble or byte c masked into the low mantissa bits of a zero-exponent fp16
// is the subnormal c * 2^-24.  Rows of the value MMA for even channels carry
// c * 2^-24, rows for odd channels c * 2^-20 (a 4-bit high nibble masked in
// place is 16 c * 2^-24); each output channel therefore has one power-of-two
// scale, undone exactly in the epilogue.
__device__ __forceinline__ uint32_t lo_nib(uint32_t x) { return x & 0x000F000Fu; }   // c * 2^-24
__device__ __forceinline__ uint32_t hi_nib(uint32_t x) { return x & 0x00F000F0u; }   // c * 2^-20
__device__ __forceinline__ uint32_t byte_lo(uint32_t x) { return x & 0x00FF00FFu; }  // c * 2^-24
__device__ __forceinline__ uint32_t byte_hi(uint32_t x) {   // c * 2^-20 = (1024 + c) 2^-20 - 2^-10, exact
  return h2u(__hfma2(u2h((x & 0x00FF00FFu) | 0x64006400u), u2h(0x00100010u) /*2^-20*/,
                     u2h(0x94009400u) /*-2^-10*/));
}
constexpr float kEvenScale = 16777216.0f;   // 2^24
constexpr float kOddScale = 1048576.0f;     // 2^20

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
  static constexpr int SW = RB == 64 ? 64 : (RB == 128 ? 128 : 0);   // TMA swizzle span
  static_assert(TS * PB <= kParamBytes, "stage params");
};

// Byte offset of (row, byte) of a code tile in shared memory after the TMA
// swizzle: the 16-byte chunk index is XOR-ed with address bits 7.. (row bits).
template <int RB, int SW>
__device__ __forceinline__ int swz(int row, int byte) {
  if (SW == 128) return row * RB + ((((byte >> 4) ^ row) & 7) << 4) + (byte & 15);
  if (SW == 64) return row * RB + ((((byte >> 4) ^ (row >> 1)) & 3) << 4) + (byte & 15);
  return row * RB + byte;
}

struct TileMaps {       // one map per code array; unused ones stay zero
  CUtensorMap k4, v4, k8, v8;
};

// Key A operand (u8) of 32-channel step kk for the thread's two rows.  Thread
// t owns channels 128c + 32t + [0, 32) of each row (c < D/128); step kk uses
// chunk c = kk/4 and its 8-channel word w = kk%4: register 0 (k = 4t .. 4t+3)
// holds channels 8w + {0, 2, 4, 6}, register 2 (k = 16 + 4t ..) 8w + {1, 3, 5, 7}.
template <bool Q8>
__device__ __forceinline__ void key_a8(const uint32_t* rg, const uint32_t* rg8, int kk, uint32_t (&a)[4]) {
  if (!Q8) {
    // a 4-bit word holds elements 0..7 at nibbles 0..7: the low nibbles are 0, 2, 4, 6
    const uint32_t x0 = rg[kk], x1 = rg8[kk];
    a[0] = x0 & 0x0F0F0F0Fu;
    a[1] = x1 & 0x0F0F0F0Fu;
    a[2] = (x0 >> 4) & 0x0F0F0F0Fu;
    a[3] = (x1 >> 4) & 0x0F0F0F0Fu;
  } else {
    // 8-bit: channels 8w .. 8w+3 in word 2w, 8w+4 .. 8w+7 in word 2w+1
    a[0] = __byte_perm(rg[2 * kk], rg[2 * kk + 1], 0x6420);
    a[1] = __byte_perm(rg8[2 * kk], rg8[2 * kk + 1], 0x6420);
    a[2] = __byte_perm(rg[2 * kk], rg[2 * kk + 1], 0x7531);
    a[3] = __byte_perm(rg8[2 * kk], rg8[2 * kk + 1], 0x7531);
  }
}

// Token order inside a 16-token tile: accumulator row r holds token pi(r),
// pi swapping 2 <-> 3 and 6 <-> 7 in each half.  With it the four value rows a
// thread reads at one time fall on both 64-byte halves of the 128-byte bank
// window, halving shared-memory bank conflicts; any permutation is correct
// because both contractions sum over tokens.
__device__ __forceinline__ int tok_perm(int r) { return r ^ ((r >> 1) & 1); }

// Value A operands for one 16-token tile: tokens T = pi(2t), pi(2t+1),
// pi(2t+8), pi(2t+9) of the tile, thread g's channels cb + [0, D/8).  Tile mv
// (channels) uses rows g -> cb + 2 mv and g + 8 -> cb + 2 mv + 1.  The codes
// enter the MMA as exact fp16 subnormals (see lo_nib); an offset form
// (1024 + code) would make the accumulator carry ~1024 x the weight sum and
// lose accuracy over long contexts.
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
    a[0] = byte_lo(__byte_perm(v0[wi], v1[wi], sa));
    a[1] = byte_hi(__byte_perm(v0[wi], v1[wi], sb));
    a[2] = byte_lo(__byte_perm(v8[wi], v9[wi], sa));
    a[3] = byte_hi(__byte_perm(v8[wi], v9[wi], sb));
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

// Per-thread byte offsets inside a stage for the warp's first tile.  Tiles
// start at multiples of 16 rows, so the token permutation and the TMA
// swizzle depend only on the row's low four bits -- a per-thread constant --
// and tile i of the warp sits a compile-time 128 * i rows further on.
// Computing these once keeps address arithmetic out of the tile loop.
template <int D, bool Q8>
struct TileOffsets {
  using G = Geo<D, Q8>;
  static constexpr int NC = D / 128;                        // 128-channel chunks
  static constexpr int NQ = G::KB / NC / 16;                // 16-byte key loads per chunk
  int k[2][NC * NQ];   // key rows pi(g), pi(g + 8)
  int v[4];            // value rows pi(2t), pi(2t+1), pi(2t+8), pi(2t+9) (thread g's bytes)
  int p[2];            // parameter rows pi(g), pi(g + 8) (the thread's two groups)
  int row[2];          // pi(g), pi(g + 8) relative to the warp's first tile

  __device__ __forceinline__ void init(int warp, int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int r0 = warp * 16;
    const int rr[2] = {tok_perm(g), tok_perm(g + 8)};
#pragma unroll
    for (int x = 0; x < 2; ++x) {
      row[x] = r0 + rr[x];
#pragma unroll
      for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          k[x][c * NQ + q] = swz<G::RB, G::SW>(row[x], c * (G::RB / NC) + t * (G::KB / NC) + q * 16);
      p[x] = row[x] * G::PB + ((G::NG == 2) ? 0 : 2 * (t & 1)) * 4;
    }
    const int vr[4] = {tok_perm(2 * t), tok_perm(2 * t + 1), tok_perm(2 * t + 8), tok_perm(2 * t + 9)};
#pragma unroll
    for (int x = 0; x < 4; ++x) v[x] = swz<G::RB, G::SW>(r0 + vr[x], g * G::VB);
  }
};

// NTILE 16-token tiles of one stage: keys for every tile, one online-softmax
// update over all of them, then values.  The running max moves only when the
// tile max exceeds it by more than kLazy (log2 units), so the accumulators are
// rescaled rarely; weights stay <= 2^kLazy.
constexpr float kLazy = 2.0f;

template <int D, int NT, bool Q8, int NTILE>
__device__ __forceinline__ void tiles(WarpState<D, NT>& st, const uint8_t* stage,
                                      const TileOffsets<D, Q8>& o, int nvalid,
                                      const uint32_t (&bq)[D / 32][NT][2][2],
                                      const float (&qs)[NT][2], const float (&ks)[NT], int lane) {
  using G = Geo<D, Q8>;
  using O = TileOffsets<D, Q8>;
  constexpr int kTileRows = kCW * 16;   // rows between a warp's tiles
  // ---- keys ----
  float sk[NTILE][NT][4];
#pragma unroll
  for (int i = 0; i < NTILE; ++i) {
    uint32_t rg[G::KB / 4], rg8[G::KB / 4];
    const uint8_t* base = stage + i * kTileRows * G::RB;
#pragma unroll
    for (int n = 0; n < O::NC * O::NQ; ++n) {
      const uint4 u = lds<uint4>(base + o.k[0][n]), u8 = lds<uint4>(base + o.k[1][n]);
      rg[4 * n] = u.x; rg[4 * n + 1] = u.y; rg[4 * n + 2] = u.z; rg[4 * n + 3] = u.w;
      rg8[4 * n] = u8.x; rg8[4 * n + 1] = u8.y; rg8[4 * n + 2] = u8.z; rg8[4 * n + 3] = u8.w;
    }
    int hi[NT][4], lo[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) hi[j][e] = lo[j][e] = 0;
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk) {
      uint32_t a[4];
      key_a8<Q8>(rg, rg8, kk, a);
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        mma_u8s8(hi[j], a, bq[kk][j][1][0], bq[kk][j][1][1]);
        mma_u8s8(lo[j], a, bq[kk][j][0][0], bq[kk][j][0][1]);
      }
    }
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) sk[i][j][e] = static_cast<float>(hi[j][e] * 256 + lo[j][e]);
  }
  // ---- per-token parameters and logits (log2 units) ----
  // D = 128: the thread's columns are (h, 0), (h, 1); D = 256: (h, 2 (t%2)), (h, 2 (t%2) + 1).
  const uint32_t* mask = reinterpret_cast<const uint32_t*>(stage + kOffMask);
  const int slot0 = reinterpret_cast<const StageMeta*>(stage + kOffMeta)->slot0;
  float logit[NTILE][NT][2];
  float ws[NTILE][2][2], wz[NTILE][2][2];   // [tile][row][e]: value scale, zero (0 unless live)
  bool live[NTILE][2];
#pragma unroll
  for (int i = 0; i < NTILE; ++i) {
    // the tile's 16 mask bits: slots slot0 + first row .. + 15 (16-aligned)
    const int s16 = slot0 + o.row[0] - tok_perm((lane >> 2)) + i * kTileRows;   // first slot of the tile
    const uint32_t mbits = mask[s16 >> 5] >> (s16 & 16);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = o.row[r] + i * kTileRows;
      const bool valid = row < nvalid;
      const bool masked = valid && ((mbits >> (row & 15)) & 1u);
      const bool lv = valid && !masked;
      live[i][r] = lv;
      const uint2 kpw = lds<uint2>(stage + kOffKP + o.p[r] + i * kTileRows * G::PB);
      const uint2 vpw = lds<uint2>(stage + kOffVP + o.p[r] + i * kTileRows * G::PB);
      const float2 k0 = __half22float2(u2h(kpw.x)), k1 = __half22float2(u2h(kpw.y));
      const float2 v0 = __half22float2(u2h(vpw.x)), v1 = __half22float2(u2h(vpw.y));
      // rows outside the range or remapped may hold any bytes (even NaN
      // parameters): select, never multiply, them away
      ws[i][r][0] = lv ? v0.x : 0.0f;
      wz[i][r][0] = lv ? v0.y : 0.0f;
      ws[i][r][1] = lv ? v1.x : 0.0f;
      wz[i][r][1] = lv ? v1.y : 0.0f;
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        float part = __fmaf_rn(k0.x, sk[i][j][2 * r], k1.x * sk[i][j][2 * r + 1]) * ks[j] +
                     __fmaf_rn(k0.y, qs[j][0], k1.y * qs[j][1]);
        if (G::NG == 4) part += __shfl_xor_sync(0xffffffffu, part, 1);
        logit[i][j][r] = !valid ? -INFINITY : (masked ? Q4KV_SENTINEL_LOGIT * kLog2e : part);
      }
    }
  }
  // ---- online softmax over the NTILE tiles ----
  uint32_t wb[NTILE][NT][2];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < NTILE; ++i) mx = fmaxf(mx, fmaxf(logit[i][j][0], logit[i][j][1]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (mx > st.m[j] + kLazy) {          // also taken on the first live tile (m = -inf)
      const float alpha = ex2(st.m[j] - mx);
      st.m[j] = mx;
      st.l[j] *= alpha;
      st.z[j][0] *= alpha;
      st.z[j][1] *= alpha;
#pragma unroll
      for (int mv = 0; mv < D / 16; ++mv)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.o[mv][j][e] *= alpha;
    }
    const float m = st.m[j];
    float lsum = 0.0f, z0 = 0.0f, z1 = 0.0f;
#pragma unroll
    for (int i = 0; i < NTILE; ++i) {
      float p[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        p[r] = logit[i][j][r] == -INFINITY ? 0.0f : ex2(logit[i][j][r] - m);
        lsum += p[r];
        const float q = live[i][r] ? p[r] : 0.0f;
        z0 = __fmaf_rn(q, wz[i][r][0], z0);
        z1 = __fmaf_rn(q, wz[i][r][1], z1);
        wb[i][j][r] = h2u(__floats2half2_rn(q * ws[i][r][0], q * ws[i][r][1]));
      }
    }
    st.l[j] += lsum;
    st.z[j][0] += z0;
    st.z[j][1] += z1;
  }
  // ---- values ----
  constexpr int VW = G::VB / 4;   // words of value codes per token row
#pragma unroll
  for (int i = 0; i < NTILE; ++i) {
    uint32_t bw[NT][2];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      bw[j][0] = movtrans(wb[i][j][0]);   // tokens pi(2t), pi(2t+1)
      bw[j][1] = movtrans(wb[i][j][1]);   // tokens pi(8+2t), pi(9+2t)
    }
    uint32_t v0[VW], v1[VW], v8[VW], v9[VW];
    const uint8_t* vc = stage + kOffV + i * kTileRows * G::RB;
    if (VW == 2) {
      const uint2 a0 = lds<uint2>(vc + o.v[0]), a1 = lds<uint2>(vc + o.v[1]);
      const uint2 a8 = lds<uint2>(vc + o.v[2]), a9 = lds<uint2>(vc + o.v[3]);
      v0[0] = a0.x; v0[1] = a0.y; v1[0] = a1.x; v1[1] = a1.y;
      v8[0] = a8.x; v8[1] = a8.y; v9[0] = a9.x; v9[1] = a9.y;
    } else {
#pragma unroll
      for (int q = 0; q < VW; q += 4) {   // 16-byte pieces of the thread's bytes (never swizzle-split)
        const uint4 a0 = lds<uint4>(vc + o.v[0] + 4 * q), a1 = lds<uint4>(vc + o.v[1] + 4 * q);
        const uint4 a8 = lds<uint4>(vc + o.v[2] + 4 * q), a9 = lds<uint4>(vc + o.v[3] + 4 * q);
        v0[q] = a0.x; v0[q + 1] = a0.y; v0[q + 2] = a0.z; v0[q + 3] = a0.w;
        v1[q] = a1.x; v1[q + 1] = a1.y; v1[q + 2] = a1.z; v1[q + 3] = a1.w;
        v8[q] = a8.x; v8[q + 1] = a8.y; v8[q + 2] = a8.z; v8[q + 3] = a8.w;
        v9[q] = a9.x; v9[q + 1] = a9.y; v9[q + 2] = a9.z; v9[q + 3] = a9.w;
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
}

// ---------------------------------------------------------------------------
// FP8 comparison cache: OCP E4M3 keys and values, no params, raw keys.  Both
// contractions run as fp16 MMAs: a code pair becomes an exact f16x2 with one
// conversion, the query (pre-scaled by scale * log2 e) enters as fp16 high +
// low parts (two MMAs, ~22 bits), and a B column is one query head.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t pair16) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(pair16 & 0xFFFFu),
                                                   __NV_E4M3);
  return static_cast<uint32_t>(h.x) | (static_cast<uint32_t>(h.y) << 16);
}

template <int D>
struct Fp8State {
  float o[D / 16][4];   // value accumulators (channels x heads)
  float m[2];           // running max of the thread's two heads (columns 2t, 2t+1), log2 units
  float l[2];           // this thread's share of their running sums
};

template <int D>
__device__ __forceinline__ void reset(Fp8State<D>& st) {
#pragma unroll
  for (int mv = 0; mv < D / 16; ++mv)
#pragma unroll
    for (int e = 0; e < 4; ++e) st.o[mv][e] = 0.0f;
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = 0.0f;
}

// NTILE tiles of an FP8 stage (8-bit geometry).  qtab: this thread's entries
// of the query table, entry ks at qtab[ks * 4] = (high b0, high b1, low b0,
// low b1) for channels 128 (ks / 8) + 32 t + 4 (ks % 8) + 0..3 of head g.
template <int D, int NTILE>
__device__ __forceinline__ void fp8_tiles(Fp8State<D>& st, const uint8_t* stage,
                                          const TileOffsets<D, true>& o, int nvalid,
                                          const uint4* __restrict__ qtab, int lane) {
  using G = Geo<D, true>;
  using O = TileOffsets<D, true>;
  constexpr int kTileRows = kCW * 16;
  float sk[NTILE][4];
#pragma unroll
  for (int i = 0; i < NTILE; ++i) {
    uint32_t rg[G::KB / 4], rg8[G::KB / 4];
    const uint8_t* base = stage + i * kTileRows * G::RB;
#pragma unroll
    for (int n = 0; n < O::NC * O::NQ; ++n) {
      const uint4 u = lds<uint4>(base + o.k[0][n]), u8 = lds<uint4>(base + o.k[1][n]);
      rg[4 * n] = u.x; rg[4 * n + 1] = u.y; rg[4 * n + 2] = u.z; rg[4 * n + 3] = u.w;
      rg8[4 * n] = u8.x; rg8[4 * n + 1] = u8.y; rg8[4 * n + 2] = u8.z; rg8[4 * n + 3] = u8.w;
    }
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t a[4];
      a[0] = e4m3x2_f16x2(rg[ks]);         // row g, channels +0, +1
      a[1] = e4m3x2_f16x2(rg8[ks]);        // row g + 8
      a[2] = e4m3x2_f16x2(rg[ks] >> 16);   // row g, channels +2, +3
      a[3] = e4m3x2_f16x2(rg8[ks] >> 16);
      const uint4 b = qtab[ks * 4];
      mma16816(acc, a, b.x, b.y);
      mma16816(acc, a, b.z, b.w);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) sk[i][e] = acc[e];
  }
  // logits (log2 units; the query carries scale * log2 e): acc e = (row e / 2, column 2t + e % 2)
  const uint32_t* mask = reinterpret_cast<const uint32_t*>(stage + kOffMask);
  const int slot0 = reinterpret_cast<const StageMeta*>(stage + kOffMeta)->slot0;
  float logit[NTILE][2][2];   // [tile][row][column]
  bool live[NTILE][2];
#pragma unroll
  for (int i = 0; i < NTILE; ++i) {
    const int s16 = slot0 + o.row[0] - tok_perm((lane >> 2)) + i * kTileRows;
    const uint32_t mbits = mask[s16 >> 5] >> (s16 & 16);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = o.row[r] + i * kTileRows;
      const bool valid = row < nvalid;
      const bool masked = valid && ((mbits >> (row & 15)) & 1u);
      live[i][r] = valid && !masked;
#pragma unroll
      for (int c = 0; c < 2; ++c)
        logit[i][r][c] = !valid ? -INFINITY : (masked ? Q4KV_SENTINEL_LOGIT * kLog2e : sk[i][2 * r + c]);
    }
  }
  // online softmax per column (head), lazy rescale
  float alpha[2] = {1.0f, 1.0f};
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < NTILE; ++i) mx = fmaxf(mx, fmaxf(logit[i][0][c], logit[i][1][c]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (mx > st.m[c] + kLazy) {
      alpha[c] = ex2(st.m[c] - mx);
      st.m[c] = mx;
      st.l[c] *= alpha[c];
    }
  }
  if (alpha[0] != 1.0f || alpha[1] != 1.0f) {
#pragma unroll
    for (int mv = 0; mv < D / 16; ++mv) {
      st.o[mv][0] *= alpha[0];
      st.o[mv][1] *= alpha[1];
      st.o[mv][2] *= alpha[0];
      st.o[mv][3] *= alpha[1];
    }
  }
  constexpr int VW = G::VB / 4;
#pragma unroll
  for (int i = 0; i < NTILE; ++i) {
    uint32_t wb[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      float p[2];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        p[c] = logit[i][r][c] == -INFINITY ? 0.0f : ex2(logit[i][r][c] - st.m[c]);
        st.l[c] += p[c];
      }
      // a remapped slot's value is 0 (its weight still counts in the sum);
      // rows past the range may hold any bytes: selected away
      wb[r] = live[i][r] ? h2u(__floats2half2_rn(p[0], p[1])) : 0u;
    }
    const uint32_t bw0 = movtrans(wb[0]), bw1 = movtrans(wb[1]);
    uint32_t v0[VW], v1[VW], v8[VW], v9[VW];
    const uint8_t* vc = stage + kOffV + i * kTileRows * G::RB;
#pragma unroll
    for (int q = 0; q < VW; q += 4) {
      const uint4 a0 = lds<uint4>(vc + o.v[0] + 4 * q), a1 = lds<uint4>(vc + o.v[1] + 4 * q);
      const uint4 a8 = lds<uint4>(vc + o.v[2] + 4 * q), a9 = lds<uint4>(vc + o.v[3] + 4 * q);
      v0[q] = a0.x; v0[q + 1] = a0.y; v0[q + 2] = a0.z; v0[q + 3] = a0.w;
      v1[q] = a1.x; v1[q + 1] = a1.y; v1[q + 2] = a1.z; v1[q + 3] = a1.w;
      v8[q] = a8.x; v8[q + 1] = a8.y; v8[q + 2] = a8.z; v8[q + 3] = a8.w;
      v9[q] = a9.x; v9[q + 1] = a9.y; v9[q + 2] = a9.z; v9[q + 3] = a9.w;
    }
#pragma unroll
    for (int mv = 0; mv < D / 16; ++mv) {
      // byte 2 mv of the thread's run = channel cb + 2 mv, byte 2 mv + 1 = cb + 2 mv + 1
      const int wi = (2 * mv) / 4, bp = (2 * mv) % 4;
      const uint32_t sa = bp | ((bp + 4) << 4), sb = (bp + 1) | ((bp + 5) << 4);   // [T0.b, T1.b]
      uint32_t a[4];
      a[0] = e4m3x2_f16x2(__byte_perm(v0[wi], v1[wi], sa));
      a[1] = e4m3x2_f16x2(__byte_perm(v0[wi], v1[wi], sb));
      a[2] = e4m3x2_f16x2(__byte_perm(v8[wi], v9[wi], sa));
      a[3] = e4m3x2_f16x2(__byte_perm(v8[wi], v9[wi], sb));
      mma16816(st.o[mv], a, bw0, bw1);
    }
  }
}

// Raw 16-bit query elements E*lane .. E*lane + E-1 of head `h` of item's
// (sequence, KV head) group, as loaded (E = 4: 8 bytes, E = 8: 16 bytes).
template <int E>
__device__ __forceinline__ uint4 load_query(const DecodeArgs& a, int item, int S, int hkv, int hq, int G,
                                            int h, int lane) {
  const int kvh = (item / S) % hkv;
  const int b = item / (S * hkv);
  const int64_t qi = (static_cast<int64_t>(b) * hq + kvh * G + h) * (E * 32) + E * lane;
  const uint8_t* p = static_cast<const uint8_t*>(a.q) + 2 * qi;
  if (E == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    return make_uint4(w.x, w.y, 0u, 0u);
  }
  return *reinterpret_cast<const uint4*>(p);
}

template <int D, int NT, bool FP8 = false>
__global__ void __launch_bounds__(kThreadsTC, 1)
    decode_tc_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ TileMaps maps,
                     int n_items) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // swizzled TMA tiles need 1024-byte aligned destinations
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kNS * kStageBytes);
  uint64_t* empty = full + kNS;
  float* qrot = reinterpret_cast<float*>(empty + kNS);                 // query digit table, 2 G D bytes
  float* qsum = qrot + 8 * D;                                          // [8][4] sums, [32 + h] scales
  float* mrg_ml = qsum + 64;                                           // [kCW][8][2]
  float* mrg_o = mrg_ml + kCW * 16;                                    // [kCW][G][D]
  __shared__ int s_flags[2];                                            // poison, timeout

  griddep_wait();   // earlier kernels in the stream (the encoder) have finished
  griddep_launch_dependents();
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
        // A stage that stays taken past the limit ends production: writing
        // the stage or arriving on its full barrier could then land in a
        // phase the consumers have not finished.  Their own bounded waits
        // run out in turn and they report the timeout.
        if (!mbar_wait(&empty[s], ((it / kNS) & 1) ^ 1)) {
          gave_up = true;
          break;
        }
        uint8_t* stg = stages + s * kStageBytes;
        StageMeta meta;
        meta.tok0 = tok;
        meta.poison = bad_seq;
        meta.pad = 0;
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
        if (meta.blk >= 0) {
          const int rows = (meta.ntok + 15) & ~15;   // whole 16-token tiles, inside the block
          const bool is8 = meta.is8;
          const int64_t phys = is8 ? meta.blk - P.n_q4 : meta.blk;
          const int64_t row = (phys * hkv + kvh) * kBlockTokens + meta.slot0;
          const int rb = is8 ? D : D / 2, pb = (D / kGroup) * 4;
          const uint8_t* kc = (is8 ? P.k_codes8 : P.k_codes4) + row * rb;
          const uint8_t* vc = (is8 ? P.v_codes8 : P.v_codes4) + row * rb;
          const uint8_t* kpp = reinterpret_cast<const uint8_t*>(is8 ? P.k_params8 : P.k_params4) + row * pb;
          const uint8_t* vpp = reinterpret_cast<const uint8_t*>(is8 ? P.v_params8 : P.v_params4) + row * pb;
          // codes: one TS-row box per tensor (the box never leaves the block)
          const int ts = is8 ? Geo<D, true>::TS : Geo<D, false>::TS;
          const uint32_t cb = static_cast<uint32_t>(ts) * rb, prb = FP8 ? 0u : rows * pb;   // FP8: no params
          mbar_arrive_tx(&full[s], 2 * cb + 2 * prb + 32);
          tma_rows(stg, is8 ? &maps.k8 : &maps.k4, static_cast<int>(row), &full[s]);
          tma_rows(stg + kOffV, is8 ? &maps.v8 : &maps.v4, static_cast<int>(row), &full[s]);
          (void)kc;
          (void)vc;
          if (!FP8) {
            bulk_g2s(stg + kOffKP, kpp, prb, &full[s]);
            bulk_g2s(stg + kOffVP, vpp, prb, &full[s]);
          }
          bulk_g2s(stg + kOffMask, P.mask + static_cast<int64_t>(meta.blk) * kMaskWords, 32, &full[s]);
        } else {
          mbar_arrive(&full[s]);
        }
        ++it;
        tok += step;
      } while (tok < t1);
      if (gave_up) break;
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
  uint32_t bq[D / 32][NT][2][2];   // [step][n-tile][digit][register]
  float qs[NT][2], ks[NT];
  uint32_t it = 0;
  bool dead = false;
  TileOffsets<D, false> off4;
  off4.init(warp, lane);
  // FP8: query table [head][ks][t] of (high b0, high b1, low b0, low b1);
  // heads past G stay zero
  Fp8State<D> fst;
  TileOffsets<D, true> off8f;
  uint4* qtab = reinterpret_cast<uint4*>(qrot);
  const uint4* qtab_t = qtab + g * (D / 16) * 4 + t;
  if constexpr (FP8) {
    off8f.init(warp, lane);
    for (int i = threadIdx.x; i < 8 * (D / 16) * 4; i += kCW * 32) qtab[i] = make_uint4(0u, 0u, 0u, 0u);
    consumer_sync();
  }

  uint4 qraw = make_uint4(0u, 0u, 0u, 0u);   // raw query of the warp's head for the coming item
  if (warp < G && blockIdx.x < n_items) qraw = load_query<D / 32>(a, blockIdx.x, S, hkv, hq, G, warp, lane);
  for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int split = item % S;
    const int kvh = (item / S) % hkv;
    const int b = item / (S * hkv);
    // ---- warp h < G: rotate query head h in registers, scale it to 16-bit
    // fixed point (max |q_rot| * 2^E <= 32000) and sum it per group ----
    if (warp < G) {
      constexpr int E = D / 32;                   // lane holds channels E*lane .. E*lane + E-1
      float x[E];
      const uint4 w = qraw;
      // the next item's query is loaded now, behind this item's stages
      const int nitem = item + gridDim.x;
      if (nitem < n_items) qraw = load_query<E>(a, nitem, S, hkv, hq, G, warp, lane);
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const uint32_t h16 = (ww[e / 2] >> (16 * (e % 2))) & 0xFFFFu;
        x[e] = a.q_dtype == Q4KV_F16 ? __half2float(__ushort_as_half(static_cast<unsigned short>(h16)))
                                     : __uint_as_float(h16 << 16);
      }
      if constexpr (FP8) {
        // q * scale * log2 e as fp16 high + low parts, in the B layout of the
        // key MMA: entry (head, ks, t) covers channels 128 (ks / 8) + 32 t + 4 (ks % 8) + 0..3
        uint32_t hw[E / 2], lw[E / 2];
#pragma unroll
        for (int p2 = 0; p2 < E / 2; ++p2) {
          const float y0 = x[2 * p2] * sc2, y1 = x[2 * p2 + 1] * sc2;
          const __half2 hi = __floats2half2_rn(y0, y1);
          const float2 hf = __half22float2(hi);
          hw[p2] = h2u(hi);
          lw[p2] = h2u(__floats2half2_rn(y0 - hf.x, y1 - hf.y));
        }
        if constexpr (E == 4) {   // channels 4 lane + 0..3: ks = lane % 8, t = lane / 8
          qtab[(warp * (D / 16) + (lane & 7)) * 4 + (lane >> 3)] = make_uint4(hw[0], hw[1], lw[0], lw[1]);
        } else {                  // channels 8 lane + 0..7: two entries
          const int ks0 = 8 * (lane >> 4) + 2 * (lane & 3), tt = (lane & 15) >> 2;
          qtab[(warp * (D / 16) + ks0) * 4 + tt] = make_uint4(hw[0], hw[1], lw[0], lw[1]);
          qtab[(warp * (D / 16) + ks0 + 1) * 4 + tt] = make_uint4(hw[2], hw[3], lw[2], lw[3]);
        }
      } else {
      if (P.k_rotated) {   // c * H q: butterflies inside the lane, then across lanes (fp32)
#pragma unroll
        for (int h = 1; h < E; h <<= 1)
#pragma unroll
          for (int e = 0; e < E; ++e)
            if ((e & h) == 0) {
              const float u = x[e], v = x[e + h];
              x[e] = u + v;
              x[e + h] = u - v;
            }
#pragma unroll
        for (int h = E; h < D; h <<= 1) {
          const int lb = h / E;
          const bool upper = (lane & lb) != 0;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float o = __shfl_xor_sync(0xffffffffu, x[e], lb);
            x[e] = upper ? o - x[e] : x[e] + o;
          }
        }
        const float c = rotation_constant(D);
#pragma unroll
        for (int e = 0; e < E; ++e) x[e] *= c;
      }
      float mx = 0.0f;
#pragma unroll
      for (int e = 0; e < E; ++e) mx = fmaxf(mx, fabsf(x[e]));
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      int ex = 0;
      if (mx > 0.0f) ex = static_cast<int>(floorf(log2f(32000.0f / mx)));
      ex = max(-100, min(100, ex));
      // digits of the fixed-point query, written straight into the B-operand
      // table: entry (h, kk, t) is 16 bytes = words (low digit, r = 0),
      // (low, r = 1), (high, r = 0), (high, r = 1); byte e of word r is the
      // digit of channel 128 (kk / 4) + 32 t + 8 (kk % 4) + r + 2 e.  With
      // q = 256 hi + lo, lo in [-128, 127]: lo = q mod 256, hi = (q + 128) >> 8.
      float part = 0.0f;
      uint32_t lo8[E], hi8[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const float qf = rintf(ldexpf(x[e], ex));
        part += qf;
        const int qv = static_cast<int>(qf);
        lo8[e] = static_cast<uint32_t>(qv) & 255u;
        hi8[e] = static_cast<uint32_t>((qv + 128) >> 8) & 255u;
      }
      uint8_t* tbl = reinterpret_cast<uint8_t*>(qrot) + warp * (D / 32) * 64;
      if constexpr (E == 8) {   // lane = channels 8 lane + [0, 8): kk = 4 (lane / 16) + lane % 4, t = (lane / 4) % 4
        const int kk = 4 * (lane >> 4) + (lane & 3), tt = (lane >> 2) & 3;
        uint4 w;
        w.x = lo8[0] | lo8[2] << 8 | lo8[4] << 16 | lo8[6] << 24;
        w.y = lo8[1] | lo8[3] << 8 | lo8[5] << 16 | lo8[7] << 24;
        w.z = hi8[0] | hi8[2] << 8 | hi8[4] << 16 | hi8[6] << 24;
        w.w = hi8[1] | hi8[3] << 8 | hi8[5] << 16 | hi8[7] << 24;
        *reinterpret_cast<uint4*>(tbl + (kk * 4 + tt) * 16) = w;
      } else {        // lane = channels 4 lane + [0, 4): bytes 2 (lane % 2), +1 of each word
        const int kk = (lane >> 1) & 3, tt = lane >> 3;
        uint16_t* h16 = reinterpret_cast<uint16_t*>(tbl + (kk * 4 + tt) * 16) + (lane & 1);
        h16[0] = static_cast<uint16_t>(lo8[0] | lo8[2] << 8);
        h16[2] = static_cast<uint16_t>(lo8[1] | lo8[3] << 8);
        h16[4] = static_cast<uint16_t>(hi8[0] | hi8[2] << 8);
        h16[6] = static_cast<uint16_t>(hi8[1] | hi8[3] << 8);
      }
      // exact group sums: the 64 / E lanes of a group are consecutive
#pragma unroll
      for (int off = 1; off < kGroup / E; off <<= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      if (lane % (kGroup / E) == 0) qsum[warp * 4 + lane / (kGroup / E)] = part;
      if (lane == 0) qsum[32 + warp] = ldexpf(1.0f, -ex);        // 2^-E of head `warp`
      }
    }
    consumer_sync();
#pragma unroll
    for (int j = 0; j < (FP8 ? 0 : NT); ++j) {
      const int col = 8 * j + g;                // this thread's B column
      const int h = col / NG, gr = col % NG;
      const uint4* tbl = reinterpret_cast<const uint4*>(qrot) + (h < G ? h : 0) * (D / 32) * 4 + t;
#pragma unroll
      for (int kk = 0; kk < D / 32; ++kk) {
        // channels of step kk for this t lie in group 2 (kk / 4) + t / 2
        const bool use = h < G && 2 * (kk / 4) + (t >> 1) == gr;
        uint4 w = tbl[kk * 4];
        if (!use) w = make_uint4(0u, 0u, 0u, 0u);
        bq[kk][j][0][0] = w.x;
        bq[kk][j][0][1] = w.y;
        bq[kk][j][1][0] = w.z;
        bq[kk][j][1][1] = w.w;
      }
      {
        const int c2 = 8 * j + 2 * t;             // the thread's accumulator columns c2, c2 + 1
        const int h2 = c2 / NG;
        const float sc = h2 < G ? sc2 * qsum[32 + h2] : 0.0f;
        ks[j] = sc;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int g2 = (c2 + e) % NG;
          qs[j][e] = h2 < G ? qsum[h2 * 4 + g2] * sc : 0.0f;
        }
      }
    }
    if constexpr (FP8) reset(fst);
    else reset(st);
    bool poison = false, timeout = false;

    // ---- the item's stages ----
    for (;;) {
      const int s = it % kNS;
      if (!dead && !mbar_wait(&full[s], (it / kNS) & 1)) dead = true;
      const uint8_t* stg = stages + s * kStageBytes;
      const StageMeta meta = *reinterpret_cast<const StageMeta*>(stg + kOffMeta);
      const bool last = dead ? true : meta.last;
      timeout |= dead;
      poison |= meta.poison;
      if (!dead && meta.blk >= 0 && warp * 16 < meta.ntok) {
        // warp w takes the stage's tiles w, w + 8, ... (rows past ntok are masked)
        if constexpr (FP8) {
          constexpr int NTL = Geo<D, true>::MTILES >= kCW ? Geo<D, true>::MTILES / kCW : 1;
          if (warp < Geo<D, true>::MTILES) fp8_tiles<D, NTL>(fst, stg, off8f, meta.ntok, qtab_t, lane);
        } else if (!meta.is8) {
          constexpr int NTL = Geo<D, false>::MTILES / kCW;
          tiles<D, NT, false, NTL>(st, stg, off4, meta.ntok, bq, qs, ks, lane);
        } else if (warp < Geo<D, true>::MTILES) {
          constexpr int NTL = Geo<D, true>::MTILES >= kCW ? Geo<D, true>::MTILES / kCW : 1;
          TileOffsets<D, true> off8;   // 8-bit blocks are rare: offsets made on demand
          off8.init(warp, lane);
          tiles<D, NT, true, NTL>(st, stg, off8, meta.ntok, bq, qs, ks, lane);
        }
      }
      __syncwarp();
      if (lane == 0 && !dead) mbar_arrive(&empty[s]);
      ++it;
      if (last) break;
    }
    if (timeout && threadIdx.x == 0) raise_error(P.error_word, Q4KV_DEVERR_TIMEOUT);

    // ---- cross-warp merge of the item ----
    if constexpr (FP8) {
      float lt[2] = {fst.l[0], fst.l[1]};
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        lt[0] += __shfl_xor_sync(0xffffffffu, lt[0], off);
        lt[1] += __shfl_xor_sync(0xffffffffu, lt[1], off);
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int h = 2 * t + c;
        if (g == 0 && h < G) {
          mrg_ml[(warp * 8 + h) * 2] = fst.m[c];
          mrg_ml[(warp * 8 + h) * 2 + 1] = lt[c];
        }
      }
#pragma unroll
      for (int mv = 0; mv < D / 16; ++mv)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int ch = (D / 8) * g + 2 * mv + (e >> 1), h = 2 * t + (e & 1);
          if (h < G) mrg_o[(warp * G + h) * D + ch] = fst.o[mv][e];
        }
    }
#pragma unroll
    for (int j = 0; j < (FP8 ? 0 : NT); ++j) {
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
            mrg_o[(warp * G + hh) * D + ch] = __fmaf_rn(st.o[mv][j][e], e < 2 ? kEvenScale : kOddScale, zz[e & 1]);
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
  return 1024 + static_cast<size_t>(kNS) * kStageBytes + 2 * kNS * sizeof(uint64_t) +
         (8 * head_dim + 64 + kCW * 16) * sizeof(float) + static_cast<size_t>(kCW) * 1024 * sizeof(float);
}

namespace {

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn tensor_map_encoder() {
  static std::once_flag once;
  static EncodeFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

// Rows of `row_bytes` codes, `box_rows` rows per copy.
bool encode_rows(EncodeFn enc, CUtensorMap* m, void* base, uint64_t rows, uint32_t row_bytes,
                 uint32_t box_rows) {
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {row_bytes, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = row_bytes == 64    ? CU_TENSOR_MAP_SWIZZLE_64B
                                : row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                                   : CU_TENSOR_MAP_SWIZZLE_NONE;
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeArgs& a, int num_sms, cudaStream_t stream) {
  const q4kv_decode_plan& p = a.plan;
  const int n_items = p.batch * p.n_kv_heads * p.n_splits;
  const int grid = min(n_items, num_sms);
  const int g = p.n_q_heads / p.n_kv_heads;
  const int nt = (g * (p.head_dim / kGroup) + 7) / 8;
  const size_t smem = decode_tc_smem_bytes(p.head_dim);

  EncodeFn enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  TileMaps maps;
  memset(&maps, 0, sizeof(maps));
  const int d = p.head_dim;
  const uint64_t per_block = static_cast<uint64_t>(a.pool.n_kv_heads) * kBlockTokens;
  const uint32_t ts4 = static_cast<uint32_t>(kCodeBytes / (d / 2)), ts8 = static_cast<uint32_t>(kCodeBytes / d);
  if (a.pool.n_q4 > 0 &&
      (!encode_rows(enc, &maps.k4, a.pool.k_codes4, a.pool.n_q4 * per_block, d / 2, ts4) ||
       !encode_rows(enc, &maps.v4, a.pool.v_codes4, a.pool.n_q4 * per_block, d / 2, ts4)))
    return cudaErrorInvalidValue;
  if (a.pool.n_q8 > 0 &&
      (!encode_rows(enc, &maps.k8, a.pool.k_codes8, a.pool.n_q8 * per_block, d, ts8) ||
       !encode_rows(enc, &maps.v8, a.pool.v_codes8, a.pool.n_q8 * per_block, d, ts8)))
    return cudaErrorInvalidValue;

  cudaError_t e = cudaSuccess;
#define Q4KV_TC(DD, NN, F8)                                                                        \
  do {                                                                                             \
    e = cudaFuncSetAttribute(decode_tc_kernel<DD, NN, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             static_cast<int>(smem));                                              \
    if (e == cudaSuccess)                                                                          \
      e = launch_pdl(decode_tc_kernel<DD, NN, F8>, dim3(grid), dim3(kThreadsTC), smem, stream, a, maps, \
                     n_items);                                                                     \
  } while (0)
  if (a.pool.fp8 && p.head_dim == 128) Q4KV_TC(128, 1, true);   // FP8 comparison cache: heads are the columns
  else if (a.pool.fp8) Q4KV_TC(256, 1, true);
  else if (p.head_dim == 128 && nt == 1) Q4KV_TC(128, 1, false);
  else if (p.head_dim == 128) Q4KV_TC(128, 2, false);
  else if (nt == 1) Q4KV_TC(256, 1, false);
  else Q4KV_TC(256, 2, false);
#undef Q4KV_TC
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace q4kv
