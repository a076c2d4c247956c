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
// shared-memory traffic, N <= 8 columns), so the register-fed mma.sync is
// the better fit for this N.
//
//   keys:   S^T[16 tokens][8 cols] += Kcodes[16 tokens][32 ch] x Qd[32 ch][8 cols]
//           (mma.sync.m16n8k32, u8 codes x s8 query digits, exact int32).
//           The rotated query is scaled to 24-bit fixed point per head
//           (max |q_rot| 2^E <= 8e6) and split into three int8 digits, one
//           MMA each; the integer dot of every 64-channel group is exact and
//           the token's (s, z) are applied in registers:
//           logit = sum_gr s_gr dot_gr 2^-E + z_gr sum(q over gr) 2^-E.
//   values: O^T[16 ch][8 cols] += Vcodes^T[16 ch][16 tokens] x W[16 tokens][8 cols]
//           (mma.sync.m16n8k16, fp16 in, fp32 accumulate): the value scale
//           is folded into the softmax weight, W = p s_V, and sum_t p z_V is
//           added per group at the end.  The weights come out of the key MMA
//           in the accumulator layout; movmatrix.trans turns them into B.
//
// Two column layouts.  "Pairs": a column is one (query head, group) pair,
// used when g * D/64 <= 8 (one n-tile holds every pair); a key step's query
// digits are zero outside the column's group.  "Heads": a column is one
// query head (g <= 8), every key MMA step stays inside one group and keeps
// its own accumulators, and the value MMAs of a group's channels take that
// group's weights W_gr = p s_V,gr; used when the pairs would need two
// n-tiles (g * D/64 > 8), where it halves the MMAs and accumulators.
//
// Warp roles.  A producer warp streams each (block, KV head) run of codes
// with 2-D TMA tensor copies (cp.async.bulk.tensor, no multicast) that
// swizzle 16-byte chunks across banks, and the run's scales/zeros and the
// block's remap mask with 1-D bulk copies, into a 4-deep ring of stages
// guarded by mbarriers.  CW consumer warps take the 16-token tiles of each
// work item round-robin.  An aux warp prepares each item's query (rotation,
// fixed point, digits laid out as every consumer lane's B operands, into one
// of two tables) one item ahead, and merges the consumer warps' partial
// softmax states of the item just finished (log-sum-exp) into the output row
// or a split partial, so consumers never wait for one another between items.
// Every mbarrier wait is bounded: on time-out the kernel raises
// Q4KV_DEVERR_TIMEOUT, poisons the affected rows and returns.
//
// Scheduling: persistent CTAs (one per SM) walk the work items
// (sequence, KV head, split) with a static stride; the producer runs ahead
// across item boundaries.
#include <cuda.h>   // CUtensorMap and its enums; the encoder is reached through the runtime
#include <math.h>
#include <string.h>

#include <mutex>
#include <type_traits>

#include "async_copy.cuh"
#include "encode.cuh"
#include "q4kv_internal.cuh"

namespace q4kv {
namespace {

#ifndef Q4KV_DEC_CODE_KB128
#define Q4KV_DEC_CODE_KB128 16   // code bytes of one tensor per stage at D = 128, in KB
#endif
#ifndef Q4KV_DEC_CW128
#define Q4KV_DEC_CW128 8         // consumer warps at D = 128
#endif
#ifndef Q4KV_DEC_HBQ_SMEM
#define Q4KV_DEC_HBQ_SMEM 1      // heads layout at D = 128 reads its B operands from shared memory
#endif
#ifndef Q4KV_DEC_SPIN
#define Q4KV_DEC_SPIN 0          // try_waits before a consumer's wait starts sleeping
#endif

// Stage ring geometry: per stage the K and V codes of one run of tokens of
// one (block, KV head), their scales/zeros, the block's mask and a header;
// stages are 1024-byte aligned (128B swizzle atoms); about 148 KB in all.
template <int D>
struct Stg {
  static constexpr int kCodeBytes = (D == 128 ? Q4KV_DEC_CODE_KB128 : 16) * 1024;
  static constexpr int kParamBytes = kCodeBytes / 8;
  static constexpr int kOffV = kCodeBytes;
  static constexpr int kOffKP = 2 * kCodeBytes;
  static constexpr int kOffVP = kOffKP + kParamBytes;
  static constexpr int kOffMask = kOffVP + kParamBytes;
  static constexpr int kOffMeta = kOffMask + 32;
  static constexpr int kStageBytes = (kOffMeta + 32 + 1023) / 1024 * 1024;
  static constexpr int kNS = kCodeBytes == 16384 ? 4 : 8;
};
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kQFix = 8000000.0f;         // fixed-point query: max |q_rot| 2^E <= kQFix < 2^23

enum Layout { kPairs = 0, kHeads = 1 };

template <int D>
struct Cfg {
  static constexpr int CW = D == 128 ? Q4KV_DEC_CW128 : 8;   // consumer warps
  static constexpr int kThreads = (CW + 2) * 32; // + producer + aux
  static constexpr int kProducer = CW;
  static constexpr int kAux = CW + 1;
  static constexpr int kAppender = CW + 2;   // fused-append instantiations only
  static constexpr int NG = D / kGroup;
  static constexpr int KK = D / 32;              // key MMA steps (32 channels each)
  static constexpr int HP = 1024 / D;            // heads per merge row (g * D <= 1024)
  // key B operands read from shared memory per tile (instead of registers)
  // where registers would otherwise spill
  template <int LAY>
  static constexpr bool kBqSmem = D == 256 || (LAY == kHeads && Q4KV_DEC_HBQ_SMEM);
  // one query table: the consumer lanes' key B operands (KK steps x 3 digits
  // x 32 lanes x 8 bytes) and 12 per-lane constants; or, for FP8 pools, the
  // fp16 query table [8 heads][D/16][4] of uint4
  static constexpr int kBqBytes = KK * 3 * 32 * 8;
  static constexpr int kQTabBytes =
      (kBqBytes + 32 * 12 * 4) > (8 * (D / 16) * 4 * 16) ? (kBqBytes + 32 * 12 * 4) : (8 * (D / 16) * 4 * 16);
  static constexpr int kOffBars = Stg<D>::kNS * Stg<D>::kStageBytes;
  static constexpr int kOffQTab = kOffBars + 256;                  // full, empty, qready, done, mfree
  static constexpr int kOffQInt = kOffQTab + 2 * kQTabBytes;        // int32 [8][D] fixed-point query
  static constexpr int kOffQAux = kOffQInt + 8 * D * 4;             // int32 gsum[8][4], float escale[8]
  static constexpr int kOffMrgO = kOffQAux + 256;                   // float [CW][D][HP]
  static constexpr int kOffMrgML = kOffMrgO + CW * D * HP * 4;      // float [CW][8][2]
  static constexpr int kOffMrgF = kOffMrgML + CW * 8 * 2 * 4;       // int flags[CW] (padded to 64)
  static constexpr int kOffAuxW = kOffMrgF + 64;                    // float f[CW][8], den[8]
  static constexpr int kSmem = kOffAuxW + CW * 8 * 4 + 8 * 4;
};
static_assert((2 * Stg<128>::kNS + 5) * 8 <= 256 && (2 * Stg<256>::kNS + 5) * 8 <= 256, "barrier area");
static_assert(Cfg<128>::kSmem + 1024 <= 227 * 1024, "shared memory (D = 128)");
static_assert(Cfg<256>::kSmem + 1024 <= 227 * 1024, "shared memory (D = 256)");

struct StageMeta {
  int32_t blk;      // unified block id, -1 if none / invalid
  int32_t tok0;     // first token of the stage within the sequence
  int16_t slot0;    // first slot within the block
  int16_t ntok;     // tokens of the stage that belong to the range
  uint8_t bits;     // code bits of the block's class (2, 4 or 8)
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
// A consumer's wait for a stage: first Q4KV_DEC_SPIN try_waits without
// sleeping in between (a stage is usually moments away), then the bounded
// wait with back-off.
__device__ __forceinline__ bool mbar_wait_hot(uint64_t* bar, uint32_t parity) {
#pragma unroll 1
  for (int i = 0; i < Q4KV_DEC_SPIN; ++i)
    if (mbar_try(bar, parity)) return true;
  return mbar_wait(bar, parity);
}

// A monotonic progress counter in shared memory: the writer publishes with
// a release store, the reader waits (bounded, sleeping between tests) for a
// value with acquire loads.
__device__ __forceinline__ void st_release_cta(uint32_t* p, uint32_t v) {
  asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire_cta(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}
__device__ __forceinline__ bool wait_count(const uint32_t* p, uint32_t v) {
  unsigned ns = 32;
  for (unsigned i = 0; i < 4 * kSpinLimit; ++i) {
    if (ld_acquire_cta(p) >= v) return true;
    __nanosleep(ns);
    ns = ns < 128 ? 2 * ns : 128;
  }
  return false;
}

// Barrier among the warps of the CTA that are not the producer.
__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ uint32_t movtrans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// Four 8x8 b16 matrices from shared memory, transposed: lane 4 g + q gets
// column g of rows 2 q and 2 q + 1 (low and high half) of matrix m in r[m];
// lanes 8 m .. 8 m + 7 give the row addresses of matrix m.
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t h2u(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u2h(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// Value codes enter the fp16 MMA as exact fp16 numbers with no offset: a
// nibble or byte c masked into the low mantissa bits of a zero-exponent fp16
// is the subnormal c * 2^-24.  Value tiles 4 gr + j of even j (even
// channels, group_values) carry c * 2^-24, those of odd j c * 2^-20 (a 4-bit
// high nibble masked in place is 16 c * 2^-24); each output channel therefore
// has one power-of-two scale, undone exactly in the epilogue.
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

// Integer dot of three query digits, as float: 65536 hi + 256 mid + lo.
// |mid * 256 + lo| < 2^25 stays exact in int32; the sum is rounded once.
__device__ __forceinline__ float digits3(int lo, int mid, int hi) {
  return fmaf(static_cast<float>(hi), 65536.0f, static_cast<float>(mid * 256 + lo));
}

// ---------------------------------------------------------------------------
// geometry
// ---------------------------------------------------------------------------
template <int D, int CB>   // CB: code bits of the block class (2, 4 or 8)
struct Geo {
  static constexpr int NG = D / kGroup;
  static constexpr int RB = D * CB / 8;                 // code bytes per token row
  static constexpr int PB = NG * 4;                     // param bytes per token row
  // tokens per stage: as many as the stage's code and parameter areas hold, at most a block
  static constexpr int TS0 = Stg<D>::kCodeBytes / RB < Stg<D>::kParamBytes / PB ? Stg<D>::kCodeBytes / RB
                                                                                  : Stg<D>::kParamBytes / PB;
  static constexpr int TS = TS0 < kBlockTokens ? TS0 : kBlockTokens;
  static constexpr int GB = kGroup * CB / 8;            // code bytes per group
  static constexpr int KB = D * CB / 32;                // key bytes a thread owns per row (pairs layout)
  static constexpr int VB = D * CB / 64;                // value bytes a thread owns per row (pairs layout)
  static constexpr int SW = RB == 32 ? 32 : (RB == 64 ? 64 : (RB == 128 ? 128 : 0));   // TMA swizzle span
  static_assert(TS * PB <= Stg<D>::kParamBytes, "stage params");
};

// Byte offset of (row, byte) of a code tile in shared memory after the TMA
// swizzle: the 16-byte chunk index is XOR-ed with address bits 7.. (row bits;
// 1, 2 or 3 of them for the 32-, 64- and 128-byte spans).
template <int RB, int SW>
__device__ __forceinline__ int swz(int row, int byte) {
  if (SW == 128) return row * RB + ((((byte >> 4) ^ row) & 7) << 4) + (byte & 15);
  if (SW == 64) return row * RB + ((((byte >> 4) ^ (row >> 1)) & 3) << 4) + (byte & 15);
  if (SW == 32) return row * RB + ((((byte >> 4) ^ (row >> 2)) & 1) << 4) + (byte & 15);
  return row * RB + byte;
}

struct TileMaps {       // one map per code array; unused ones stay zero
  CUtensorMap k4, v4, k8, v8, k2, v2;
};

// Token order inside a 16-token tile: accumulator row r holds token pi(r),
// pi swapping 2 <-> 3 and 6 <-> 7 in each half.  With it the four value rows a
// thread reads at one time fall on both 64-byte halves of the 128-byte bank
// window, halving shared-memory bank conflicts; any permutation is correct
// because both contractions sum over tokens.
__device__ __forceinline__ int tok_perm(int r) { return r ^ ((r >> 1) & 1); }

__device__ __forceinline__ void store_out(void* p, int dtype, int64_t i, float x) {
  if (dtype == Q4KV_F32) static_cast<float*>(p)[i] = x;
  else if (dtype == Q4KV_F16) static_cast<__half*>(p)[i] = __float2half_rn(x);
  else static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
}

// Key A operand (u8), 32-channel step, from the thread's two rows' words.
// A 4-bit word holds channels 8w .. 8w+7 at nibbles 0..7: register 0
// (k = 4t .. 4t+3) takes the low nibbles (channels +0, +2, +4, +6), register
// 2 (k = 16 + 4t ..) the high nibbles (+1, +3, +5, +7).  An 8-bit pair of
// words holds the same 8 channels one per byte; the even and odd bytes go to
// the same k slots, so one query table serves 4- and 8-bit blocks alike.
__device__ __forceinline__ void key_a4(uint32_t x0, uint32_t x1, uint32_t (&a)[4]) {
  a[0] = x0 & 0x0F0F0F0Fu;
  a[1] = x1 & 0x0F0F0F0Fu;
  a[2] = (x0 >> 4) & 0x0F0F0F0Fu;
  a[3] = (x1 >> 4) & 0x0F0F0F0Fu;
}
__device__ __forceinline__ void key_a8(uint32_t x0l, uint32_t x0h, uint32_t x1l, uint32_t x1h, uint32_t (&a)[4]) {
  a[0] = __byte_perm(x0l, x0h, 0x6420);
  a[1] = __byte_perm(x1l, x1h, 0x6420);
  a[2] = __byte_perm(x0l, x0h, 0x7531);
  a[3] = __byte_perm(x1l, x1h, 0x7531);
}

// 2-bit: 16 bits hold channels 0..7 at bits 2e; nibble i holds the pair
// (2i, 2i + 1), spread to byte i, then the even channels are the low two
// bits of each byte and the odd channels the next two.
__device__ __forceinline__ uint32_t spread_nibbles(uint32_t x16) {
  return __byte_perm(x16 & 0x0F0Fu, (x16 >> 4) & 0x0F0Fu, 0x5140);   // [n0, n1, n2, n3]
}
__device__ __forceinline__ void key_a2(uint32_t x0, uint32_t x1, uint32_t (&a)[4]) {
  const uint32_t y0 = spread_nibbles(x0 & 0xFFFFu), y1 = spread_nibbles(x1 & 0xFFFFu);
  a[0] = y0 & 0x03030303u;
  a[1] = y1 & 0x03030303u;
  a[2] = (y0 >> 2) & 0x03030303u;
  a[3] = (y1 >> 2) & 0x03030303u;
}

// 8- and 2-bit value operands in the transposed mapping (value tile 4 gr + j:
// channel 64 gr + 4 g + j in rows g, that + 32 in rows g + 8; even j scaled
// 2^-24, odd j 2^-20), from plain 32-bit loads.  8-bit: x and y hold
// channels 4g .. 4g + 3 of a half group for two tokens; the operand pairs
// their bytes j.
__device__ __forceinline__ uint32_t vt_a8(uint32_t x, uint32_t y, int j) {
  const uint32_t p = __byte_perm(x, y, j | ((j + 4) << 8));
  return j % 2 == 0 ? byte_lo(p) : byte_hi(p);
}
// 2-bit: p holds in bytes 0 and 2 the code byte of channels 4g .. 4g + 3 for
// two tokens (channel 4g + j at bits 2j); even j go to bits 0-1, odd j to
// bits 4-5 (16 c * 2^-24).
__device__ __forceinline__ uint32_t vt_a2(uint32_t p, int j) {
  if (j == 0) return p & 0x00030003u;
  if (j == 1) return (p << 2) & 0x00300030u;
  if (j == 2) return (p >> 4) & 0x00030003u;
  return (p >> 2) & 0x00300030u;
}
// One group's four value MMAs of a tile (B operand bw0, bw1: the weights of
// tokens pi(2t), pi(2t+1) and pi(8+2t), pi(9+2t)).  Value tile 4 gr + j holds
// channels 64 gr + 4 g + j (rows g) and 64 gr + 32 + 4 g + j (rows g + 8),
// scaled 2^-24 for even j and 2^-20 for odd j, for every code width, so
// blocks of all widths add into the same accumulators.
//
// 4-bit: one ldmatrix.x4.trans (b16 elements; matrices: tokens 0-7 and 8-15
// of the tile x the two 16-byte halves of the group, row addresses off.lv)
// gives lane (g, t) tokens (2t, 2t+1) and (2t+8, 2t+9) of channels
// 64 gr + 4 g + [0, 4) and of the same channels + 32; nibble masks and one
// 8-bit shift make the operands.  8- and 2-bit: plain 32-bit loads,
// off.vt[x][h] ^ (gr * GB) being the word of token pi(2t), pi(2t+1),
// pi(2t+8) or pi(2t+9) (x) that holds channels 64 gr + 32 h + 4 g .. (8-bit)
// or their byte (2-bit: byte g % 4 of the word, picked by off.sel2).  A group
// is a power-of-two byte span of the row and the swizzle XORs only bits inside
// the row, so group gr's offset is group 0's with gr * GB XORed in.
template <int D, int CB, class O>
__device__ __forceinline__ void group_values(float (&acc)[D / 16][4], const uint8_t* vc, const O& off, int gr,
                                             uint32_t bw0, uint32_t bw1) {
  if constexpr (CB == 4) {
    uint32_t r[4];
    ldsm_x4_trans(static_cast<uint32_t>(__cvta_generic_to_shared(vc)) + off.lv[gr], r);
    const uint32_t s[4] = {r[0] >> 8, r[1] >> 8, r[2] >> 8, r[3] >> 8};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t* x = j < 2 ? r : s;
      uint32_t a[4];
      if (j % 2 == 0) {
        a[0] = lo_nib(x[0]); a[1] = lo_nib(x[2]); a[2] = lo_nib(x[1]); a[3] = lo_nib(x[3]);
      } else {
        a[0] = hi_nib(x[0]); a[1] = hi_nib(x[2]); a[2] = hi_nib(x[1]); a[3] = hi_nib(x[3]);
      }
      mma16816(acc[4 * gr + j], a, bw0, bw1);
    }
  } else {
    uint32_t w[4][2];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int h = 0; h < 2; ++h) w[x][h] = lds<uint32_t>(vc + (off.vt[x][h] ^ (gr * Geo<D, CB>::GB)));
    uint32_t p[4];
    if (CB == 2) {
      p[0] = __byte_perm(w[0][0], w[1][0], off.sel2);
      p[1] = __byte_perm(w[0][1], w[1][1], off.sel2);
      p[2] = __byte_perm(w[2][0], w[3][0], off.sel2);
      p[3] = __byte_perm(w[2][1], w[3][1], off.sel2);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t a[4];
      if (CB == 8) {
        a[0] = vt_a8(w[0][0], w[1][0], j);
        a[1] = vt_a8(w[0][1], w[1][1], j);
        a[2] = vt_a8(w[2][0], w[3][0], j);
        a[3] = vt_a8(w[2][1], w[3][1], j);
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) a[k] = vt_a2(p[k], j);
      }
      mma16816(acc[4 * gr + j], a, bw0, bw1);
    }
  }
}

// Mask bit and validity of the thread's two key rows in tile `tile` of a stage.
struct RowFlags {
  bool valid[2], masked[2];
};
// Rows row[0..1] (relative to the offsets' base row) of the tile `dr` rows
// past that base: the stage's slot of the base row is sb, and rows below nv
// (relative to the base) hold tokens of the range.
template <int D>
__device__ __forceinline__ RowFlags row_flags(const uint8_t* stage, int dr, int sb, int nv, const int (&row)[2]) {
  const uint32_t* mask = reinterpret_cast<const uint32_t*>(stage + Stg<D>::kOffMask);
  const int s16 = sb + dr;   // first slot of the tile, 16-aligned
  const uint32_t mbits = mask[s16 >> 5] >> (s16 & 16);
  RowFlags f;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    f.valid[r] = dr + row[r] < nv;
    f.masked[r] = f.valid[r] && ((mbits >> row[r]) & 1u);
  }
  return f;
}

// One tile's place: stage, row delta from the offsets' base row, the stage
// slot of that base row, valid rows counted from it.
struct TileAt {
  const uint8_t* stg;
  int dr, sb, nv;
};

// The consumer lane's key B operands (KK steps x 3 digits x 2 registers),
// held in registers or read from the item's query table in shared memory
// (lane-major: one 8-byte load per step and digit, conflict-free).
template <int KK>
struct BqRegs {
  uint32_t r[KK][3][2];
  __device__ __forceinline__ uint32_t b0(int kk, int d) const { return r[kk][d][0]; }
  __device__ __forceinline__ uint32_t b1(int kk, int d) const { return r[kk][d][1]; }
  __device__ __forceinline__ void load(const uint2* tab, int lane) {
#pragma unroll
    for (int kk = 0; kk < KK; ++kk)
#pragma unroll
      for (int d = 0; d < 3; ++d) {
        const uint2 w = tab[(kk * 3 + d) * 32 + lane];
        r[kk][d][0] = w.x;
        r[kk][d][1] = w.y;
      }
  }
};
template <int KK>
struct BqSmem {
  const uint2* p;
  uint2 cur;
  __device__ __forceinline__ void load(const uint2* tab, int lane) { p = tab + lane; }
  __device__ __forceinline__ uint2 get(int kk, int d) const { return p[(kk * 3 + d) * 32]; }
};
template <int KK>
__device__ __forceinline__ void mma_key(int (&acc)[4], const uint32_t (&a)[4], const BqRegs<KK>& bq, int kk, int d) {
  mma_u8s8(acc, a, bq.b0(kk, d), bq.b1(kk, d));
}
template <int KK>
__device__ __forceinline__ void mma_key(int (&acc)[4], const uint32_t (&a)[4], const BqSmem<KK>& bq, int kk, int d) {
  const uint2 w = bq.get(kk, d);
  mma_u8s8(acc, a, w.x, w.y);
}

// ---------------------------------------------------------------------------
// "Pairs" layout: column n = (query head n / NG, group n % NG)
// ---------------------------------------------------------------------------
template <int D>
struct PairState {
  float o[D / 16][4];   // value accumulators (channels x (head, group) columns)
  float m;              // running max of the thread's head, log2 units
  float l;              // this thread's share of its running sum
  float z[2];           // sum p * zero for the thread's two columns
};

struct PairConst {
  float qs[2];   // sc2 2^-E sum(q over the column's group), the thread's two columns
  float ks;      // sc2 2^-E of the thread's head
};

template <int D>
__device__ __forceinline__ void reset(PairState<D>& st) {
#pragma unroll
  for (int mv = 0; mv < D / 16; ++mv)
#pragma unroll
    for (int e = 0; e < 4; ++e) st.o[mv][e] = 0.0f;
  st.m = -INFINITY;
  st.l = 0.0f;
  st.z[0] = st.z[1] = 0.0f;
}

// Per-thread byte offsets of tile 0 of a stage.  Tiles start at multiples of
// 16 rows, so the token permutation and the TMA swizzle depend only on the
// row's low four bits, and tile i sits i * 16 rows further on.
// Group-0 word offsets for group_values_vt (8- and 2-bit codes; 4-bit leaves them unset).
template <class G>
__device__ __forceinline__ void init_vt(int (&vt)[4][2], uint32_t& sel2, int base, const int (&vr)[4], int g) {
  constexpr int CB = G::GB * 8 / kGroup;
  static_assert((G::GB & (G::GB - 1)) == 0 && G::RB % G::GB == 0, "groups are power-of-two spans of a row");
  sel2 = static_cast<uint32_t>((g & 3) | (((g & 3) + 4) << 8));
  if constexpr (CB != 4) {
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        vt[x][h] = swz<G::RB, G::SW>(base + vr[x], CB == 8 ? 32 * h + 4 * g : 8 * h + 4 * (g >> 2));
  }
}

template <int D, int CB>
struct PairOffsets {
  using G = Geo<D, CB>;
  static constexpr int NC = D / 128;                        // 128-channel chunks
  static constexpr int KC = G::KB / NC;                     // key bytes per chunk: 8, 16 or 32
  static constexpr int NQ = KC >= 16 ? KC / 16 : 1;         // key loads per chunk (16 bytes, or one of 8)
  int k[2][NC * NQ];   // key rows pi(g), pi(g + 8)
  int v[4];            // value rows pi(2t), pi(2t+1), pi(2t+8), pi(2t+9) (thread g's bytes)
  int lv[G::NG];       // ldmatrix row address of the lane, per group (4-bit values)
  int vt[4][2];        // 8- and 2-bit value words of group 0 in the transposed mapping (group_values_vt)
  uint32_t sel2;       // 2-bit: byte g % 4 of two words into bytes 0 and 2
  int p[2];            // parameter rows pi(g), pi(g + 8) (the thread's two groups)
  int row[2];          // pi(g), pi(g + 8), relative to the base row

  // base: a multiple of 16 (the swizzle and token order repeat every 16 rows)
  __device__ __forceinline__ void init(int lane, int base) {
    const int g = lane >> 2, t = lane & 3;
    row[0] = tok_perm(g);
    row[1] = tok_perm(g + 8);
#pragma unroll
    for (int x = 0; x < 2; ++x) {
#pragma unroll
      for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int q = 0; q < NQ; ++q)
          k[x][c * NQ + q] = swz<G::RB, G::SW>(base + row[x], c * (G::RB / NC) + t * KC + q * 16);
      p[x] = (base + row[x]) * G::PB + ((G::NG == 2) ? 0 : 2 * (t & 1)) * 4;
    }
    const int vr[4] = {tok_perm(2 * t), tok_perm(2 * t + 1), tok_perm(2 * t + 8), tok_perm(2 * t + 9)};
#pragma unroll
    for (int x = 0; x < 4; ++x) v[x] = swz<G::RB, G::SW>(base + vr[x], g * G::VB);
    // matrix m = lane / 8: tokens 8 (m & 1) + [0, 8), channel half m >> 1 of
    // the group (16 bytes); row i of a matrix is token pi(i) of its half tile
    const int m = lane >> 3, i = lane & 7;
#pragma unroll
    for (int gr = 0; gr < G::NG; ++gr)
      lv[gr] = swz<G::RB, G::SW>(base + tok_perm(8 * (m & 1) + i), gr * G::GB + 16 * (m >> 1));
    init_vt<G>(vt, sel2, base, vr, g);
  }
};

// The lazy online softmax: the running max moves only when a tile's max
// exceeds it by more than kLazy (log2 units), so the accumulators are
// rescaled rarely; weights stay <= 2^kLazy.
constexpr float kLazy = 2.0f;

// NTL 16-token tiles in the pairs layout (tile i: tile[i] of stage stg[i],
// whose first nvalid[i] rows belong to the range), with one online-softmax
// update over all of them: two tiles give the scheduler two independent
// key-MMA chains and halve the softmax bookkeeping.  Thread t owns channels
// 128c + 32t + [0, 32) of each key row; step kk uses chunk c = kk / 4, word
// kk % 4.
template <int D, int CB, int NTL, class BQ>
__device__ __forceinline__ void pair_tiles(PairState<D>& st, const TileAt (&ta)[NTL],
                                           const PairOffsets<D, CB>& o, const BQ& bq, const PairConst& qc) {
  using G = Geo<D, CB>;
  using O = PairOffsets<D, CB>;
  // ---- keys ----
  float sk[NTL][4];
#pragma unroll
  for (int i = 0; i < NTL; ++i) {
    uint32_t rg[G::KB / 4], rg8[G::KB / 4];
    const uint8_t* base = ta[i].stg + ta[i].dr * G::RB;
#pragma unroll
    for (int n = 0; n < O::NC * O::NQ; ++n) {
      if (O::KC >= 16) {
        const uint4 u = lds<uint4>(base + o.k[0][n]), u8 = lds<uint4>(base + o.k[1][n]);
        rg[4 * n] = u.x; rg[4 * n + 1] = u.y; rg[4 * n + 2] = u.z; rg[4 * n + 3] = u.w;
        rg8[4 * n] = u8.x; rg8[4 * n + 1] = u8.y; rg8[4 * n + 2] = u8.z; rg8[4 * n + 3] = u8.w;
      } else {
        const uint2 u = lds<uint2>(base + o.k[0][n]), u8 = lds<uint2>(base + o.k[1][n]);
        rg[2 * n] = u.x; rg[2 * n + 1] = u.y;
        rg8[2 * n] = u8.x; rg8[2 * n + 1] = u8.y;
      }
    }
    int acc[3][4];
#pragma unroll
    for (int d = 0; d < 3; ++d)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[d][e] = 0;
#pragma unroll
    for (int kk = 0; kk < D / 32; ++kk) {
      uint32_t a[4];
      if (CB == 4) key_a4(rg[kk], rg8[kk], a);
      else if (CB == 8) key_a8(rg[2 * kk], rg[2 * kk + 1], rg8[2 * kk], rg8[2 * kk + 1], a);
      else key_a2(rg[kk / 2] >> (16 * (kk % 2)), rg8[kk / 2] >> (16 * (kk % 2)), a);
#pragma unroll
      for (int d = 0; d < 3; ++d) mma_key(acc[d], a, bq, kk, d);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) sk[i][e] = digits3(acc[0][e], acc[1][e], acc[2][e]);
  }
  // ---- per-token parameters and logits (log2 units) ----
  // D = 128: the thread's columns are (h, 0), (h, 1); D = 256: (h, 2 (t%2)), (h, 2 (t%2) + 1).
  float logit[NTL][2], ws[NTL][2][2], wz[NTL][2][2];
  bool live[NTL][2];
#pragma unroll
  for (int i = 0; i < NTL; ++i) {
    const RowFlags f = row_flags<D>(ta[i].stg, ta[i].dr, ta[i].sb, ta[i].nv, o.row);
    const int pr = ta[i].dr * G::PB;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const bool lv = f.valid[r] && !f.masked[r];
      live[i][r] = lv;
      const uint2 kpw = lds<uint2>(ta[i].stg + Stg<D>::kOffKP + o.p[r] + pr);
      const uint2 vpw = lds<uint2>(ta[i].stg + Stg<D>::kOffVP + o.p[r] + pr);
      const float2 k0 = __half22float2(u2h(kpw.x)), k1 = __half22float2(u2h(kpw.y));
      const float2 v0 = __half22float2(u2h(vpw.x)), v1 = __half22float2(u2h(vpw.y));
      // rows outside the range or remapped may hold any bytes (even NaN
      // parameters): select, never multiply, them away
      ws[i][r][0] = lv ? v0.x : 0.0f;
      wz[i][r][0] = lv ? v0.y : 0.0f;
      ws[i][r][1] = lv ? v1.x : 0.0f;
      wz[i][r][1] = lv ? v1.y : 0.0f;
      float part = __fmaf_rn(k0.x, sk[i][2 * r], k1.x * sk[i][2 * r + 1]) * qc.ks +
                   __fmaf_rn(k0.y, qc.qs[0], k1.y * qc.qs[1]);
      if (G::NG == 4) part += __shfl_xor_sync(0xffffffffu, part, 1);
      logit[i][r] = !f.valid[r] ? -INFINITY : (f.masked[r] ? Q4KV_SENTINEL_LOGIT * kLog2e : part);
    }
  }
  // ---- online softmax ----
  // The column max (a shuffle reduction) is needed only when some logit
  // exceeds the running max by more than kLazy; a warp vote finds out.
  bool grow = false;
#pragma unroll
  for (int i = 0; i < NTL; ++i) grow |= fmaxf(logit[i][0], logit[i][1]) > st.m + kLazy;
  if (__any_sync(0xffffffffu, grow)) {
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < NTL; ++i) mx = fmaxf(mx, fmaxf(logit[i][0], logit[i][1]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (mx > st.m + kLazy) {          // also taken on the first live tile (m = -inf)
      const float alpha = ex2(st.m - mx);
      st.m = mx;
      st.l *= alpha;
      st.z[0] *= alpha;
      st.z[1] *= alpha;
#pragma unroll
      for (int mv = 0; mv < D / 16; ++mv)
#pragma unroll
        for (int e = 0; e < 4; ++e) st.o[mv][e] *= alpha;
    }
  }
  uint32_t wb[NTL][2];
#pragma unroll
  for (int i = 0; i < NTL; ++i)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float p = logit[i][r] == -INFINITY ? 0.0f : ex2(logit[i][r] - st.m);
      st.l += p;
      const float q = live[i][r] ? p : 0.0f;
      st.z[0] = __fmaf_rn(q, wz[i][r][0], st.z[0]);
      st.z[1] = __fmaf_rn(q, wz[i][r][1], st.z[1]);
      wb[i][r] = h2u(__floats2half2_rn(q * ws[i][r][0], q * ws[i][r][1]));
    }
  // ---- values: every group with the tile's weights ----
#pragma unroll
  for (int i = 0; i < NTL; ++i) {
    const uint32_t bw0 = movtrans(wb[i][0]);   // tokens pi(2t), pi(2t+1)
    const uint32_t bw1 = movtrans(wb[i][1]);   // tokens pi(8+2t), pi(9+2t)
    const uint8_t* vc = ta[i].stg + Stg<D>::kOffV + ta[i].dr * G::RB;
#pragma unroll
    for (int gr = 0; gr < G::NG; ++gr) group_values<D, CB>(st.o, vc, o, gr, bw0, bw1);
  }
}

// ---------------------------------------------------------------------------
// "Heads" layout: column n = query head n
// ---------------------------------------------------------------------------
template <int D>
struct HeadState {
  float o[D / 16][4];        // channels x heads (2t, 2t+1)
  float m[2];                // running max of heads 2t, 2t+1, log2 units
  float l[2];
  float z[2][D / kGroup];    // sum p * zero_V per (head, group)
};

template <int D>
struct HeadConst {
  float ks[2];                 // sc2 2^-E of heads 2t, 2t+1
  float qs[2][D / kGroup];     // sc2 2^-E sum(q over group)
};

template <int D>
__device__ __forceinline__ void reset(HeadState<D>& st) {
#pragma unroll
  for (int mv = 0; mv < D / 16; ++mv)
#pragma unroll
    for (int e = 0; e < 4; ++e) st.o[mv][e] = 0.0f;
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    st.m[c] = -INFINITY;
    st.l[c] = 0.0f;
#pragma unroll
    for (int gr = 0; gr < D / kGroup; ++gr) st.z[c][gr] = 0.0f;
  }
}

// Per-thread offsets in the heads layout.  Keys: per group, thread t's 16
// channels 64 gr + 16 t + [0, 16) of rows pi(g), pi(g + 8) (4, 8 or 16
// bytes); step 2 gr + hf takes channels 64 gr + 16 t + 8 hf + [0, 8).
// Values: per group, thread g's 8 channels 64 gr + 8 g + [0, 8) of the four
// rows pi(2t), pi(2t+1), pi(2t+8), pi(2t+9), so every value m-tile (16
// channel rows) lies inside one group.
template <int D, int CB>
struct HeadOffsets {
  using G = Geo<D, CB>;
  static constexpr int NG = G::NG;
  int k[2][NG];
  int lv[NG];   // ldmatrix row address of the lane, per group (4-bit values)
  int vt[4][2];       // 8- and 2-bit value words of group 0 in the transposed mapping (group_values_vt)
  uint32_t sel2;      // 2-bit: byte g % 4 of two words into bytes 0 and 2
  int p[2];
  int row[2];   // relative to the base row

  __device__ __forceinline__ void init(int lane, int base) {
    const int g = lane >> 2, t = lane & 3;
    row[0] = tok_perm(g);
    row[1] = tok_perm(g + 8);
    const int kb = 2 * CB;   // bytes of 16 channels
#pragma unroll
    for (int x = 0; x < 2; ++x) {
#pragma unroll
      for (int gr = 0; gr < NG; ++gr) k[x][gr] = swz<G::RB, G::SW>(base + row[x], gr * G::GB + t * kb);
      p[x] = (base + row[x]) * G::PB;
    }
    const int vr[4] = {tok_perm(2 * t), tok_perm(2 * t + 1), tok_perm(2 * t + 8), tok_perm(2 * t + 9)};
    // matrix m = lane / 8: tokens 8 (m & 1) + [0, 8), channel half m >> 1 of
    // the group (16 bytes); row i of a matrix is token pi(i) of its half tile
    const int m = lane >> 3, i = lane & 7;
#pragma unroll
    for (int gr = 0; gr < NG; ++gr)
      lv[gr] = swz<G::RB, G::SW>(base + tok_perm(8 * (m & 1) + i), gr * G::GB + 16 * (m >> 1));
    init_vt<G>(vt, sel2, base, vr, g);
  }
};

// NTL tiles in the heads layout, one online-softmax update over all of them.
template <int D, int CB, int NTL, class BQ>
__device__ __forceinline__ void head_tiles(HeadState<D>& st, const TileAt (&ta)[NTL],
                                           const HeadOffsets<D, CB>& o, const BQ& bq, const HeadConst<D>& qc) {
  using G = Geo<D, CB>;
  constexpr int NG = G::NG;
  // ---- keys: per group, two 32-channel steps x three digits ----
  float dot[NTL][NG][4];
#pragma unroll
  for (int i = 0; i < NTL; ++i) {
    const uint8_t* base = ta[i].stg + ta[i].dr * G::RB;
#pragma unroll
    for (int gr = 0; gr < NG; ++gr) {
      int acc[3][4];
#pragma unroll
      for (int d = 0; d < 3; ++d)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[d][e] = 0;
      if (CB == 4) {
        const uint2 u = lds<uint2>(base + o.k[0][gr]), u8 = lds<uint2>(base + o.k[1][gr]);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t a[4];
          key_a4(hf ? u.y : u.x, hf ? u8.y : u8.x, a);
#pragma unroll
          for (int d = 0; d < 3; ++d) mma_key(acc[d], a, bq, 2 * gr + hf, d);
        }
      } else if (CB == 2) {
        const uint32_t u = lds<uint32_t>(base + o.k[0][gr]), u8 = lds<uint32_t>(base + o.k[1][gr]);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t a[4];
          key_a2(u >> (16 * hf), u8 >> (16 * hf), a);
#pragma unroll
          for (int d = 0; d < 3; ++d) mma_key(acc[d], a, bq, 2 * gr + hf, d);
        }
      } else {
        const uint4 u = lds<uint4>(base + o.k[0][gr]), u8 = lds<uint4>(base + o.k[1][gr]);
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t a[4];
          key_a8(hf ? u.z : u.x, hf ? u.w : u.y, hf ? u8.z : u8.x, hf ? u8.w : u8.y, a);
#pragma unroll
          for (int d = 0; d < 3; ++d) mma_key(acc[d], a, bq, 2 * gr + hf, d);
        }
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) dot[i][gr][e] = digits3(acc[0][e], acc[1][e], acc[2][e]);
    }
  }
  // ---- logits: accumulator element e = (row e / 2, head column e % 2) ----
  float logit[NTL][2][2], sv[NTL][2][NG], zv[NTL][2][NG];
  bool live[NTL][2];
#pragma unroll
  for (int i = 0; i < NTL; ++i) {
    const RowFlags f = row_flags<D>(ta[i].stg, ta[i].dr, ta[i].sb, ta[i].nv, o.row);
    const int pr = ta[i].dr * G::PB;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const bool lv = f.valid[r] && !f.masked[r];
      live[i][r] = lv;
      float2 kp[NG], vp[NG];
      if (NG == 2) {
        const uint2 kw = lds<uint2>(ta[i].stg + Stg<D>::kOffKP + o.p[r] + pr);
        const uint2 vw = lds<uint2>(ta[i].stg + Stg<D>::kOffVP + o.p[r] + pr);
        kp[0] = __half22float2(u2h(kw.x)); kp[NG - 1] = __half22float2(u2h(kw.y));
        vp[0] = __half22float2(u2h(vw.x)); vp[NG - 1] = __half22float2(u2h(vw.y));
      } else {
        const uint4 kw = lds<uint4>(ta[i].stg + Stg<D>::kOffKP + o.p[r] + pr);
        const uint4 vw = lds<uint4>(ta[i].stg + Stg<D>::kOffVP + o.p[r] + pr);
        const uint32_t kk4[4] = {kw.x, kw.y, kw.z, kw.w}, vv4[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
        for (int gr = 0; gr < NG; ++gr) {
          kp[gr] = __half22float2(u2h(kk4[gr & 3]));
          vp[gr] = __half22float2(u2h(vv4[gr & 3]));
        }
      }
#pragma unroll
      for (int gr = 0; gr < NG; ++gr) {
        sv[i][r][gr] = lv ? vp[gr].x : 0.0f;
        zv[i][r][gr] = lv ? vp[gr].y : 0.0f;
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float sd = 0.0f, zq = 0.0f;
#pragma unroll
        for (int gr = 0; gr < NG; ++gr) {
          sd = __fmaf_rn(kp[gr].x, dot[i][gr][2 * r + c], sd);
          zq = __fmaf_rn(kp[gr].y, qc.qs[c][gr], zq);
        }
        const float part = __fmaf_rn(sd, qc.ks[c], zq);
        logit[i][r][c] = !f.valid[r] ? -INFINITY : (f.masked[r] ? Q4KV_SENTINEL_LOGIT * kLog2e : part);
      }
    }
  }
  // ---- online softmax per head column (max reduction only when a warp vote
  // finds a logit above the running max + kLazy) ----
  bool grow = false;
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int i = 0; i < NTL; ++i) grow |= fmaxf(logit[i][0][c], logit[i][1][c]) > st.m[c] + kLazy;
  if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < NTL; ++i) mx = fmaxf(mx, fmaxf(logit[i][0][c], logit[i][1][c]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      if (mx > st.m[c] + kLazy) {
        const float alpha = ex2(st.m[c] - mx);
        st.m[c] = mx;
        st.l[c] *= alpha;
#pragma unroll
        for (int gr = 0; gr < NG; ++gr) st.z[c][gr] *= alpha;
#pragma unroll
        for (int mv = 0; mv < D / 16; ++mv) {
          st.o[mv][c] *= alpha;
          st.o[mv][2 + c] *= alpha;
        }
      }
    }
  }
  float q[NTL][2][2];
#pragma unroll
  for (int i = 0; i < NTL; ++i)
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const float p = logit[i][r][c] == -INFINITY ? 0.0f : ex2(logit[i][r][c] - st.m[c]);
        st.l[c] += p;
        q[i][r][c] = live[i][r] ? p : 0.0f;
#pragma unroll
        for (int gr = 0; gr < NG; ++gr) st.z[c][gr] = __fmaf_rn(q[i][r][c], zv[i][r][gr], st.z[c][gr]);
      }
  // ---- values, one group at a time with that group's weights ----
#pragma unroll
  for (int i = 0; i < NTL; ++i) {
    const uint8_t* vc = ta[i].stg + Stg<D>::kOffV + ta[i].dr * G::RB;
#pragma unroll
    for (int gr = 0; gr < NG; ++gr) {
      const uint32_t bw0 =
          movtrans(h2u(__floats2half2_rn(q[i][0][0] * sv[i][0][gr], q[i][0][1] * sv[i][0][gr])));
      const uint32_t bw1 =
          movtrans(h2u(__floats2half2_rn(q[i][1][0] * sv[i][1][gr], q[i][1][1] * sv[i][1][gr])));
      group_values<D, CB>(st.o, vc, o, gr, bw0, bw1);
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

// One tile of an FP8 stage (8-bit geometry).  qtab: this thread's entries of
// the query table, entry ks at qtab[ks * 4] = (high b0, high b1, low b0, low
// b1) for channels 128 (ks / 8) + 32 t + 4 (ks % 8) + 0..3 of head g.
template <int D>
__device__ __forceinline__ void fp8_tile(Fp8State<D>& st, const TileAt& ta, const PairOffsets<D, 8>& o,
                                         const uint4* __restrict__ qtab) {
  using G = Geo<D, 8>;
  using O = PairOffsets<D, 8>;
  const uint8_t* stage = ta.stg;
  const int r0 = ta.dr;
  float sk[4];
  {
    uint32_t rg[G::KB / 4], rg8[G::KB / 4];
    const uint8_t* base = stage + r0 * G::RB;
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
    for (int e = 0; e < 4; ++e) sk[e] = acc[e];
  }
  // logits (log2 units; the query carries scale * log2 e): acc e = (row e / 2, column 2t + e % 2)
  const RowFlags f = row_flags<D>(stage, ta.dr, ta.sb, ta.nv, o.row);
  float logit[2][2];   // [row][column]
  bool live[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    live[r] = f.valid[r] && !f.masked[r];
#pragma unroll
    for (int c = 0; c < 2; ++c)
      logit[r][c] = !f.valid[r] ? -INFINITY : (f.masked[r] ? Q4KV_SENTINEL_LOGIT * kLog2e : sk[2 * r + c]);
  }
#pragma unroll
  for (int c = 0; c < 2; ++c) {
    float mx = fmaxf(logit[0][c], logit[1][c]);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (mx > st.m[c] + kLazy) {
      const float alpha = ex2(st.m[c] - mx);
      st.m[c] = mx;
      st.l[c] *= alpha;
#pragma unroll
      for (int mv = 0; mv < D / 16; ++mv) {
        st.o[mv][c] *= alpha;
        st.o[mv][2 + c] *= alpha;
      }
    }
  }
  uint32_t wb[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float p[2];
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      p[c] = logit[r][c] == -INFINITY ? 0.0f : ex2(logit[r][c] - st.m[c]);
      st.l[c] += p[c];
    }
    // a remapped slot's value is 0 (its weight still counts in the sum);
    // rows past the range may hold any bytes: selected away
    wb[r] = live[r] ? h2u(__floats2half2_rn(p[0], p[1])) : 0u;
  }
  const uint32_t bw0 = movtrans(wb[0]), bw1 = movtrans(wb[1]);
  constexpr int VW = G::VB / 4;
  uint32_t v0[VW], v1[VW], v8[VW], v9[VW];
  const uint8_t* vc = stage + Stg<D>::kOffV + r0 * G::RB;
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

// ---------------------------------------------------------------------------
// aux warp: query preparation and the per-item merge
// ---------------------------------------------------------------------------
// Work item -> (sequence, KV head, split), splits varying fastest.  (After
// an append, moving the last splits' items, which hold the blocks it
// writes, to the end of the order was measured slower than this order.)
__device__ __forceinline__ void item_coords(const DecodeArgs& a, int item, int& b, int& kvh, int& split) {
  const int S = a.plan.n_splits, hkv = a.plan.n_kv_heads;
  split = item % S;
  kvh = (item / S) % hkv;
  b = item / (S * hkv);
}

// Raw 16-bit query elements E*lane .. E*lane + E-1 of query head `qh` as floats.
template <int E>
__device__ __forceinline__ void load_query(const DecodeArgs& a, int64_t qh, int lane, float (&x)[E]) {
  const uint8_t* p = static_cast<const uint8_t*>(a.q) + 2 * (qh * (E * 32) + E * lane);
  uint32_t ww[4];
  if (E == 4) {
    const uint2 w = *reinterpret_cast<const uint2*>(p);
    ww[0] = w.x; ww[1] = w.y; ww[2] = ww[3] = 0u;
  } else {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    ww[0] = w.x; ww[1] = w.y; ww[2] = w.z; ww[3] = w.w;
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const uint32_t h16 = (ww[e / 2] >> (16 * (e % 2))) & 0xFFFFu;
    x[e] = a.q_dtype == Q4KV_F16 ? __half2float(__ushort_as_half(static_cast<unsigned short>(h16)))
                                 : __uint_as_float(h16 << 16);
  }
}

// c * H x across the warp (lane holds channels E*lane .. E*lane + E-1): stages
// of stride 1 .. E/2 in the lane, then E .. D/2 across lanes, then times c.
template <int D, int E>
__device__ __forceinline__ void rotate(float (&x)[E], int lane) {
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

// Signed 8-bit digits of q = 65536 d2 + 256 d1 + d0, each in [-128, 127].
__device__ __forceinline__ void split3(int q, uint32_t (&d)[3]) {
  const int q1 = (q + 128) >> 8;        // q - d0 over 256, d0 = q mod 256 as a signed byte
  d[0] = static_cast<uint32_t>(q) & 255u;
  d[1] = static_cast<uint32_t>(q1) & 255u;
  d[2] = static_cast<uint32_t>((q1 + 128) >> 8) & 255u;
}

// Query preparation of one item, in three pieces so that one warp can run
// them all (items after the first) or every warp a share (the first item).
//
// prep_head: query head h, by one warp: rotate (keys stored rotated), scale
// to fixed point (max |q_rot| 2^E <= kQFix), keep the exact group sums.
template <int D>
__device__ __forceinline__ void prep_head(const DecodeArgs& a, int b, int kvh, int h, int* qint, int* gsum,
                                          float* escale, int lane) {
  constexpr int E = D / 32;
  const int hq = a.plan.n_q_heads, G = hq / a.pool.n_kv_heads;
  float x[E];
  load_query<E>(a, static_cast<int64_t>(b) * hq + kvh * G + h, lane, x);
  if (a.pool.k_rotated) rotate<D, E>(x, lane);
  float mx = 0.0f;
#pragma unroll
  for (int e = 0; e < E; ++e) mx = fmaxf(mx, fabsf(x[e]));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  int ex = 0;
  if (mx > 0.0f) ex = static_cast<int>(floorf(log2f(kQFix / mx)));
  ex = max(-100, min(100, ex));
  int part = 0;
  int qv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] = static_cast<int>(rintf(ldexpf(x[e], ex)));   // |qv| <= 8e6: exact in binary32
    part += qv[e];
  }
  *reinterpret_cast<int4*>(qint + h * D + E * lane) = make_int4(qv[0], qv[1], qv[2], qv[3]);
  if (E == 8)
    *reinterpret_cast<int4*>(qint + h * D + E * lane + 4) = make_int4(qv[E - 4], qv[E - 3], qv[E - 2], qv[E - 1]);
  // exact group sums (|sum| <= 64 * 8e6 < 2^31): the 64 / E lanes of a group are consecutive
#pragma unroll
  for (int off = 1; off < kGroup / E; off <<= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
  if (lane % (kGroup / E) == 0) gsum[h * 4 + lane / (kGroup / E)] = part;
  if (lane == 0) escale[h] = ldexpf(1.0f, -ex);
}

// prep_entry: the B operands of consumer lane L = (g, t) for key step kk,
// three digits, from the fixed-point query (its B column is n = g).
template <int D, int LAY>
__device__ __forceinline__ void prep_entry(int kk, int L, int G, const int* qint, uint8_t* tab) {
  constexpr int NG = D / kGroup;
  const int g = L >> 2, t = L & 3;
  int h, base;
  bool use;
  if (LAY == kPairs) {
    h = g / NG;
    base = 128 * (kk / 4) + 32 * t + 8 * (kk % 4);
    use = h < G && 2 * (kk / 4) + (t >> 1) == g % NG;
  } else {
    h = g;
    base = 64 * (kk / 2) + 16 * t + 8 * (kk % 2);
    use = h < G;
  }
  int4 lo = make_int4(0, 0, 0, 0), hi = make_int4(0, 0, 0, 0);
  if (use) {
    lo = *reinterpret_cast<const int4*>(qint + h * D + base);
    hi = *reinterpret_cast<const int4*>(qint + h * D + base + 4);
  }
  // b0: channels base + {0, 2, 4, 6}; b1: base + {1, 3, 5, 7}
  const int ev[4] = {lo.x, lo.z, hi.x, hi.z}, od[4] = {lo.y, lo.w, hi.y, hi.w};
  uint32_t b0[3] = {0u, 0u, 0u}, b1[3] = {0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t de[3], dd[3];
    split3(ev[i], de);
    split3(od[i], dd);
#pragma unroll
    for (int d = 0; d < 3; ++d) {
      b0[d] |= de[d] << (8 * i);
      b1[d] |= dd[d] << (8 * i);
    }
  }
  uint2* bqt = reinterpret_cast<uint2*>(tab);
#pragma unroll
  for (int d = 0; d < 3; ++d) bqt[(kk * 3 + d) * 32 + L] = make_uint2(b0[d], b1[d]);
}

// prep_consts: consumer lane L's constants: pairs -- sc2 2^-E sum(q) of its
// two columns and sc2 2^-E of its head; heads -- sc2 2^-E of heads 2t, 2t+1
// and sc2 2^-E sum(q) per (head, group).
template <int D, int LAY>
__device__ __forceinline__ void prep_consts(const DecodeArgs& a, int L, int G, const int* gsum,
                                            const float* escale, uint8_t* tab) {
  constexpr int NG = D / kGroup;
  const int t = L & 3;
  float* cst = reinterpret_cast<float*>(tab + Cfg<D>::kBqBytes) + L * 12;
  const float sc2 = a.scale * kLog2e;
  if (LAY == kPairs) {
    const int c2 = 2 * t, h2 = c2 / NG;
    const float ks = h2 < G ? sc2 * escale[h2] : 0.0f;
    cst[0] = h2 < G ? ks * static_cast<float>(gsum[h2 * 4 + c2 % NG]) : 0.0f;
    cst[1] = h2 < G ? ks * static_cast<float>(gsum[h2 * 4 + (c2 + 1) % NG]) : 0.0f;
    cst[2] = ks;
  } else {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int h = 2 * t + c;
      const float ks = h < G ? sc2 * escale[h] : 0.0f;
      cst[c] = ks;
#pragma unroll
      for (int gr = 0; gr < NG; ++gr)
        cst[2 + c * NG + gr] = h < G ? ks * static_cast<float>(gsum[h * 4 + gr]) : 0.0f;
    }
  }
}

// One item's whole table, by one warp.
template <int D, int LAY>
__device__ void prep_q4(const DecodeArgs& a, int item, uint8_t* tab, int* qint, int* gsum, float* escale,
                        int lane) {
  const int hkv = a.pool.n_kv_heads, G = a.plan.n_q_heads / hkv;
  int b, kvh, split;
  item_coords(a, item, b, kvh, split);
  for (int h = 0; h < G; ++h) prep_head<D>(a, b, kvh, h, qint, gsum, escale, lane);
  __syncwarp();
#pragma unroll 1
  for (int kk = 0; kk < Cfg<D>::KK; ++kk) prep_entry<D, LAY>(kk, lane, G, qint, tab);
  prep_consts<D, LAY>(a, lane, G, gsum, escale, tab);
}

// FP8 query table [head][ks][t]: q * scale * log2 e as fp16 high + low parts
// in the B layout of the key MMA (entry (head, ks, t) covers channels
// 128 (ks / 8) + 32 t + 4 (ks % 8) + 0..3); heads past G stay zero.
template <int D>
__device__ __forceinline__ void prep_fp8_head(const DecodeArgs& a, int b, int kvh, int h, uint8_t* tab, int lane) {
  constexpr int E = D / 32;
  const int hkv = a.pool.n_kv_heads, hq = a.plan.n_q_heads, G = hq / hkv;
  uint4* qtab = reinterpret_cast<uint4*>(tab);
  const float sc2 = a.scale * kLog2e;
  {
    float x[E];
    load_query<E>(a, static_cast<int64_t>(b) * hq + kvh * G + h, lane, x);
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
      qtab[(h * (D / 16) + (lane & 7)) * 4 + (lane >> 3)] = make_uint4(hw[0], hw[1], lw[0], lw[1]);
    } else {                  // channels 8 lane + 0..7: two entries
      const int ks0 = 8 * (lane >> 4) + 2 * (lane & 3), tt = (lane & 15) >> 2;
      qtab[(h * (D / 16) + ks0) * 4 + tt] = make_uint4(hw[0], hw[1], lw[0], lw[1]);
      qtab[(h * (D / 16) + ks0 + 1) * 4 + tt] = make_uint4(hw[E / 2 - 2], hw[E / 2 - 1], lw[E / 2 - 2], lw[E / 2 - 1]);
    }
  }
}

template <int D>
__device__ void prep_fp8(const DecodeArgs& a, int item, uint8_t* tab, int lane) {
  const int hkv = a.pool.n_kv_heads, G = a.plan.n_q_heads / hkv;
  int b, kvh, split;
  item_coords(a, item, b, kvh, split);
  for (int h = 0; h < G; ++h) prep_fp8_head<D>(a, b, kvh, h, tab, lane);
}

// Merge the consumer warps' states of one item (log-sum-exp over warps) and
// write its output row (one split) or split partial.
template <int D>
__device__ void merge_item(const DecodeArgs& a, int item, const float* mrg_o, const float* mrg_ml,
                           const int* mrg_flag, float* fw, float* den, bool extra_bad, int lane) {
  using C = Cfg<D>;
  const int hkv = a.pool.n_kv_heads, hq = a.plan.n_q_heads, G = hq / hkv, S = a.plan.n_splits;
  int b, kvh, split;
  item_coords(a, item, b, kvh, split);
  int flag = 0;
#pragma unroll
  for (int w = 0; w < C::CW; ++w) flag |= mrg_flag[w];
  const bool bad = flag != 0 || extra_bad;
  float Mh = -INFINITY;
  if (lane < G) {
#pragma unroll
    for (int w = 0; w < C::CW; ++w) Mh = fmaxf(Mh, mrg_ml[(w * 8 + lane) * 2]);
    float dn = 0.0f;
#pragma unroll
    for (int w = 0; w < C::CW; ++w) {
      const float f = Mh == -INFINITY ? 0.0f : ex2(mrg_ml[(w * 8 + lane) * 2] - Mh);
      fw[w * 8 + lane] = f;
      dn = __fmaf_rn(mrg_ml[(w * 8 + lane) * 2 + 1], f, dn);
    }
    den[lane] = dn;
    if (S > 1) {
      const int64_t qrow = static_cast<int64_t>(b) * hq + kvh * G + lane;
      a.ws_ml[(qrow * S + split) * 2] = Mh == -INFINITY ? -INFINITY : Mh / kLog2e;
      a.ws_ml[(qrow * S + split) * 2 + 1] = bad ? -1.0f : dn;
    }
  }
  __syncwarp();
  for (int ch = lane; ch < D; ch += 32) {
    float num[C::HP];
#pragma unroll
    for (int h = 0; h < C::HP; ++h) num[h] = 0.0f;
#pragma unroll
    for (int w = 0; w < C::CW; ++w) {
      const float4* src = reinterpret_cast<const float4*>(mrg_o + (w * D + ch) * C::HP);
#pragma unroll
      for (int q4 = 0; q4 < C::HP / 4; ++q4) {
        const float4 v = src[q4];
        num[4 * q4] = __fmaf_rn(v.x, fw[w * 8 + 4 * q4], num[4 * q4]);
        num[4 * q4 + 1] = __fmaf_rn(v.y, fw[w * 8 + 4 * q4 + 1], num[4 * q4 + 1]);
        num[4 * q4 + 2] = __fmaf_rn(v.z, fw[w * 8 + 4 * q4 + 2], num[4 * q4 + 2]);
        num[4 * q4 + 3] = __fmaf_rn(v.w, fw[w * 8 + 4 * q4 + 3], num[4 * q4 + 3]);
      }
    }
#pragma unroll
    for (int h = 0; h < C::HP; ++h) {
      if (h >= G) break;
      const int64_t qrow = static_cast<int64_t>(b) * hq + kvh * G + h;
      if (S == 1) {
        const float dn = den[h];
        store_out(a.out, a.out_dtype, qrow * D + ch, (!bad && dn > 0.0f) ? num[h] / dn : 0.0f);
      } else {
        a.ws_o[(qrow * S + split) * D + ch] = num[h];
      }
    }
  }
  __syncwarp();   // fw / den are rewritten by the next item
}

// ---------------------------------------------------------------------------
// Fused append: the appender warp encodes the new rows of an item's (sequence, KV
// head) whose positions fall in the item's split, with the append kernel's
// encoding steps (encode.cuh): up to VPW tokens of one block per pass (a
// lane holds 16 channels of one token), so the block and its code width are
// the same for the whole warp and every shuffle runs converged.  Each such
// item clears the new slots' mask bits (the bits are shared by the KV heads;
// clearing is idempotent).  The proxy fence orders these stores before the
// producer's bulk copies of the block, which follow the appender's count.
// ---------------------------------------------------------------------------
template <int D, bool MIXED>
__device__ __forceinline__ void append_rows(const DecodeArgs& a, int item, int lane) {
  using S = Shape<D>;
  const PoolView& P = a.pool;
  int b, kvh, split;
  item_coords(a, item, b, kvh, split);
  const int old = a.seq_lens[b];
  // add_const is max_new here: rows past it are not read (as in the append kernel)
  const int nn = a.add_lens != nullptr ? min(a.add_lens[b], a.add_const) : a.add_const;
  const int tps = a.plan.tokens_per_split, mb = a.plan.max_blocks_per_seq;
  const int64_t cap = static_cast<int64_t>(mb) * kBlockTokens;
  // new rows i whose position old + i lies in this split
  const int64_t lo = max(static_cast<int64_t>(0), static_cast<int64_t>(split) * tps - old);
  const int64_t hi = min(static_cast<int64_t>(nn), static_cast<int64_t>(split + 1) * tps - old);
  if (old < 0 || lo >= hi) return;
  const int r = lane / S::LPV, j = lane % S::LPV;
  const bool rot = P.k_rotated != 0;
  const float ks = rot ? kRotScale<D> : 1.0f;
  for (int64_t i0 = lo; i0 < hi;) {
    const int64_t p0 = old + i0;
    const int64_t i1 = min(min(i0 + S::VPW, hi), i0 + (kBlockTokens - p0 % kBlockTokens));   // one block
    const bool live = i0 + r < i1;
    const int64_t i = live ? i0 + r : i1 - 1;   // lanes past the pass's rows read a real row, store nothing
    const int32_t blk = p0 < cap ? __ldg(a.tables + static_cast<int64_t>(b) * mb + p0 / kBlockTokens) : -1;
    const bool ok = blk >= 0 && blk < P.n_blocks();
    if (!ok && lane == 0) raise_error(P.error_word, p0 < cap ? Q4KV_DEVERR_BLOCK_ID : Q4KV_DEVERR_SEQ_LEN);
    const int bk = ok ? blk : 0;
    const int slot = static_cast<int>((old + i) % kBlockTokens);
    const int64_t src = b * a.app_seq_stride + i * a.app_token_stride + kvh * D + j * kEPL;
    const uint4* kp = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.app_k) + src);
    const uint4* vp = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.app_v) + src);
    const uint4 k0 = __ldg(kp), k1 = __ldg(kp + 1), v0 = __ldg(vp), v1 = __ldg(vp + 1);
    float2 xk[8], xv[8];
    if (a.app_dtype == Q4KV_BF16) {
      unpack16<__nv_bfloat16>(k0, k1, xk);
      unpack16<__nv_bfloat16>(v0, v1, xv);
    } else {
      unpack16<__half>(k0, k1, xk);
      unpack16<__half>(v0, v1, xv);
    }
    if (rot) rotate_pairs<D>(xk, j);
    const bool valid = live && ok;
    const int bits = MIXED ? P.bits_of(bk) : 4;   // the same for the whole pass
    const int64_t phys = bits == 4 ? bk : (bits == 8 ? bk - P.n_q4 : bk - P.n_q4 - P.n_q8);
    const int64_t row = (phys * P.n_kv_heads + kvh) * kBlockTokens + slot;   // (block, head, slot)
    if (MIXED && bits == 8)
      encode_kv<8>(xk, ks, xv, j, valid, P.k_codes8 + row * D, P.k_params8 + row * S::NG, P.v_codes8 + row * D,
                   P.v_params8 + row * S::NG);
    else if (MIXED && bits == 2)
      encode_kv<2>(xk, ks, xv, j, valid, P.k_codes2 + row * (D / 4), P.k_params2 + row * S::NG,
                   P.v_codes2 + row * (D / 4), P.v_params2 + row * S::NG);
    else
      encode_kv<4>(xk, ks, xv, j, valid, P.k_codes4 + row * (D / 2), P.k_params4 + row * S::NG,
                   P.v_codes4 + row * (D / 2), P.v_params4 + row * S::NG);
    if (valid && j == 0)
      atomicAnd(P.mask + static_cast<int64_t>(bk) * kMaskWords + slot / 32, ~(1u << (slot % 32)));
    i0 = i1;
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
// MIXED: the pool may hold 8- or 2-bit blocks beside the 4-bit ones; a pool
// of 4-bit blocks only runs an instantiation without those paths (fewer
// registers held for them).  APP: a fused append (DecodeArgs::app_k), done by
// one more warp (the appender); a plain decode runs an instantiation without
// it.
template <int D, int LAY, bool FP8, bool MIXED, bool APP>
__global__ void __launch_bounds__(Cfg<D>::kThreads + (APP ? 32 : 0), 1)
    decode_tc_kernel(const __grid_constant__ DecodeArgs a, const __grid_constant__ TileMaps maps,
                     int n_items) {
  using C = Cfg<D>;
  constexpr int CW = C::CW;
  constexpr int kNS = Stg<D>::kNS, kStageBytes = Stg<D>::kStageBytes;
  constexpr int kOffV = Stg<D>::kOffV, kOffKP = Stg<D>::kOffKP, kOffVP = Stg<D>::kOffVP;
  constexpr int kOffMask = Stg<D>::kOffMask, kOffMeta = Stg<D>::kOffMeta;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // swizzled TMA tiles need 1024-byte aligned destinations
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* empty = full + kNS;
  uint64_t* qready = empty + kNS;   // [2] aux -> consumers: query table of an item ready
  uint64_t* done = qready + 2;      // [2] consumers -> aux: item merged-in, its table free
  uint64_t* mfree = done + 2;       // aux -> consumers: merge buffer read
  // appender -> producer: how many of the CTA's items have their appended rows in the pool
  uint32_t* n_enc = reinterpret_cast<uint32_t*>(mfree + 1);
  uint8_t* qtab0 = smem + C::kOffQTab;
  int* qint = reinterpret_cast<int*>(smem + C::kOffQInt);
  int* gsum = reinterpret_cast<int*>(smem + C::kOffQAux);
  float* escale = reinterpret_cast<float*>(smem + C::kOffQAux + 128);
  float* mrg_o = reinterpret_cast<float*>(smem + C::kOffMrgO);
  float* mrg_ml = reinterpret_cast<float*>(smem + C::kOffMrgML);
  int* mrg_flag = reinterpret_cast<int*>(smem + C::kOffMrgF);
  float* aux_f = reinterpret_cast<float*>(smem + C::kOffAuxW);
  float* aux_den = aux_f + CW * 8;

  // Earlier kernels in the stream (the encoder) have finished -- unless the
  // one before is an append, whose blocks only the producer waits for.
  if (!a.defer_wait) griddep_wait();
  griddep_launch_dependents();
  const PoolView& P = a.pool;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hkv = P.n_kv_heads, hq = a.plan.n_q_heads, G = hq / hkv;
  const int tps = a.plan.tokens_per_split, mb = a.plan.max_blocks_per_seq;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], CW);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&qready[i], 1);
      mbar_init(&done[i], CW);
    }
    mbar_init(mfree, 1);
    *n_enc = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (FP8) {   // heads past G of the FP8 query tables stay zero
    for (int i = threadIdx.x; i < 2 * C::kQTabBytes / 16; i += C::kThreads)
      reinterpret_cast<uint4*>(qtab0)[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();

  // -------------------------------------------------------------------------
  // producer warp
  // -------------------------------------------------------------------------
  if (warp == C::kProducer) {
    if (lane != 0) return;
    // the first copies need the tensor maps: fetch their descriptors now
    const CUtensorMap* used[2] = {FP8 ? &maps.k8 : &maps.k4, FP8 ? &maps.v8 : &maps.v4};
    for (int m = 0; m < 2; ++m)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(used[m])) : "memory");
    uint32_t it = 0;
    bool gave_up = false;
    // Global reads are issued ahead of the waits that follow them: the next
    // item's sequence length one item ahead, and a stage's block-table entry
    // before the wait for its free slot.  Read only after the slot frees,
    // their latency (about a microsecond under load) would add to every
    // stage's time in flight.
    // (x = the length before an append, y = the length decoded)
    auto seq_of = [&](int item) {
      int b, kvh, split;
      item_coords(a, item, b, kvh, split);
      return make_int2(a.seq_lens[b], seq_len_of(a, b));
    };
    // An append just before: its writes land in blocks at or past the old
    // length, which are read only after waiting for the append grid.
    bool waited = !a.defer_wait;
    // A fused append: item k's rows are in the pool once the appender's count
    // passes k, waited for before the item's first block at or past the old
    // length.
    constexpr bool fused = APP && !FP8;
    int2 seq_next = blockIdx.x < n_items ? seq_of(blockIdx.x) : make_int2(0, 0);
    int k = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++k) {
      int b, kvh, split;
      item_coords(a, item, b, kvh, split);
      bool enc_wait = fused;
      const int seq = seq_next.y, fresh_blk = seq_next.x / kBlockTokens;
      if (item + static_cast<int>(gridDim.x) < n_items) seq_next = seq_of(item + gridDim.x);
      const bool bad_seq = seq < 0 || seq > mb * kBlockTokens;
      if (bad_seq && split == 0 && kvh == 0) raise_error(P.error_word, Q4KV_DEVERR_SEQ_LEN);
      const int t0 = split * tps;
      const int t1 = bad_seq ? t0 : min(t0 + tps, seq);
      int tok = t0;
      do {
        const int s = it % kNS;
        // (read whenever the position is inside the table row, so the load
        // does not wait for the sequence length it is checked against)
        const int32_t blk_read =
            tok < mb * kBlockTokens ? a.tables[static_cast<int64_t>(b) * mb + tok / kBlockTokens] : -1;
        // A stage that stays taken past the limit ends production: writing
        // the stage or arriving on its full barrier could then land in a
        // phase the consumers have not finished.  Their own bounded waits
        // run out in turn and they report the timeout.
        if (!mbar_wait_idle(&empty[s], ((it / kNS) & 1) ^ 1, 32, 128)) {
          gave_up = true;
          break;
        }
        if (enc_wait && tok < t1 && tok / kBlockTokens >= fresh_blk) {
          if (!wait_count(n_enc, static_cast<uint32_t>(k + 1))) {
            gave_up = true;
            break;
          }
          enc_wait = false;
        }
        uint8_t* stg = stages + s * kStageBytes;
        StageMeta meta;
        meta.tok0 = tok;
        meta.poison = bad_seq;
        meta.pad = 0;
        meta.blk = -1;
        meta.bits = 4;
        meta.slot0 = static_cast<int16_t>(tok % kBlockTokens);
        int step = Geo<D, 4>::TS;
        if (tok < t1) {
          // a stage never crosses a block boundary, whatever the split length
          const int32_t blk = blk_read;
          if (blk < 0 || blk >= P.n_blocks()) {
            raise_error(P.error_word, Q4KV_DEVERR_BLOCK_ID);
            meta.poison = 1;
          } else {
            meta.blk = blk;
            meta.bits = static_cast<uint8_t>(P.bits_of(blk));
            if (meta.bits == 8) step = Geo<D, 8>::TS;
            if (meta.bits == 2) step = Geo<D, 2>::TS;
          }
          step = min(step, kBlockTokens - tok % kBlockTokens);
        }
        meta.ntok = static_cast<int16_t>(max(0, min(step, t1 - tok)));
        meta.last = (tok + step >= t1) ? 1 : 0;
        *reinterpret_cast<StageMeta*>(stg + kOffMeta) = meta;
        if (meta.blk >= 0) {
          if (!waited && tok / kBlockTokens >= fresh_blk) {
            griddep_wait();
            waited = true;
          }
          const int rows = (meta.ntok + 15) & ~15;   // whole 16-token tiles, inside the block
          const int bits = meta.bits;
          const int64_t phys = bits == 4 ? meta.blk : (bits == 8 ? meta.blk - P.n_q4 : meta.blk - P.n_q4 - P.n_q8);
          const int64_t row = (phys * hkv + kvh) * kBlockTokens + meta.slot0;
          const int pb = (D / kGroup) * 4;
          const __half2* kp = bits == 4 ? P.k_params4 : (bits == 8 ? P.k_params8 : P.k_params2);
          const __half2* vp = bits == 4 ? P.v_params4 : (bits == 8 ? P.v_params8 : P.v_params2);
          const uint8_t* kpp = reinterpret_cast<const uint8_t*>(kp) + row * pb;
          const uint8_t* vpp = reinterpret_cast<const uint8_t*>(vp) + row * pb;
          // codes: one TS-row box per tensor (rows past the block are never read as valid)
          const int ts = bits == 4 ? Geo<D, 4>::TS : (bits == 8 ? Geo<D, 8>::TS : Geo<D, 2>::TS);
          const int rb = D * bits / 8;
          const uint32_t cb = static_cast<uint32_t>(ts) * rb, prb = FP8 ? 0u : rows * pb;   // FP8: no params
          const CUtensorMap* km = bits == 4 ? &maps.k4 : (bits == 8 ? &maps.k8 : &maps.k2);
          const CUtensorMap* vm = bits == 4 ? &maps.v4 : (bits == 8 ? &maps.v8 : &maps.v2);
          mbar_arrive_tx(&full[s], 2 * cb + 2 * prb + 32);
          tma_rows(stg, km, static_cast<int>(row), &full[s]);
          tma_rows(stg + kOffV, vm, static_cast<int>(row), &full[s]);
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
    if (!waited) griddep_wait();   // this grid never completes before the append
    return;
  }

  // -------------------------------------------------------------------------
  // appender warp (fused append): every item's new rows, in item order
  // -------------------------------------------------------------------------
  if constexpr (APP && !FP8) {
    if (warp == C::kAppender) {
      uint32_t k = 0;
      for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        append_rows<D, MIXED>(a, item, lane);
        __syncwarp();
        if (lane == 0) st_release_cta(n_enc, ++k);
      }
      return;
    }
  }

  // -------------------------------------------------------------------------
  // the first item's query table, prepared by the consumer warps and the aux
  // warp together (heads, then table entries, spread over the warps)
  // -------------------------------------------------------------------------
  {
    constexpr int NT = (CW + 1) * 32;
    const int wid = warp < CW ? warp : CW;
    int b0, kvh0, split0;
    item_coords(a, blockIdx.x, b0, kvh0, split0);
    for (int h = wid; h < G; h += CW + 1) {
      if (FP8) prep_fp8_head<D>(a, b0, kvh0, h, qtab0, lane);
      else prep_head<D>(a, b0, kvh0, h, qint, gsum, escale, lane);
    }
    if (!FP8) {
      named_sync(1, NT);
      for (int e = wid * 32 + lane; e < C::KK * 32 + 32; e += NT) {
        if (e < C::KK * 32) prep_entry<D, LAY>(e / 32, e % 32, G, qint, qtab0);
        else prep_consts<D, LAY>(a, e - C::KK * 32, G, gsum, escale, qtab0);
      }
    }
    named_sync(1, NT);
    if (warp == C::kAux && lane == 0) mbar_arrive(&qready[0]);
  }

  // -------------------------------------------------------------------------
  // aux warp: query tables one item ahead, merge of the item just finished
  // -------------------------------------------------------------------------
  if (warp == C::kAux) {
    auto prep = [&](int item, int buf) {
      uint8_t* tab = qtab0 + buf * C::kQTabBytes;
      if (FP8) prep_fp8<D>(a, item, tab, lane);
      else prep_q4<D, LAY>(a, item, tab, qint, gsum, escale, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&qready[buf]);
    };
    const int i0 = blockIdx.x, i1 = blockIdx.x + gridDim.x;
    if (i1 < n_items) prep(i1, 1);
    int k = 0;
    bool timed_out = false;
    for (int item = i0; item < n_items; item += gridDim.x, ++k) {
      const int buf = k & 1;
      bool late = false;
      // back-off capped at 256 ns: the wait after the CTA's last item is on
      // the kernel's critical path
      if (!timed_out && !mbar_wait_idle(&done[buf], (k >> 1) & 1, 64, 256)) {
        timed_out = late = true;
        if (lane == 0) raise_error(P.error_word, Q4KV_DEVERR_TIMEOUT);
      }
      merge_item<D>(a, item, mrg_o, mrg_ml, mrg_flag, aux_f, aux_den, late || timed_out, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(mfree);
      const int nitem = item + 2 * gridDim.x;
      if (nitem < n_items && !timed_out) prep(nitem, buf);
    }
    return;
  }

  // -------------------------------------------------------------------------
  // consumer warps
  // -------------------------------------------------------------------------
  const int g = lane >> 2, t = lane & 3;
  uint32_t it = 0;
  bool dead = false;
  const int row0 = warp * 16;   // the warp's base row: its first tile of a whole stage
  PairOffsets<D, 4> poff4;
  HeadOffsets<D, 4> hoff4;
  PairOffsets<D, 8> off8f;
  if (LAY == kPairs) poff4.init(lane, row0);
  else hoff4.init(lane, row0);
  if (FP8) off8f.init(lane, row0);
  PairState<D> pst;
  HeadState<D> hst;
  Fp8State<D> fst;
  using BQ = typename std::conditional<C::template kBqSmem<LAY>, BqSmem<D / 32>, BqRegs<D / 32>>::type;
  BQ bq;
  PairConst pc;
  HeadConst<D> hc;
  int k = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++k) {
    const int buf = k & 1;
    if (!dead && !mbar_wait(&qready[buf], (k >> 1) & 1)) dead = true;
    const uint8_t* tab = qtab0 + buf * C::kQTabBytes;
    const uint4* qtab_t = reinterpret_cast<const uint4*>(tab) + g * (D / 16) * 4 + t;
    if (!FP8) {
      bq.load(reinterpret_cast<const uint2*>(tab), lane);
      const float* cst = reinterpret_cast<const float*>(tab + C::kBqBytes) + lane * 12;
      if (LAY == kPairs) {
        pc.qs[0] = cst[0];
        pc.qs[1] = cst[1];
        pc.ks = cst[2];
      } else {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          hc.ks[c] = cst[c];
#pragma unroll
          for (int gr = 0; gr < C::NG; ++gr) hc.qs[c][gr] = cst[2 + c * C::NG + gr];
        }
      }
    }
    if (FP8) reset(fst);
    else if (LAY == kPairs) reset(pst);
    else reset(hst);
    bool poison = false;
    int tau = 0;   // 16-token tiles of this item before the current stage

    // Tiles of one block class, one or two at a time (two share one softmax
    // update; 8- and 2-bit offsets are made on demand).
    // Tile places are row deltas from the warp's base row (warp * 16).
    auto run = [&](auto ntl, const TileAt (&ta)[decltype(ntl)::value], int cb) {
      constexpr int NTL = decltype(ntl)::value;
      if constexpr (FP8) {
#pragma unroll
        for (int x = 0; x < NTL; ++x) fp8_tile<D>(fst, ta[x], off8f, qtab_t);
      } else if (!MIXED || cb == 4) {
        if (LAY == kPairs) pair_tiles<D, 4, NTL>(pst, ta, poff4, bq, pc);
        else head_tiles<D, 4, NTL>(hst, ta, hoff4, bq, hc);
      } else if (cb == 8) {
        if (LAY == kPairs) {
          PairOffsets<D, 8> o8;
          o8.init(lane, row0);
          pair_tiles<D, 8, NTL>(pst, ta, o8, bq, pc);
        } else {
          HeadOffsets<D, 8> o8;
          o8.init(lane, row0);
          head_tiles<D, 8, NTL>(hst, ta, o8, bq, hc);
        }
      } else {
        if (LAY == kPairs) {
          PairOffsets<D, 2> o2;
          o2.init(lane, row0);
          pair_tiles<D, 2, NTL>(pst, ta, o2, bq, pc);
        } else {
          HeadOffsets<D, 2> o2;
          o2.init(lane, row0);
          head_tiles<D, 2, NTL>(hst, ta, o2, bq, hc);
        }
      }
    };
    // Two tiles per call where registers allow it (D = 128); at D = 256 the
    // value accumulators alone take 64 registers, and tiles go one at a time.
    constexpr bool kPairTiles = D == 128 && !FP8;
    using One = std::integral_constant<int, 1>;
    using Two = std::integral_constant<int, 2>;
    // A single tile of a stage waits for a partner from the item's next stage
    // (same block class); its stage is released once it has been processed.
    bool has_p = false;
    int p8 = 4;   // the pending tile's code bits
    TileAt pend = {stages, 0, 0, 0};
    int p_s = 0;
    auto flush = [&]() {
      if (!has_p) return;
      const TileAt ta[1] = {pend};
      run(One{}, ta, p8);
      __syncwarp();
      if (lane == 0 && !dead) mbar_arrive(&empty[p_s]);
      has_p = false;
    };

    // ---- the item's stages; warp w takes the item's tiles w, w + CW, ... ----
    for (;;) {
      const int s = it % kNS;
      if (!dead && !mbar_wait_hot(&full[s], (it / kNS) & 1)) dead = true;
      const uint8_t* stg = stages + s * kStageBytes;
      const StageMeta meta = *reinterpret_cast<const StageMeta*>(stg + kOffMeta);
      const bool last = dead ? true : meta.last;
      poison |= meta.poison;
      bool release = true;
      if (!dead && meta.blk >= 0) {
        const int q8 = meta.bits;
        const int ntiles = (meta.ntok + 15) >> 4;   // <= 16 <= 2 CW: at most two are this warp's
        const int i0 = (warp - tau % CW + CW) % CW, i1 = i0 + CW;
        const int sb = meta.slot0 + row0, nv = meta.ntok - row0;
        if (!kPairTiles) {
#pragma unroll 1
          for (int i = i0; i < ntiles; i += CW) {
            const TileAt ta[1] = {{stg, 16 * i - row0, sb, nv}};
            run(One{}, ta, q8);
          }
        } else if (i1 < ntiles) {
          flush();
          const TileAt ta[2] = {{stg, 16 * i0 - row0, sb, nv}, {stg, 16 * i1 - row0, sb, nv}};
          run(Two{}, ta, q8);
        } else if (i0 < ntiles) {
          const TileAt cur = {stg, 16 * i0 - row0, sb, nv};
          if (has_p && p8 == q8) {
            const TileAt ta[2] = {pend, cur};
            run(Two{}, ta, q8);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[p_s]);
            has_p = false;
          } else {
            flush();
            if (last) {
              const TileAt ta[1] = {cur};
              run(One{}, ta, q8);
            } else {
              has_p = true;
              p8 = q8;
              pend = cur;
              p_s = s;
              release = false;
            }
          }
        }
        tau += ntiles;
      }
      if (last) flush();
      __syncwarp();
      if (lane == 0 && !dead && release) mbar_arrive(&empty[s]);
      ++it;
      if (last) break;
    }

    // ---- hand the item's state to the aux warp ----
    if (k > 0 && !dead && !mbar_wait(mfree, (k - 1) & 1)) dead = true;
    float* mo = mrg_o + warp * D * C::HP;
    float* mml = mrg_ml + warp * 16;
    if (FP8) {
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
          mml[h * 2] = fst.m[c];
          mml[h * 2 + 1] = lt[c];
        }
      }
      if (2 * t < G) {
#pragma unroll
        for (int mv = 0; mv < D / 16; ++mv)
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int ch = (D / 8) * g + 2 * mv + r;
            *reinterpret_cast<float2*>(mo + ch * C::HP + 2 * t) = make_float2(fst.o[mv][2 * r], fst.o[mv][2 * r + 1]);
          }
      }
    } else if (LAY == kPairs) {
      constexpr int NG = C::NG;
      float lt = pst.l, z0 = pst.z[0], z1 = pst.z[1];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        lt += __shfl_xor_sync(0xffffffffu, lt, off);
        z0 += __shfl_xor_sync(0xffffffffu, z0, off);
        z1 += __shfl_xor_sync(0xffffffffu, z1, off);
      }
      const int c0 = 2 * t;
      const int h = c0 / NG;
      if (g == 0 && h < G && (NG == 2 || (t & 1) == 0)) {
        mml[h * 2] = pst.m;
        mml[h * 2 + 1] = lt;
      }
      const float zz[2] = {z0, z1};
#pragma unroll
      for (int mv = 0; mv < D / 16; ++mv) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int ch = kGroup * (mv / 4) + 32 * (e >> 1) + 4 * g + mv % 4;   // value tile mv = 4 gr + j
          const int col = c0 + (e & 1);
          const int hh = col / NG, gr = col % NG;
          const float sc = mv % 2 == 0 ? kEvenScale : kOddScale;
          if (hh < G && gr == ch / kGroup) mo[ch * C::HP + hh] = __fmaf_rn(pst.o[mv][e], sc, zz[e & 1]);
        }
      }
    } else {
      constexpr int NG = C::NG;
      float lt[2] = {hst.l[0], hst.l[1]};
      float zz[2][NG];
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int gr = 0; gr < NG; ++gr) zz[c][gr] = hst.z[c][gr];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          lt[c] += __shfl_xor_sync(0xffffffffu, lt[c], off);
#pragma unroll
          for (int gr = 0; gr < NG; ++gr) zz[c][gr] += __shfl_xor_sync(0xffffffffu, zz[c][gr], off);
        }
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int h = 2 * t + c;
        if (g == 0 && h < G) {
          mml[h * 2] = hst.m[c];
          mml[h * 2 + 1] = lt[c];
        }
      }
      if (2 * t < G) {
#pragma unroll
        for (int mv = 0; mv < D / 16; ++mv) {
          const int gr = mv / 4;
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int ch = kGroup * gr + 32 * r + 4 * g + mv % 4;   // value tile mv = 4 gr + j
            const float sc = mv % 2 == 0 ? kEvenScale : kOddScale;
            *reinterpret_cast<float2*>(mo + ch * C::HP + 2 * t) =
                make_float2(__fmaf_rn(hst.o[mv][2 * r], sc, zz[0][gr]),
                            __fmaf_rn(hst.o[mv][2 * r + 1], sc, zz[1][gr]));
          }
        }
      }
    }
    if (lane == 0) mrg_flag[warp] = (poison || dead) ? 1 : 0;
    __syncwarp();
    if (lane == 0) mbar_arrive(&done[buf]);
    if (dead && lane == 0) raise_error(P.error_word, Q4KV_DEVERR_TIMEOUT);
  }
}

}  // namespace

size_t decode_tc_smem_bytes(int head_dim) {
  return 1024 + static_cast<size_t>(head_dim == 128 ? Cfg<128>::kSmem : Cfg<256>::kSmem);
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
  const CUtensorMapSwizzle sw = row_bytes == 32    ? CU_TENSOR_MAP_SWIZZLE_32B
                                : row_bytes == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
                                : row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                                   : CU_TENSOR_MAP_SWIZZLE_NONE;
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Column layout for a shape: pairs when every (head, group) pair fits one
// 8-column n-tile, else heads.
int decode_tc_layout(int head_dim, int g) { return g * (head_dim / kGroup) <= 8 ? kPairs : kHeads; }

cudaError_t launch_decode_tc(const DecodeArgs& a, int num_sms, cudaStream_t stream) {
  const q4kv_decode_plan& p = a.plan;
  const int n_items = p.batch * p.n_kv_heads * p.n_splits;
  const int grid = min(n_items, num_sms);
  const int g = p.n_q_heads / p.n_kv_heads;
  const size_t smem = decode_tc_smem_bytes(p.head_dim);
  if (g > 8 || g * p.head_dim > 1024) return cudaErrorInvalidValue;

  EncodeFn enc = tensor_map_encoder();
  if (enc == nullptr) return cudaErrorNotSupported;
  TileMaps maps;
  memset(&maps, 0, sizeof(maps));
  const int d = p.head_dim;
  const uint64_t per_block = static_cast<uint64_t>(a.pool.n_kv_heads) * kBlockTokens;
  const uint32_t ts4 = d == 128 ? Geo<128, 4>::TS : Geo<256, 4>::TS;
  const uint32_t ts8 = d == 128 ? Geo<128, 8>::TS : Geo<256, 8>::TS;
  const uint32_t ts2 = d == 128 ? Geo<128, 2>::TS : Geo<256, 2>::TS;
  if (a.pool.n_q4 > 0 &&
      (!encode_rows(enc, &maps.k4, a.pool.k_codes4, a.pool.n_q4 * per_block, d / 2, ts4) ||
       !encode_rows(enc, &maps.v4, a.pool.v_codes4, a.pool.n_q4 * per_block, d / 2, ts4)))
    return cudaErrorInvalidValue;
  if (a.pool.n_q8 > 0 &&
      (!encode_rows(enc, &maps.k8, a.pool.k_codes8, a.pool.n_q8 * per_block, d, ts8) ||
       !encode_rows(enc, &maps.v8, a.pool.v_codes8, a.pool.n_q8 * per_block, d, ts8)))
    return cudaErrorInvalidValue;
  if (a.pool.n_q2 > 0 &&
      (!encode_rows(enc, &maps.k2, a.pool.k_codes2, a.pool.n_q2 * per_block, d / 4, ts2) ||
       !encode_rows(enc, &maps.v2, a.pool.v_codes2, a.pool.n_q2 * per_block, d / 4, ts2)))
    return cudaErrorInvalidValue;

  cudaError_t e = cudaSuccess;
#define Q4KV_TC(DD, LL, F8, MX, AP)                                                                 \
  do {                                                                                             \
    e = cudaFuncSetAttribute(decode_tc_kernel<DD, LL, F8, MX, AP>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                             static_cast<int>(smem));                                              \
    if (e == cudaSuccess)                                                                          \
      e = launch_pdl(decode_tc_kernel<DD, LL, F8, MX, AP>, dim3(grid), dim3(Cfg<DD>::kThreads + (AP ? 32 : 0)), \
                     smem, stream, a, maps, n_items);                                              \
  } while (0)
#define Q4KV_TCM(DD, LL)                           \
  do {                                             \
    if (mixed && app) Q4KV_TC(DD, LL, false, true, true);   \
    else if (mixed) Q4KV_TC(DD, LL, false, true, false);    \
    else if (app) Q4KV_TC(DD, LL, false, false, true);      \
    else Q4KV_TC(DD, LL, false, false, false);              \
  } while (0)
  const int lay = decode_tc_layout(d, g);
  const bool mixed = a.pool.n_q8 > 0 || a.pool.n_q2 > 0;
  const bool app = a.app_k != nullptr;   // never set for FP8 pools (their appends run the append kernel)
  if (a.pool.fp8 && d == 128) Q4KV_TC(128, kHeads, true, false, false);   // FP8 comparison cache: heads are the columns
  else if (a.pool.fp8) Q4KV_TC(256, kHeads, true, false, false);
  else if (d == 128 && lay == kPairs) Q4KV_TCM(128, kPairs);
  else if (d == 128) Q4KV_TCM(128, kHeads);
  else if (lay == kPairs) Q4KV_TCM(256, kPairs);
  else Q4KV_TCM(256, kHeads);
#undef Q4KV_TCM
#undef Q4KV_TC
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace q4kv
