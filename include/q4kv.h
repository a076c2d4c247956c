/*
 * q4kv.h -- C ABI of the B200 (sm_100a) 4-bit paged KV cache and its decode
 * attention.
 *
 * Source pages (cited by title and section):
 *   [AMBP] "Agent Memory Below the Prompt: Persistent Q4 KV Cache for
 *          Multi-Agent LLM Inference on Edge Devices" (gist.science summary of
 *          arXiv 2603.04428).  Sec. 2.1 item 1: 256-token blocks per agent.
 *          Sec. 2.1 item 2: 4-bit codes packed in uint32 words, one 16-bit
 *          scale and one 16-bit bias per group, read by attention directly
 *          ("direct restore").  Sec. 2.1 item 3: attention batched over many
 *          agents' quantised caches, one agent decoding while another's
 *          cache is brought in.  Sec. 2.1 item 4: a prompt that extends a
 *          cached prefix (EXTEND match) grows the cache instead of being
 *          prefilled again.  Sec. 2.2: GQA.
 *   [UQ]   UltraQuant news item (poko-everyday.com, arXiv 2606.20474),
 *          section "技術/ビジネス面": Walsh-Hadamard rotation before 4-bit
 *          quantisation; keys and values treated asymmetrically.
 *   [IKV]  IntentKV article (Qiita), section "詰め直さずに「無効化」する":
 *          evicted slots are re-pointed to a sentinel slot with key -1e4,
 *          whose softmax weight is zero; surviving slots do not move.
 *   [QKVS] QKVShare (gist.science summary of arXiv 2605.03884),
 *          "Méthodologie": per-token widths from {2, 4, 8, FP16}; the
 *          receiver dequantises the shared cache before use.
 *
 * Format (fixed by this library):
 *   - 256 tokens per block; one block holds every KV head of those tokens.
 *   - Groups of 64 consecutive values along head_dim of one (token, head)
 *     vector; per group an fp16 scale s and an fp16 zero z (additive offset);
 *     value = code * s + z.
 *   - K is stored rotated by c*H_D (Sylvester Walsh-Hadamard, c = binary32
 *     nearest 1/sqrt(D), butterfly strides 1, 2, ..., D/2 in that order);
 *     V is stored unrotated.  The query is rotated by the same transform
 *     inside attention, so no inverse rotation is needed on the output.
 *   - 4-bit codes: two per byte, element 2i in the low nibble of byte i
 *     (element j of a little-endian uint32 word at bits 4*(j%8)).
 *     8-bit codes: one per byte.
 *   - Codes are computed from the stored fp16 s and z:
 *       s = fl((max - min) / L), L = 15 or 255;  z = fp16(min)
 *       code = 0 if fp16(s) == 0 else clamp(rne(fl(fl(x - z) / s)), 0, L)
 *     with binary32 IEEE subtraction and division (bit-exact everywhere).
 *   - An evicted slot is flagged in a per-block 256-bit mask shared by all
 *     KV heads; its data stays in place.  Attention gives it logit -1e4 and
 *     value 0, so its weight is exactly 0 whenever any live logit exceeds
 *     -9896; a sequence whose every slot is evicted returns 0.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates or frees device memory.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and returns without waiting, except q4kv_read_device_error.
 *   - Arguments are checked on the host first; on any failure the call
 *     returns an error status and launches nothing.
 *   - Faults found on the device (an out-of-range block id in a table or a
 *     block-id list, an out-of-range slot id, a sequence length beyond its
 *     table) never trap: the offending item is skipped, the affected output
 *     row is written as 0, and a Q4KV_DEVERR_* bit is OR-ed into
 *     pool->error_word when that pointer is non-NULL.
 *   - No C++ exception crosses this interface.
 */
#ifndef Q4KV_H
#define Q4KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define Q4KV_ABI_VERSION 4
#define Q4KV_BLOCK_TOKENS 256
#define Q4KV_GROUP 64
#define Q4KV_MASK_WORDS 8            /* uint32 words of remap mask per block */
#define Q4KV_SENTINEL_LOGIT (-1.0e4f)

typedef enum {
  Q4KV_OK = 0,
  Q4KV_ERR_INVALID_ARG = 1,   /* NULL pointer, negative size, misaligned pointer or stride, bad dtype */
  Q4KV_ERR_UNSUPPORTED = 2,   /* well-formed but outside what the kernels cover (head_dim, GQA ratio) */
  Q4KV_ERR_CUDA = 3,          /* a CUDA runtime call or a kernel launch failed */
  Q4KV_ERR_WORKSPACE = 4,     /* workspace NULL or smaller than plan->workspace_bytes */
  Q4KV_ERR_DEVICE = 5         /* q4kv_read_device_error found device error bits set */
} q4kv_status;

/* Bits of pool->error_word. */
#define Q4KV_DEVERR_BLOCK_ID 1u  /* a block id outside [0, n_q4_blocks + n_q8_blocks + n_q2_blocks) */
#define Q4KV_DEVERR_SEQ_LEN 2u   /* seq_len < 0 or > max_blocks_per_seq * 256 */
#define Q4KV_DEVERR_SLOT_ID 4u   /* a slot id outside [0, 256 * (n_q4 + n_q8 + n_q2 blocks)) */
#define Q4KV_DEVERR_TIMEOUT 8u   /* a bounded device-side wait gave up */
#define Q4KV_DEVERR_IMAGE 16u    /* a block image or card whose header or layout does not fit */
#define Q4KV_DEVERR_WIDTH 32u    /* a card token width outside {2, 4, 8, 16} */

typedef enum { Q4KV_F16 = 0, Q4KV_BF16 = 1, Q4KV_F32 = 2 } q4kv_dtype;

/*
 * Value formats of a pool (q4kv_pool.value_format).
 *   Q4KV_FORMAT_INT  4-bit (and optional 8- and 2-bit) integer codes with a
 *                    scale and a zero per group of 64, as described above.
 *   Q4KV_FORMAT_FP8  the FP8 cache the 4-bit cache is compared against ([UQ]
 *                    "技術/ビジネス面": TTFT and throughput are reported against
 *                    an FP8 KV cache).  Every value is one OCP E4M3 byte
 *                    (1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
 *                    no infinities; largest finite 448) holding the input value
 *                    rounded to nearest, ties to even, saturated to +-448; no
 *                    scale and no rotation.  Such a pool has n_q4_blocks = 0,
 *                    n_q2_blocks = 0 and k_rotated = 0, keeps its codes in k_codes8 / v_codes8
 *                    [n_q8][Hkv][256][D], and has no params (their pointers are
 *                    ignored).  Quantise, append, dequantise, invalidate and
 *                    decode all accept it.
 */
#define Q4KV_FORMAT_INT 0
#define Q4KV_FORMAT_FP8 1

/*
 * The paged pool ([AMBP] sec. 2.1 items 1-2; 8- and 2-bit blocks: [QKVS]
 * "Méthodologie", widths from {2, 4, 8, FP16} in one cache, here per block).
 * Unified block ids: [0, n_q4_blocks) are 4-bit blocks, stored at index id
 * of the *4 arrays; [n_q4_blocks, n_q4_blocks + n_q8_blocks) are 8-bit blocks,
 * stored at index id - n_q4_blocks of the *8 arrays; the next n_q2_blocks ids
 * are 2-bit blocks, stored at index id - n_q4_blocks - n_q8_blocks of the *2
 * arrays.  Every class codes a group of 64 values with the same steps and
 * L = 2^bits - 1 levels.
 * Every array pointer must be 16-byte aligned.  Layouts (row-major):
 *   k_codes4, v_codes4   uint8 [n_q4][Hkv][256][D/2]    (element 2i in the low nibble of byte i)
 *   k_params4, v_params4 half2 [n_q4][Hkv][256][D/64]   (.x = scale, .y = zero)
 *   k_codes8, v_codes8   uint8 [n_q8][Hkv][256][D]      (may be NULL if n_q8 == 0)
 *   k_params8, v_params8 half2 [n_q8][Hkv][256][D/64]
 *   k_codes2, v_codes2   uint8 [n_q2][Hkv][256][D/4]    (element 4i + m at bits 2m of byte i;
 *                                                        may be NULL if n_q2 == 0)
 *   k_params2, v_params2 half2 [n_q2][Hkv][256][D/64]
 *   remap_mask           uint32 [n_q4 + n_q8 + n_q2][8]; bit (s % 32) of word s / 32
 *                        set = slot s of that block is remapped to the sentinel
 *   error_word           optional uint32 (NULL = do not report)
 * The descriptor itself is read on the host during each call and may be
 * reused or freed afterwards.
 */
typedef struct {
  int32_t head_dim;     /* D: 128 or 256 */
  int32_t n_kv_heads;   /* Hkv >= 1 */
  int32_t k_rotated;    /* 1 = K stored Walsh-Hadamard rotated ([UQ]); 0 = raw */
  int32_t n_q4_blocks;  /* >= 0 */
  int32_t n_q8_blocks;  /* >= 0 */
  int32_t value_format; /* Q4KV_FORMAT_INT (0) or Q4KV_FORMAT_FP8 (1) */
  uint8_t *k_codes4, *v_codes4;
  void *k_params4, *v_params4;
  uint8_t *k_codes8, *v_codes8;
  void *k_params8, *v_params8;
  uint32_t *remap_mask;
  uint32_t *error_word;
  int32_t n_q2_blocks;  /* >= 0; 0 for an FP8 pool */
  int32_t reserved;     /* must be 0 */
  uint8_t *k_codes2, *v_codes2;
  void *k_params2, *v_params2;
} q4kv_pool;

/* Human-readable name of a status code (static storage). */
const char *q4kv_status_string(q4kv_status status);

/* Q4KV_ABI_VERSION of the loaded library. */
int32_t q4kv_abi_version(void);

/*
 * Bytes of one codes array and of one params array for `n_blocks` blocks of
 * width `bits` (2, 4 or 8), so a caller can size the pool ([AMBP] sec. 2.1
 * item 2: 144 bytes per token and KV head at D = 128, 4 bits, i.e. 71.875 %
 * below fp16).  Host-only; touches no device.
 */
q4kv_status q4kv_pool_array_bytes(int32_t head_dim, int32_t n_kv_heads, int64_t n_blocks,
                                  int32_t bits, size_t *codes_bytes, size_t *params_bytes);

/*
 * Quantise and store K/V of `n_tokens` tokens ([AMBP] sec. 2.1 item 2, [UQ]).
 *   k, v         device, dtype in_dtype (Q4KV_F16 or Q4KV_BF16); element
 *                (t, h, j) at index t*token_stride + h*D + j; 16-byte aligned;
 *                token_stride >= Hkv*D and token_stride*elem_size % 16 == 0.
 *                Values must be finite.
 *   block_ids    device int32 [ceil(n_tokens/256)]: token t is written to
 *                block block_ids[t/256], slot t % 256 (4- or 8-bit per the id).
 *   Writing a slot clears its remap bit (a freshly written slot is live).
 *   Codes, scales, zeros and packed bytes are bit-identical to the format's
 *   definition above.  n_tokens == 0 is a no-op.  A block id out of range
 *   skips its tokens and raises Q4KV_DEVERR_BLOCK_ID.
 */
q4kv_status q4kv_quantize_blocks(const q4kv_pool *pool, const void *k, const void *v,
                                 int32_t in_dtype, int64_t n_tokens, int64_t token_stride,
                                 const int32_t *block_ids, void *stream);

/*
 * Append new tokens to each sequence's cache at its own position ([AMBP]
 * sec. 2.1 items 3-4: decoding and EXTEND both grow a cached sequence in
 * place instead of prefilling it again).
 *   k, v         device, dtype in_dtype (Q4KV_F16 or Q4KV_BF16); token i of
 *                sequence b is the [Hkv][D] row at index
 *                b*seq_stride + i*token_stride (elements), rows contiguous;
 *                16-byte aligned, both strides * elem_size % 16 == 0,
 *                token_stride >= Hkv*D.  Values must be finite.
 *   batch, max_new  sequences and tokens per sequence in k / v.
 *   n_new        device int32 [batch] with 0 <= n_new[b] <= max_new, the
 *                tokens sequence b appends; NULL = every sequence appends
 *                max_new.
 *   tables       device int32 [batch][max_blocks]: logical block i of
 *                sequence b is physical block tables[b*max_blocks + i].
 *   seq_lens     device int32 [batch], lengths BEFORE the append (not
 *                modified; the caller adds n_new afterwards).
 *   Token i of sequence b is written to position p = seq_lens[b] + i, i.e.
 *   slot p % 256 of block tables[b][p / 256], encoded exactly as
 *   q4kv_quantize_blocks encodes the same row, and its remap bit is cleared.
 *   The positions written must map to distinct slots.  A position at or
 *   past max_blocks*256 (or a negative length) skips the token and raises
 *   Q4KV_DEVERR_SEQ_LEN; a block id out of range skips it and raises
 *   Q4KV_DEVERR_BLOCK_ID.  batch == 0 or max_new == 0 is a no-op.
 */
q4kv_status q4kv_append_tokens(const q4kv_pool *pool, const void *k, const void *v,
                               int32_t in_dtype, int32_t batch, int32_t max_new,
                               const int32_t *n_new, int64_t seq_stride, int64_t token_stride,
                               const int32_t *tables, int32_t max_blocks, const int32_t *seq_lens,
                               void *stream);

/*
 * Dequantise whole blocks ([QKVS] "Méthodologie": dequantise before use).
 *   block_ids    device int32 [n_blocks]
 *   k_out, v_out device [n_blocks][Hkv][256][D] of out_dtype (Q4KV_F32 or
 *                Q4KV_F16), 16-byte aligned; value = fl(code*s + z), fp16
 *                output rounds that to nearest even.
 *   unrotate_k   1 = apply c*H (its own inverse) to K after dequantisation,
 *                with the same butterfly order as the encoder (bit-exact).
 *   Remapped slots read the sentinel: K = -1e4 in every channel, V = 0.
 *   A block id out of range writes zeros for that block and raises
 *   Q4KV_DEVERR_BLOCK_ID.
 */
q4kv_status q4kv_dequantize(const q4kv_pool *pool, const int32_t *block_ids, int32_t n_blocks,
                            void *k_out, void *v_out, int32_t out_dtype, int32_t unrotate_k,
                            void *stream);

/*
 * Remap slots to the sentinel ([IKV]): sets their remap bits; data stays in
 * place and positions do not change.
 *   slot_ids     device int64 [n_slots], slot = block_id*256 + offset.
 *   Out-of-range ids are skipped and raise Q4KV_DEVERR_SLOT_ID.
 */
q4kv_status q4kv_invalidate_slots(const q4kv_pool *pool, const int64_t *slot_ids, int64_t n_slots,
                                  void *stream);

/*
 * Mean |K| of each 256-token chunk of raw (unrotated) keys, accumulated in
 * fp64 ([QKVS]: choose wider codes for the most demanding blocks).
 *   k            as in q4kv_quantize_blocks (same layout and alignment rules)
 *   out          device double [ceil(n_tokens/256)]; a short last chunk is
 *                averaged over its own tokens.
 */
q4kv_status q4kv_block_absmean(const void *k, int32_t in_dtype, int64_t n_tokens,
                               int64_t token_stride, int32_t n_kv_heads, int32_t head_dim,
                               double *out, void *stream);

/*
 * Block ids for a mixed 4/8-bit cache: the n_q8 chunks of highest absmean
 * (ties to the lower chunk index) get 8-bit ids, the rest 4-bit ids, each in
 * chunk order: the k-th 8-bit chunk gets q8_first + k, the k-th 4-bit chunk
 * q4_first + k.  absmean and block_ids are device arrays of n_chunks
 * entries; 0 <= n_q8 <= n_chunks <= 65536.
 */
q4kv_status q4kv_mixed_block_ids(const double *absmean, int32_t n_chunks, int32_t n_q8,
                                 int32_t q4_first, int32_t q8_first, int32_t *block_ids,
                                 void *stream);

/*
 * Launch plan of one decode-attention shape.  The context of every sequence
 * is cut into n_splits ranges of tokens_per_split tokens; each range yields a
 * partial (max, sum, weighted value) per query head, merged by log-sum-exp.
 */
typedef struct {
  int32_t batch;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t max_blocks_per_seq;  /* width of the block table */
  int32_t n_splits;
  int32_t tokens_per_split;    /* multiple of 64 */
  int32_t kernel;              /* kernel variant: 1 = tensor-core pipeline (what
                                  q4kv_decode_plan_make picks), 0 = the CUDA-core
                                  kernel (4/8-bit pools only; one CTA per item);
                                  any other value is rejected */
  size_t workspace_bytes;      /* device scratch the call needs (0 when n_splits == 1) */
} q4kv_decode_plan;

/*
 * Fill `plan` for a shape.  n_splits > 0 forces that split count (clamped to
 * the context); 0 lets the library choose from num_sms.  num_sms > 0 is used
 * as given; 0 queries the current CUDA device.  Host-only otherwise.
 * Supported: head_dim 128 or 256, 1 <= n_q_heads / n_kv_heads <= 8 and
 * (n_q_heads / n_kv_heads) * head_dim / 64 <= 16.
 */
q4kv_status q4kv_decode_plan_make(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                  int32_t head_dim, int32_t max_blocks_per_seq, int32_t n_splits,
                                  int32_t num_sms, q4kv_decode_plan *plan);

/*
 * Single-token paged GQA decode attention over the quantised cache
 * ([AMBP] sec. 2.1 items 2-3 and 2.2; [IKV] for remapped slots).
 *   q            device [batch][n_q_heads][D], q_dtype Q4KV_F16 or Q4KV_BF16
 *   block_tables device int32 [batch][max_blocks_per_seq]
 *   seq_lens     device int32 [batch], 0 <= seq_len <= max_blocks_per_seq*256
 *   softmax_scale  <= 0 selects 1/sqrt(D)
 *   out          device [batch][n_q_heads][D] of out_dtype (F32, F16 or BF16)
 *   workspace    device scratch of at least plan->workspace_bytes (may be
 *                NULL when that is 0), 256-byte aligned, not shared with a
 *                concurrent call.
 * Query head h reads KV head h / (n_q_heads / n_kv_heads).  Logits are
 * softmax_scale * <c*H q, K_hat> (or <q, K_hat> when K is stored raw); an
 * empty or fully remapped sequence returns 0.
 */
q4kv_status q4kv_decode_attention(const q4kv_pool *pool, const q4kv_decode_plan *plan,
                                  const void *q, int32_t q_dtype, const int32_t *block_tables,
                                  const int32_t *seq_lens, float softmax_scale, void *out,
                                  int32_t out_dtype, void *workspace, size_t workspace_bytes,
                                  void *stream);

/*
 * One generation step: append each sequence's new tokens, then decode over
 * the grown cache ([AMBP] sec. 2.1 item 4: EXTEND grows the cache in place,
 * then attention reads it).  Equal to q4kv_append_tokens followed by
 * q4kv_decode_attention with lengths seq_lens[b] + n_new[b] (the same pool
 * bytes and the same output), but faster.  For pools of 4-, 8- and 2-bit
 * blocks with plan->kernel == 1 it is one decode launch (plus the split
 * merge): one extra warp per CTA encodes the new rows of the CTA's items, and
 * the CTA reads a block at or past position seq_lens[b] -- the only blocks an
 * append writes -- only after those rows are in.  For FP8 pools and plan
 * kernel 0 the append kernel runs first and the decode starts while it runs
 * (programmatic dependent launch), waiting for it only before such blocks.
 *   plan         as for q4kv_decode_attention; plan->batch sequences and
 *                plan->max_blocks_per_seq block-table columns for both steps
 *   k_new, v_new, in_dtype, max_new, n_new, seq_stride, token_stride
 *                the new tokens, as for q4kv_append_tokens (batch =
 *                plan->batch); max_new == 0 decodes without appending
 *   q, q_dtype, block_tables, softmax_scale, out, out_dtype, workspace,
 *   workspace_bytes  as for q4kv_decode_attention
 *   seq_lens     device int32 [batch], the lengths BEFORE the append (not
 *                modified); sequence b is decoded over seq_lens[b] +
 *                n_new[b] tokens (+ max_new when n_new is NULL)
 * Errors as for the two calls; nothing is launched unless both sets of
 * arguments are valid.  Device-side errors (Q4KV_DEVERR_*) of either step go
 * to the pool's error word.
 */
q4kv_status q4kv_append_decode(const q4kv_pool *pool, const q4kv_decode_plan *plan, const void *k_new,
                               const void *v_new, int32_t in_dtype, int32_t max_new, const int32_t *n_new,
                               int64_t seq_stride, int64_t token_stride, const void *q, int32_t q_dtype,
                               const int32_t *block_tables, const int32_t *seq_lens, float softmax_scale,
                               void *out, int32_t out_dtype, void *workspace, size_t workspace_bytes,
                               void *stream);

/*
 * Decode attention for callers that cannot allocate device memory.
 * (The source pages have no counterpart: this is an interface convenience.)
 *
 * Some callers cannot call cudaMalloc or hand the library a scratch buffer:
 * runtimes whose device memory is owned by another allocator the library
 * cannot reach, code with a fixed memory budget decided before it runs, or
 * latency-critical loops where a fresh cudaMalloc would stall the device.
 * For them this variant of q4kv_decode_attention takes the same arguments
 * minus the workspace, and keeps its split partials in one file-scope device
 * array of Q4KV_STATIC_SCRATCH_BYTES (16 MiB) instead.  Every GPU that loads
 * the library holds that array until the process exits.
 *   - A plan whose workspace_bytes exceeds Q4KV_STATIC_SCRATCH_BYTES is
 *     rejected with Q4KV_ERR_WORKSPACE before anything runs; force fewer
 *     splits (q4kv_decode_plan_make n_splits) or use q4kv_decode_attention.
 *   - Every call looks up the array's device address for the device current
 *     at that moment (cudaGetSymbolAddress, which allocates nothing), so the
 *     address stays right after a device reset.  The first call on a device
 *     also loads the library's device code there; make that first call
 *     before any stream capture.
 *   - All calls share the array and it keeps the last call's contents; the
 *     kernels overwrite every partial they later read, so nothing needs to
 *     start at zero.  Calls that overlap on the GPU (other streams, other
 *     host threads) race on the array and must be serialised by the caller.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * Results equal those of q4kv_decode_attention with the same plan.
 */
#define Q4KV_STATIC_SCRATCH_BYTES (16u << 20)
q4kv_status q4kv_decode_attention_static_scratch(const q4kv_pool *pool,
                                                 const q4kv_decode_plan *plan, const void *q,
                                                 int32_t q_dtype, const int32_t *block_tables,
                                                 const int32_t *seq_lens, float softmax_scale,
                                                 void *out, int32_t out_dtype, void *stream);

/*
 * Diagnostic (no counterpart on the pages): launch one CTA that waits on a
 * shared-memory barrier nothing ever completes, with the bounded wait every
 * kernel of this library uses, limited to `tries` rounds (1 <= tries <=
 * 2^21; each round sleeps up to ~1 us).  When the limit runs out the kernel
 * ORs Q4KV_DEVERR_TIMEOUT into *error_word (device uint32) and returns, so the
 * context stays usable; tests use it to check that waits end.
 */
q4kv_status q4kv_selftest_bounded_wait(uint32_t *error_word, int32_t tries, void *stream);

/*
 * Per-token widths {2, 4, 8, FP16} in one cache: the card ([QKVS]
 * "Méthodologie": each token gets a width from {2, 4, 8, FP16}; the cache
 * travels as a compact artifact of quantised groups, per-token widths and
 * metadata; the receiver rebuilds FP16 keys and values from it).
 *
 * Card layout (device memory, 16-byte aligned, little-endian):
 *   header 64 B: uint32 magic 0x43564B51 ("QKVC"), uint32 version 1,
 *     uint32 head_dim, uint32 n_kv_heads, uint64 n_tokens, uint32 k_rotated,
 *     uint32 raw dtype of FP16 tokens (0 fp16, 1 bf16), int64 payload bytes,
 *     zeros to 64
 *   widths: one byte per token, padded to a multiple of 16
 *   offsets: int64 [n_tokens + 1], byte offset of each token's record from
 *     the payload start, then the payload size; padded to 16
 *   payload: token records in order.  The record of token t is, for every KV
 *     head in order: K codes (D*w/8 bytes), V codes, K (s, z) half2 pairs
 *     (D/64), V pairs -- the pool's group coding with L = 2^w - 1 (w = 2: four
 *     codes per byte, element 4i+m at bits 2m of byte i; w = 4: the nibble
 *     order; w = 8: one per byte), K rotated when k_rotated -- or, for
 *     w = 16, the raw K row then the raw V row (2*D bytes each, the input's
 *     own 16-bit values).  Per (token, head): 80 / 144 / 272 / 512 bytes at
 *     D = 128 for w = 2 / 4 / 8 / 16.
 *
 * q4kv_card_max_bytes: the card size when every token is FP16 (host-only);
 * a card of that size always fits.
 */
q4kv_status q4kv_card_max_bytes(int32_t head_dim, int32_t n_kv_heads, int64_t n_tokens, size_t *bytes);

/*
 * Encode n_tokens tokens into a card.
 *   k, v        as in q4kv_quantize_blocks (fp16 or bf16, token stride rules)
 *   widths      device uint8 [n_tokens], each 2, 4, 8 or 16; any other value
 *               gives the token no record and raises Q4KV_DEVERR_WIDTH
 *   card        device, 16-byte aligned, card_bytes >= q4kv_card_max_bytes
 *   k_rotated   1 = code keys after the Walsh-Hadamard rotation (as the pool
 *               does); FP16 tokens are always stored raw
 * Codes, scales and zeros are bit-identical to the pool's coding of the same
 * row at that width.  The payload size is written into the header.
 */
q4kv_status q4kv_card_encode(int32_t head_dim, int32_t n_kv_heads, int32_t k_rotated, const void *k,
                             const void *v, int32_t in_dtype, int64_t n_tokens, int64_t token_stride,
                             const uint8_t *widths, void *card, size_t card_bytes, uint32_t *error_word,
                             void *stream);

/*
 * Rebuild K and V from a card (the receiver's injection path of [QKVS]).
 *   k_out, v_out  device [n_tokens][Hkv][D] of out_dtype (Q4KV_F32 or
 *                 Q4KV_F16), 16-byte aligned.  x_hat = fl(code*s + z); keys
 *                 coded rotated are un-rotated (c*H, bit-exact); FP16 tokens
 *                 are their raw values; a token with an invalid width reads 0.
 * The header must hold (head_dim, n_kv_heads, n_tokens) and every record must
 * lie inside card_bytes; otherwise the affected rows read 0 and
 * Q4KV_DEVERR_IMAGE is raised (a damaged card is never read out of bounds).
 */
q4kv_status q4kv_card_decode(const void *card, size_t card_bytes, int32_t head_dim, int32_t n_kv_heads,
                             int64_t n_tokens, void *k_out, void *v_out, int32_t out_dtype,
                             uint32_t *error_word, void *stream);

/*
 * Block images: paging blocks between device and host memory ([AMBP] sec.
 * 2.1 item 1: the pool pages 256-token blocks between fast memory and
 * storage; item 3: one agent's cache is brought in while another agent
 * decodes; sec. 5: storage as the cache's swap space).  The storage tier
 * itself (files, safetensors) is the caller's.
 *
 * An image is one block in one contiguous run of bytes, every section a
 * multiple of 16 bytes:
 *   header  16 B: uint32 magic 0x424B3451 ("Q4KB"), uint16 class (4 = 4-bit,
 *           8 = 8-bit, 0x108 = FP8), uint16 head_dim, uint32 n_kv_heads,
 *           int32 the block id it was exported from (informational)
 *   K codes [Hkv][256][row] bytes, row = D/2 (4-bit) or D (8-bit, FP8)
 *   V codes the same
 *   K params [Hkv][256][D/64] half2, then V params (absent for FP8 pools)
 *   remap mask 8 uint32
 * i.e. the block's bytes exactly as the pool holds them.  Images of one call
 * sit at a fixed stride, the size of the pool's largest block class; a
 * smaller class leaves the rest of its stride unused.
 */
q4kv_status q4kv_block_image_stride(const q4kv_pool *pool, size_t *stride_bytes);

/*
 * Write the images of blocks block_ids[0 .. n_blocks) to host memory.
 *   block_ids    device int32 [n_blocks]
 *   host_images  page-locked host memory the device can address
 *                (cudaHostAlloc, or cudaHostRegister'ed), 16-byte aligned,
 *                at least n_blocks * stride bytes; image i at i * stride.
 * One kernel reads the pool and stores straight into host memory over the
 * bus, so the call can run on a stream of its own beside other work.  The
 * images are complete once `stream` has reached this point.  An
 * out-of-range id leaves its image unwritten and raises
 * Q4KV_DEVERR_BLOCK_ID.  n_blocks == 0 is a no-op.  Pageable host memory is
 * refused with Q4KV_ERR_INVALID_ARG.
 */
q4kv_status q4kv_export_blocks(const q4kv_pool *pool, const int32_t *block_ids, int32_t n_blocks,
                               void *host_images, void *stream);

/*
 * Load images from host memory into blocks block_ids[0 .. n_blocks): image i
 * replaces block block_ids[i] entirely (codes, params, remap mask).  Each
 * image's header must fit its target block (magic, class, head_dim, Hkv);
 * one that does not leaves the block unchanged and raises Q4KV_DEVERR_IMAGE.
 * Same memory rules as q4kv_export_blocks; the host bytes must stay
 * unchanged until `stream` has passed the call.  Target ids must be distinct,
 * and no other work may read or write those blocks while the copy runs
 * (decode of other blocks may run concurrently on another stream).
 */
q4kv_status q4kv_import_blocks(const q4kv_pool *pool, const void *host_images, const int32_t *block_ids,
                               int32_t n_blocks, void *stream);

/*
 * The same two moves with the block ids in HOST memory, done by the copy
 * engines: no kernel runs and no SM is used, so a block can page in while
 * decode keeps every SM (the way [AMBP] sec. 2.1 item 3 hides loading).
 *   block_ids    host int32 [n_blocks], each in range (else
 *                Q4KV_ERR_INVALID_ARG before anything is enqueued)
 *   host_images  as above (page-locked, 16-byte aligned, image i at i*stride)
 * Export writes every image's header from the host at call time and
 * enqueues the section copies; import reads and checks every header at call
 * time (so the images must already be complete then) and returns
 * Q4KV_ERR_INVALID_ARG, enqueuing nothing, if one does not fit its target
 * block.  Each run of consecutive ids of one block class, at consecutive
 * images, moves as one strided 2-D copy per section.  The results equal those
 * of q4kv_export_blocks / q4kv_import_blocks.
 */
q4kv_status q4kv_export_blocks_host_ids(const q4kv_pool *pool, const int32_t *block_ids, int32_t n_blocks,
                                        void *host_images, void *stream);
q4kv_status q4kv_import_blocks_host_ids(const q4kv_pool *pool, const void *host_images,
                                        const int32_t *block_ids, int32_t n_blocks, void *stream);

/*
 * Wait for `stream`, read pool->error_word into *bits, and zero it when
 * `clear` is nonzero.  Returns Q4KV_ERR_DEVICE when any bit was set,
 * Q4KV_OK otherwise (and *bits = 0 when pool->error_word is NULL).
 */
q4kv_status q4kv_read_device_error(const q4kv_pool *pool, uint32_t *bits, int32_t clear,
                                   void *stream);

#ifdef __cplusplus
}
#endif

#endif /* Q4KV_H */
