// Split-K paged GQA decode attention over the packed 4/8-bit cache.
//
// "Agent Memory Below the Prompt" (arXiv 2603.04428 summary), sec. 2.1
// item 2: attention reads the quantised cache directly ("direct restore");
// item 3: one batched pass over many agents' caches; sec. 2.2: GQA.
// IntentKV article (Qiita), "詰め直さずに「無効化」する": remapped slots
// get logit -1e4 and contribute no value.
//
// Grid: (split, KV head, sequence).  A CTA owns the g query heads that share
// one KV head and one token range of one sequence; it keeps a running max and
// sum per head (online softmax) and writes either the final row (one split)
// or a partial (o, max, sum) merged afterwards by log-sum-exp.
#include <math.h>

#include "q4kv_internal.cuh"

namespace q4kv {
namespace {

constexpr int kThreads = 128;
constexpr int kTile = 128;   // tokens per iteration: one token per thread in the key pass
constexpr int kMaxG = 8;

__device__ __forceinline__ float load_in(const void* p, int dtype, int64_t i) {
  return dtype == Q4KV_F16 ? __half2float(static_cast<const __half*>(p)[i])
                           : __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}

__device__ __forceinline__ void store_out(void* p, int dtype, int64_t i, float x) {
  if (dtype == Q4KV_F32) static_cast<float*>(p)[i] = x;
  else if (dtype == Q4KV_F16) static_cast<__half*>(p)[i] = __float2half_rn(x);
  else static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
}

template <int D>
__global__ void __launch_bounds__(kThreads) decode_simple_kernel(const DecodeArgs a) {
  constexpr int NG = D / kGroup;
  constexpr int CP = D / 2;              // channel pairs, one per thread in the value pass
  constexpr int NPH = kThreads / CP;     // token phases in the value pass (2 or 1)
  __shared__ float qs[kMaxG][D];
  __shared__ float lg[kMaxG][kTile];     // logits, then value weights
  __shared__ int32_t tok_blk[kTile];     // unified block id of a live token, -1 otherwise
  __shared__ int32_t tok_slot[kTile];
  __shared__ float m_run[kMaxG], l_run[kMaxG], alpha[kMaxG];
  __shared__ float ored[kMaxG][D];
  __shared__ int poison;

  const PoolView& P = a.pool;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int hq = a.plan.n_q_heads, g = hq / P.n_kv_heads;
  const int S = a.plan.n_splits, tps = a.plan.tokens_per_split, mb = a.plan.max_blocks_per_seq;
  const int seq = seq_len_of(a, b);
  const bool bad_seq = seq < 0 || seq > mb * kBlockTokens;
  if (bad_seq && split == 0 && kvh == 0 && tid == 0) raise_error(P.error_word, Q4KV_DEVERR_SEQ_LEN);

  for (int i = tid; i < g * D; i += kThreads) {
    const int h = i / D, j = i % D;
    qs[h][j] = load_in(a.q, a.q_dtype, (static_cast<int64_t>(b) * hq + kvh * g + h) * D + j);
  }
  if (tid < kMaxG) {
    m_run[tid] = -INFINITY;
    l_run[tid] = 0.0f;
  }
  if (tid == 0) poison = bad_seq ? 1 : 0;
  __syncthreads();
  if (P.k_rotated) {   // q_rot = c * H q, any summation order (fp32)
    for (int hs = 1; hs < D; hs <<= 1) {
      for (int i = tid; i < g * (D / 2); i += kThreads) {
        const int h = i / (D / 2), p = i % (D / 2);
        const int lo = (p / hs) * 2 * hs + (p % hs), hi = lo + hs;
        const float x = qs[h][lo], y = qs[h][hi];
        qs[h][lo] = x + y;
        qs[h][hi] = x - y;
      }
      __syncthreads();
    }
    const float c = rotation_constant(D);
    for (int i = tid; i < g * D; i += kThreads) qs[i / D][i % D] *= c;
    __syncthreads();
  }

  const int t_begin = split * tps;
  const int t_end = bad_seq ? t_begin : min(t_begin + tps, seq);
  const int cp = tid % CP, ph = tid / CP;
  float o0[kMaxG], o1[kMaxG];
#pragma unroll
  for (int h = 0; h < kMaxG; ++h) o0[h] = o1[h] = 0.0f;

  for (int tile0 = t_begin; tile0 < t_end; tile0 += kTile) {
    // ---- key pass: one token per thread ----
    const int t = tile0 + tid;
    bool present = t < t_end;
    int32_t blk = -1;
    int slot = t % kBlockTokens;
    if (present) {
      blk = a.tables[static_cast<int64_t>(b) * mb + t / kBlockTokens];
      if (blk < 0 || blk >= P.n_q4 + P.n_q8) {
        raise_error(P.error_word, Q4KV_DEVERR_BLOCK_ID);
        poison = 1;
        present = false;
      }
    }
    bool masked = false;
    if (present)
      masked = (P.mask[static_cast<int64_t>(blk) * kMaskWords + slot / 32] >> (slot % 32)) & 1u;
    if (present && !masked) {
      float acc[kMaxG];
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) acc[h] = 0.0f;
      const bool is8 = blk >= P.n_q4;
      const int64_t phys = is8 ? blk - P.n_q4 : blk;
      const int64_t row = (phys * P.n_kv_heads + kvh) * kBlockTokens + slot;
      const __half2* par = (is8 ? P.k_params8 : P.k_params4) + row * NG;
#pragma unroll 1
      for (int gr = 0; gr < NG; ++gr) {
        const float s = __low2float(par[gr]), z = __high2float(par[gr]);
#pragma unroll 2
        for (int j8 = 0; j8 < kGroup; j8 += 8) {
          const int j0 = gr * kGroup + j8;
          uint32_t w0, w1 = 0;
          if (is8) {
            const uint2 u = *reinterpret_cast<const uint2*>(P.k_codes8 + row * D + j0);
            w0 = u.x;
            w1 = u.y;
          } else {
            w0 = *reinterpret_cast<const uint32_t*>(P.k_codes4 + row * (D / 2) + j0 / 2);
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t c = is8 ? ((e < 4 ? w0 : w1) >> (8 * (e % 4))) & 255u : (w0 >> (4 * e)) & 15u;
            const float kv = __fmaf_rn(static_cast<float>(c), s, z);
#pragma unroll
            for (int h = 0; h < kMaxG; ++h)
              if (h < g) acc[h] = fmaf(qs[h][j0 + e], kv, acc[h]);
          }
        }
      }
#pragma unroll
      for (int h = 0; h < kMaxG; ++h)
        if (h < g) lg[h][tid] = acc[h] * a.scale;
    } else {
#pragma unroll
      for (int h = 0; h < kMaxG; ++h)
        if (h < g) lg[h][tid] = present ? Q4KV_SENTINEL_LOGIT : -INFINITY;
    }
    tok_blk[tid] = (present && !masked) ? blk : -1;
    tok_slot[tid] = slot;
    __syncthreads();

    // ---- online softmax: warp w updates heads w, w+4 ----
    {
      const int warp = tid >> 5, lane = tid & 31;
      for (int h = warp; h < g; h += kThreads / 32) {
        float v[kTile / 32];
        float mx = -INFINITY;
#pragma unroll
        for (int q = 0; q < kTile / 32; ++q) {
          v[q] = lg[h][lane + 32 * q];
          mx = fmaxf(mx, v[q]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_old = m_run[h];
        const float m_new = fmaxf(m_old, mx);
        float al = 1.0f, sum = 0.0f;
        if (m_new != -INFINITY) {
          al = m_old == -INFINITY ? 0.0f : expf(m_old - m_new);
#pragma unroll
          for (int q = 0; q < kTile / 32; ++q) {
            v[q] = v[q] == -INFINITY ? 0.0f : expf(v[q] - m_new);
            sum += v[q];
          }
        } else {
#pragma unroll
          for (int q = 0; q < kTile / 32; ++q) v[q] = 0.0f;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
#pragma unroll
        for (int q = 0; q < kTile / 32; ++q)
          lg[h][lane + 32 * q] = tok_blk[lane + 32 * q] >= 0 ? v[q] : 0.0f;
        if (lane == 0) {
          l_run[h] = l_run[h] * al + sum;
          m_run[h] = m_new;
          alpha[h] = al;
        }
      }
    }
    __syncthreads();

    // ---- value pass: one channel pair per thread ----
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
      if (h < g) {
        o0[h] *= alpha[h];
        o1[h] *= alpha[h];
      }
    }
    const int n_in_tile = min(kTile, t_end - tile0);
    for (int tt = ph; tt < n_in_tile; tt += NPH) {
      const int32_t vb = tok_blk[tt];
      if (vb < 0) continue;
      const bool is8 = vb >= P.n_q4;
      const int64_t phys = is8 ? vb - P.n_q4 : vb;
      const int64_t row = (phys * P.n_kv_heads + kvh) * kBlockTokens + tok_slot[tt];
      const __half2 pr = (is8 ? P.v_params8 : P.v_params4)[row * NG + (2 * cp) / kGroup];
      const float s = __low2float(pr), z = __high2float(pr);
      uint32_t c0, c1;
      if (is8) {
        const uint32_t two = *reinterpret_cast<const uint16_t*>(P.v_codes8 + row * D + 2 * cp);
        c0 = two & 255u;
        c1 = two >> 8;
      } else {
        const uint32_t byte = P.v_codes4[row * (D / 2) + cp];
        c0 = byte & 15u;
        c1 = byte >> 4;
      }
      const float v0 = __fmaf_rn(static_cast<float>(c0), s, z);
      const float v1 = __fmaf_rn(static_cast<float>(c1), s, z);
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) {
        if (h < g) {
          const float w = lg[h][tt];
          o0[h] = fmaf(w, v0, o0[h]);
          o1[h] = fmaf(w, v1, o1[h]);
        }
      }
    }
    __syncthreads();
  }

  // combine the token phases
  if (NPH > 1) {
    if (ph == 1) {
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) {
        if (h < g) {
          ored[h][2 * cp] = o0[h];
          ored[h][2 * cp + 1] = o1[h];
        }
      }
    }
    __syncthreads();
    if (ph == 0) {
#pragma unroll
      for (int h = 0; h < kMaxG; ++h) {
        if (h < g) {
          o0[h] += ored[h][2 * cp];
          o1[h] += ored[h][2 * cp + 1];
        }
      }
    }
  }
  if (ph != 0) return;
  const bool poisoned = poison != 0;
  for (int h = 0; h < g; ++h) {
    const int64_t qrow = static_cast<int64_t>(b) * hq + kvh * g + h;
    if (S == 1) {
      const float l = l_run[h];
      const float inv = (!poisoned && l > 0.0f) ? 1.0f / l : 0.0f;
      store_out(a.out, a.out_dtype, qrow * D + 2 * cp, poisoned ? 0.0f : o0[h] * inv);
      store_out(a.out, a.out_dtype, qrow * D + 2 * cp + 1, poisoned ? 0.0f : o1[h] * inv);
    } else {
      float* po = a.ws_o + (qrow * S + split) * D;
      po[2 * cp] = o0[h];
      po[2 * cp + 1] = o1[h];
      if (cp == 0) {
        a.ws_ml[(qrow * S + split) * 2] = m_run[h];
        a.ws_ml[(qrow * S + split) * 2 + 1] = poisoned ? -1.0f : l_run[h];
      }
    }
  }
}

// Log-sum-exp merge of the splits of one (sequence, query head) row:
//   M = max m_i, L = sum l_i e^(m_i - M), out = sum o_i e^(m_i - M) / L.
// A poisoned split (l < 0) or an empty row (M = -inf) gives 0.
// Log-sum-exp merge of the S partials of one query row:
//   M = max m_i,  w_i = e^(m_i - M),  out = sum w_i o_i / sum w_i l_i.
// A poisoned split (l < 0) or a row with no token gives 0.  Thread i owns
// channels 4i .. 4i+3; the weights are computed once per split and shared
// through shared memory, so the channel loop is one float4 load and four
// FMAs per split.
template <int T>
__device__ __forceinline__ float block_reduce(float x, bool is_max, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, x, off);
    x = is_max ? fmaxf(x, y) : x + y;
  }
  if (T > 32) {
    __syncthreads();   // red may still be read by the previous reduction
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = x;
    __syncthreads();
    x = red[0];
#pragma unroll
    for (int w = 1; w < T / 32; ++w) x = is_max ? fmaxf(x, red[w]) : x + red[w];
  }
  return x;
}

constexpr int kFewSplits = 16;

template <int D>
__global__ void __launch_bounds__(D / 4) merge_kernel(const DecodeArgs a) {
  constexpr int T = D / 4;
  constexpr int kChunk = 256;   // splits whose weights are staged at a time
  __shared__ float wgt[kChunk];
  __shared__ float red[T / 32];
  griddep_wait();
  griddep_launch_dependents();
  const int64_t row = blockIdx.x;
  const int S = a.plan.n_splits;
  const float2* ml = reinterpret_cast<const float2*>(a.ws_ml) + row * S;
  if (S <= kFewSplits) {
    // few splits: every thread loads all (m, l) pairs and its partials in one
    // round of loads and merges them itself, without a block reduction
    const float4* op = reinterpret_cast<const float4*>(a.ws_o + row * S * D) + threadIdx.x;
    float2 st[kFewSplits];
    float4 ov[kFewSplits];
#pragma unroll
    for (int i = 0; i < kFewSplits; ++i)
      if (i < S) {
        st[i] = ml[i];
        ov[i] = op[static_cast<int64_t>(i) * T];
      }
    float M = -INFINITY;
    bool pois = false;
#pragma unroll
    for (int i = 0; i < kFewSplits; ++i)
      if (i < S) {
        M = fmaxf(M, st[i].x);
        pois |= st[i].y < 0.0f;
      }
    float L = 0.0f;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
    for (int i = 0; i < kFewSplits; ++i)
      if (i < S && M != -INFINITY && st[i].x != -INFINITY) {   // an empty split adds nothing
        const float w = expf(st[i].x - M);
        L = fmaf(st[i].y, w, L);
        acc.x = fmaf(ov[i].x, w, acc.x);
        acc.y = fmaf(ov[i].y, w, acc.y);
        acc.z = fmaf(ov[i].z, w, acc.z);
        acc.w = fmaf(ov[i].w, w, acc.w);
      }
    const bool ok = !pois && M != -INFINITY && L > 0.0f;
    const int64_t base = row * D + 4 * threadIdx.x;
    store_out(a.out, a.out_dtype, base, ok ? acc.x / L : 0.0f);
    store_out(a.out, a.out_dtype, base + 1, ok ? acc.y / L : 0.0f);
    store_out(a.out, a.out_dtype, base + 2, ok ? acc.z / L : 0.0f);
    store_out(a.out, a.out_dtype, base + 3, ok ? acc.w / L : 0.0f);
    return;
  }
  float M = -INFINITY, pois = 0.0f;
  for (int i = threadIdx.x; i < S; i += T) {
    const float2 v = ml[i];
    M = fmaxf(M, v.x);
    pois = fmaxf(pois, v.y < 0.0f ? 1.0f : 0.0f);
  }
  M = block_reduce<T>(M, true, red);
  pois = block_reduce<T>(pois, true, red);
  float L = 0.0f;
  float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  const float4* o = reinterpret_cast<const float4*>(a.ws_o + row * S * D) + threadIdx.x;
  for (int c0 = 0; c0 < S; c0 += kChunk) {
    const int n = min(kChunk, S - c0);
    __syncthreads();   // the previous chunk's weights are consumed
    for (int i = threadIdx.x; i < n; i += T) {
      const float2 v = ml[c0 + i];
      const float w = (M == -INFINITY || v.x == -INFINITY) ? 0.0f : expf(v.x - M);
      wgt[i] = w;
      L = fmaf(v.y, w, L);
    }
    __syncthreads();
#pragma unroll 4
    for (int i = 0; i < n; ++i) {
      const float w = wgt[i];
      if (w == 0.0f) continue;   // an empty split adds nothing
      const float4 x = o[static_cast<int64_t>(c0 + i) * T];
      acc.x = fmaf(x.x, w, acc.x);
      acc.y = fmaf(x.y, w, acc.y);
      acc.z = fmaf(x.z, w, acc.z);
      acc.w = fmaf(x.w, w, acc.w);
    }
  }
  L = block_reduce<T>(L, false, red);
  const bool ok = pois == 0.0f && M != -INFINITY && L > 0.0f;
  const int64_t base = row * D + 4 * threadIdx.x;
  store_out(a.out, a.out_dtype, base, ok ? acc.x / L : 0.0f);
  store_out(a.out, a.out_dtype, base + 1, ok ? acc.y / L : 0.0f);
  store_out(a.out, a.out_dtype, base + 2, ok ? acc.z / L : 0.0f);
  store_out(a.out, a.out_dtype, base + 3, ok ? acc.w / L : 0.0f);
}

}  // namespace

int device_sm_count() {
  static int cached[128] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return 0;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cached[dev] = n;
  }
  return cached[dev];
}

cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t stream) {
  const q4kv_decode_plan& p = a.plan;
  const unsigned rows = static_cast<unsigned>(p.batch) * p.n_q_heads;
  if (p.head_dim == 128) return launch_pdl(merge_kernel<128>, dim3(rows), dim3(32), 0, stream, a);
  return launch_pdl(merge_kernel<256>, dim3(rows), dim3(64), 0, stream, a);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const q4kv_decode_plan& p = a.plan;
  cudaError_t e;
  if (p.kernel == 1) {
    const int sms = device_sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    e = launch_decode_tc(a, sms, stream);
  } else {
    const dim3 grid(p.n_splits, p.n_kv_heads, p.batch);
    if (p.head_dim == 128)
      decode_simple_kernel<128><<<grid, kThreads, 0, stream>>>(a);
    else
      decode_simple_kernel<256><<<grid, kThreads, 0, stream>>>(a);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess || p.n_splits == 1) return e;
  return launch_merge(a, stream);
}

}  // namespace q4kv
