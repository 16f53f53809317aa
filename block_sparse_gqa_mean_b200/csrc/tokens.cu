// Token-granular sparse attention for one new query per sequence (decode).
//
// "Sparse Attention + Linear Backbones: How LLM Long-Context Architectures Are
// Evolving", sections 5.1-5.3 and 5.5: a lightweight multi-head indexer
// without positional encoding rates all earlier positions, the top-K
// positions are kept, and the main attention runs over those positions only.
// The indexer's form is not given; it is read here the way the block score is
// defined: s(t, u) = sum over indexer heads h of qI[h] . kI[u], exp-free,
// computed as qbar = qI[0] + qI[1] + ... (fp32, left to right) and one fp32
// fma chain over the coordinates in order; the own position t is always kept,
// plus the top K-1 earlier positions, ties to the lower position.
//
//   tok_score_kernel   one score per earlier position (indexer keys are paged
//                      with the KV cache's page table, one row per position)
//   tok_select_kernel  one CTA per sequence: radix select of the (K-1)-th
//                      largest score on order-preserving 32-bit keys (four
//                      8-bit passes), then an ordered compaction that keeps
//                      every larger key and the lowest positions among the
//                      equal ones, so the list comes out ascending
//   tok_attn_kernel    one CTA per (sequence, KV group): the kept tokens' K and
//                      V rows gathered 32 at a time through shared memory, an
//                      fp32 online softmax per query head (expf)
#include "common.cuh"

namespace msa {

namespace {

constexpr int kScoreChunk = 1024;  // positions per score CTA (256 threads x 4)
constexpr int kSelThreads = 1024;
constexpr int kTokChunk = 32;      // tokens gathered per attention step

__device__ __forceinline__ unsigned order_key(float f) {
  const unsigned b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// exclusive scan of one value per thread over a 1024-thread block
__device__ __forceinline__ unsigned block_scan_1024(unsigned v, unsigned* warp_tot,
                                                    unsigned* total) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  unsigned incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const unsigned wv = warp_tot[lane];
    unsigned wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned x = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += x;
    }
    warp_tot[lane] = wi - wv;  // exclusive prefix of the warp totals
    if (lane == 31) warp_tot[32] = wi;
  }
  __syncthreads();
  const unsigned r = warp_tot[warp] + incl - v;
  *total = warp_tot[32];
  __syncthreads();
  return r;
}

}  // namespace

template <typename T, int D>
__global__ void __launch_bounds__(256) tok_score_kernel(
    const T* __restrict__ qi, const T* __restrict__ ki_pages, const int32_t* __restrict__ page_table,
    const int32_t* __restrict__ seq_lens, uint32_t* status, int hi, int B, int num_pages,
    int max_blocks, int max_len, float* __restrict__ scores) {
  __shared__ float qbar[D];
  const int b = blockIdx.y;
  const int L = seq_lens[b];
  if (L < 1 || L > max_blocks * B) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(status, MSA_DEV_BAD_LENGTH);
    return;
  }
  const int t = L - 1;  // the query's position: positions 0 .. t-1 are scored
  const int u0 = blockIdx.x * kScoreChunk;
  if (u0 >= t) return;
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    const T* p = qi + (size_t)b * hi * D + i;
    float s = to_f32(p[0]);
    for (int h = 1; h < hi; ++h) s += to_f32(p[(size_t)h * D]);
    qbar[i] = s;
  }
  __syncthreads();
  for (int m = 0; m < kScoreChunk / 256; ++m) {
    const int u = u0 + m * 256 + threadIdx.x;
    if (u >= t) break;
    const int pg = page_table[(size_t)b * max_blocks + u / B];
    float acc = -INFINITY;
    if (pg >= 0 && pg < num_pages) {
      const T* kr = ki_pages + ((size_t)pg * B + u % B) * D;
      acc = 0.f;
#pragma unroll 4
      for (int i = 0; i < D; ++i) acc = fmaf(qbar[i], to_f32(kr[i]), acc);
    } else {
      report(status, MSA_DEV_BAD_PAGE);
    }
    scores[(size_t)b * max_len + u] = acc;
  }
}

__global__ void __launch_bounds__(kSelThreads) tok_select_kernel(
    const float* __restrict__ scores, const int32_t* __restrict__ seq_lens, int max_blocks, int B,
    int max_len, int top_k, int32_t* __restrict__ tok_idx) {
  __shared__ unsigned hist[256];
  __shared__ unsigned warp_tot[33];
  __shared__ unsigned s_prefix, s_remaining;
  const int b = blockIdx.x, tid = threadIdx.x;
  const int L = seq_lens[b];
  int32_t* out = tok_idx + (size_t)b * top_k;
  if (L < 1 || L > max_blocks * B) {  // reported by the score kernel
    for (int i = tid; i < top_k; i += kSelThreads) out[i] = -1;
    return;
  }
  const int t = L - 1, n = t;  // candidates: the earlier positions 0 .. t-1
  const int keep = min(top_k - 1, n);
  if (keep == n) {
    for (int i = tid; i < top_k; i += kSelThreads) out[i] = i < n ? i : (i == n ? t : -1);
    return;
  }
  const float* sc = scores + (size_t)b * max_len;
  // radix select: the key of the keep-th largest score, and how many keys equal
  // to it are kept (the lowest positions among them)
  unsigned prefix = 0u, pmask = 0u, remaining = (unsigned)keep;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0u;
    __syncthreads();
    for (int u = tid; u < n; u += kSelThreads) {
      const unsigned k = order_key(sc[u]);
      if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      unsigned cum = 0u;
      int d = 255;
      for (; d > 0; --d) {
        if (cum + hist[d] >= remaining) break;
        cum += hist[d];
      }
      s_prefix = prefix | ((unsigned)d << shift);
      s_remaining = remaining - cum;
    }
    __syncthreads();
    prefix = s_prefix;
    remaining = s_remaining;
    pmask |= 255u << shift;
    __syncthreads();
  }
  const unsigned T_key = prefix;
  // ordered compaction over contiguous segments of positions
  const int per = (n + kSelThreads - 1) / kSelThreads;
  const int a0 = min(n, tid * per), a1 = min(n, a0 + per);
  unsigned eq = 0u;
  for (int u = a0; u < a1; ++u) eq += order_key(sc[u]) == T_key;
  unsigned tot;
  unsigned eq_before = block_scan_1024(eq, warp_tot, &tot);
  unsigned cnt = 0u;
  {
    unsigned e2 = eq_before;
    for (int u = a0; u < a1; ++u) {
      const unsigned k = order_key(sc[u]);
      const bool s = k > T_key || (k == T_key && e2 < remaining);
      e2 += k == T_key;
      cnt += s;
    }
  }
  unsigned pos = block_scan_1024(cnt, warp_tot, &tot);
  {
    unsigned e2 = eq_before;
    for (int u = a0; u < a1; ++u) {
      const unsigned k = order_key(sc[u]);
      const bool s = k > T_key || (k == T_key && e2 < remaining);
      e2 += k == T_key;
      if (s && pos < (unsigned)keep) out[pos++] = u;
    }
  }
  for (int i = keep + tid; i < top_k; i += kSelThreads) out[i] = (i == keep) ? t : -1;
}

template <typename T, int D>
__global__ void __launch_bounds__(128) tok_attn_kernel(
    const T* __restrict__ q, const T* __restrict__ k_pages, const T* __restrict__ v_pages,
    const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens, uint32_t* status,
    const int32_t* __restrict__ tok_idx, int top_k, int hq, int hkv, int B, int num_pages,
    int max_blocks, float scale, T* __restrict__ out, float* __restrict__ lse) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int G = hq / hkv;
  float* qs = reinterpret_cast<float*>(smem_raw);  // [G][D]
  float* os = qs + G * D;                          // [G][D]
  float* ks = os + G * D;                          // [kTokChunk][D+1]
  float* vs = ks + kTokChunk * (D + 1);            // [kTokChunk][D]
  float* ps = vs + kTokChunk * D;                  // [G][kTokChunk]
  __shared__ float m_s[16], l_s[16], a_s[16];
  __shared__ int s_row[kTokChunk];                 // K/V row offset of each gathered token, -1: none

  const int g = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x;
  const int L = seq_lens[b];
  if (L < 1 || L > max_blocks * B) {
    if (tid == 0) report(status, MSA_DEV_BAD_LENGTH);
    return;
  }
  const int t = L - 1;
  for (int e = tid; e < G * D; e += blockDim.x) {
    qs[e] = to_f32(q[((size_t)b * hq + g * G) * D + e]);
    os[e] = 0.f;
  }
  if (tid < G) {
    m_s[tid] = -INFINITY;
    l_s[tid] = 0.f;
  }
  const int32_t* list = tok_idx + (size_t)b * top_k;
  for (int c0 = 0; c0 < top_k; c0 += kTokChunk) {
    __syncthreads();  // the previous chunk fully consumed
    if (tid < kTokChunk) {
      const int s = c0 + tid;
      int row = -1;
      if (s < top_k) {
        const int u = list[s];
        // a position past the query, or repeated in the adjacent slot, is skipped
        if (u >= 0 && u <= t && !(s > 0 && list[s - 1] == u)) {
          const int pg = page_table[(size_t)b * max_blocks + u / B];
          if (pg >= 0 && pg < num_pages) row = ((pg * hkv + g) * B + u % B);
          else report(status, MSA_DEV_BAD_PAGE);
        } else if (u > t) {
          report(status, MSA_DEV_BAD_INDEX);
        }
      }
      s_row[tid] = row;
    }
    __syncthreads();
    for (int e = tid; e < kTokChunk * D; e += blockDim.x) {
      const int kk = e / D, i = e % D;
      const int row = s_row[kk];
      ks[kk * (D + 1) + i] = row >= 0 ? to_f32(k_pages[(size_t)row * D + i]) : 0.f;
      vs[e] = row >= 0 ? to_f32(v_pages[(size_t)row * D + i]) : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < G * kTokChunk; e += blockDim.x) {
      const int h = e / kTokChunk, kk = e % kTokChunk;
      float acc = -INFINITY;
      if (s_row[kk] >= 0) {
        const float* qh = qs + h * D;
        const float* kr = ks + kk * (D + 1);
        acc = 0.f;
        for (int i = 0; i < D; ++i) acc = fmaf(qh[i], kr[i], acc);
        acc *= scale;
      }
      ps[h * kTokChunk + kk] = acc;
    }
    __syncthreads();
    // per-head online-softmax update, one warp per head
    for (int h = tid / 32; h < G; h += blockDim.x / 32) {
      const int lane = tid % 32;
      const float x = ps[h * kTokChunk + lane];
      float mx = x;
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m_s[h], mx);
      const float p = (m_new == -INFINITY) ? 0.f : expf(x - m_new);  // no token yet: weight 0
      ps[h * kTokChunk + lane] = p;
      float sum = p;
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        const float alpha = (m_s[h] == -INFINITY) ? 0.f : expf(m_s[h] - m_new);
        a_s[h] = alpha;
        l_s[h] = l_s[h] * alpha + sum;
        m_s[h] = m_new;
      }
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += blockDim.x) {
      const int h = e / D, i = e % D;
      const float* ph = ps + h * kTokChunk;
      float acc = os[e] * a_s[h];
      for (int kk = 0; kk < kTokChunk; ++kk) acc = fmaf(ph[kk], vs[kk * D + i], acc);
      os[e] = acc;
    }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += blockDim.x) {
    const int h = e / D;
    out[((size_t)b * hq + g * G) * D + e] = from_f32<T>(l_s[h] > 0.f ? os[e] / l_s[h] : 0.f);
  }
  if (lse && tid < G)
    lse[(size_t)b * hq + g * G + tid] = l_s[tid] > 0.f ? m_s[tid] + logf(l_s[tid]) : -INFINITY;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t tokens_ws(const msa_paged_kv_t* kv) {
  return (size_t)kv->batch * kv->max_blocks_per_seq * kv->block_size * sizeof(float);
}

template <typename T, int D>
static cudaError_t launch_tok_select(const msa_paged_kv_t* kv, const void* ki_pages, const void* qi,
                                     int hi, int top_k, int32_t* tok_idx, void* ws,
                                     cudaStream_t st) {
  const int max_len = kv->max_blocks_per_seq * kv->block_size;
  float* scores = (float*)ws;
  dim3 grid((max_len + kScoreChunk - 1) / kScoreChunk, kv->batch);
  tok_score_kernel<T, D><<<grid, 256, 0, st>>>((const T*)qi, (const T*)ki_pages, kv->page_table,
                                               kv->seq_lens, kv->status_word, hi, kv->block_size,
                                               kv->num_pages, kv->max_blocks_per_seq, max_len,
                                               scores);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  tok_select_kernel<<<kv->batch, kSelThreads, 0, st>>>(scores, kv->seq_lens,
                                                       kv->max_blocks_per_seq, kv->block_size,
                                                       max_len, top_k, tok_idx);
  return cudaGetLastError();
}

cudaError_t select_tokens(const msa_paged_kv_t* kv, const void* ki_pages, const void* qi, int hi,
                          int top_k, int32_t* tok_idx, void* ws, cudaStream_t st) {
  const bool bf = kv->dtype == MSA_DTYPE_BF16;
  if (kv->head_dim == 128)
    return bf ? launch_tok_select<bf16, 128>(kv, ki_pages, qi, hi, top_k, tok_idx, ws, st)
              : launch_tok_select<float, 128>(kv, ki_pages, qi, hi, top_k, tok_idx, ws, st);
  return bf ? launch_tok_select<bf16, 64>(kv, ki_pages, qi, hi, top_k, tok_idx, ws, st)
            : launch_tok_select<float, 64>(kv, ki_pages, qi, hi, top_k, tok_idx, ws, st);
}

template <typename T, int D>
static cudaError_t launch_tok_attn(const msa_paged_kv_t* kv, const void* q, const int32_t* tok_idx,
                                   int top_k, float scale, void* out, float* lse, cudaStream_t st) {
  const int G = kv->num_q_heads / kv->num_kv_heads;
  const size_t smem = ((size_t)2 * G * D + (size_t)kTokChunk * (D + 1) + (size_t)kTokChunk * D +
                       (size_t)G * kTokChunk) * 4;
  auto kern = tok_attn_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(kv->num_kv_heads, kv->batch);
  kern<<<grid, 128, smem, st>>>((const T*)q, (const T*)kv->k_pages, (const T*)kv->v_pages,
                                 kv->page_table, kv->seq_lens, kv->status_word, tok_idx, top_k,
                                 kv->num_q_heads, kv->num_kv_heads, kv->block_size, kv->num_pages,
                                 kv->max_blocks_per_seq, scale, (T*)out, lse);
  return cudaGetLastError();
}

cudaError_t attn_tokens(const msa_paged_kv_t* kv, const void* q, const int32_t* tok_idx, int top_k,
                        float scale, void* out, float* lse, cudaStream_t st) {
  const bool bf = kv->dtype == MSA_DTYPE_BF16;
  if (kv->head_dim == 128)
    return bf ? launch_tok_attn<bf16, 128>(kv, q, tok_idx, top_k, scale, out, lse, st)
              : launch_tok_attn<float, 128>(kv, q, tok_idx, top_k, scale, out, lse, st);
  return bf ? launch_tok_attn<bf16, 64>(kv, q, tok_idx, top_k, scale, out, lse, st)
            : launch_tok_attn<float, 64>(kv, q, tok_idx, top_k, scale, out, lse, st);
}

}  // namespace msa
