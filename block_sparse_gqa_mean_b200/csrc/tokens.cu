// Token-granular sparse attention for one new query per sequence (decode).
//
// "Sparse Attention + Linear Backbones: How LLM Long-Context Architectures Are
// Evolving", sections 5.1-5.3 and 5.5: a lightweight multi-head indexer
// without positional encoding rates all earlier positions, the top-K
// positions are kept, and the main attention runs over those positions only.
// The indexer's form is not given; it is read here the way the block score is
// defined: s(t, u) = sum over indexer heads h of qI[h] . kI[u], exp-free,
// computed as qbar = qI[0] + qI[1] + ... (fp32, left to right), an fp32 fma
// chain over each 16-byte chunk of the key and a butterfly sum of the chunks'
// partials; the own position t is always kept,
// plus the top K-1 earlier positions, ties to the lower position.
//
//   tok_score_kernel   one score per earlier position (indexer keys are paged
//                      with the KV cache's page table, one row per position),
//                      read as whole rows by half-warps
//   tok_select_kernel  one CTA per row: radix select of the (K-1)-th largest
//                      score on order-preserving 32-bit keys (four 8-bit
//                      passes), then an ordered compaction that keeps every
//                      larger key and the lowest positions among the equal
//                      ones, so the list comes out ascending. Long rows first
//                      narrow the keys to the candidates above a threshold
//                      read off a sorted regular sample and run both steps on
//                      those alone, in shared memory
//   tok_attn_tc_kernel one CTA per (sequence, KV group) for bf16, head_dim 128:
//                      the kept tokens' K and V rows gathered 64 at a time by
//                      16-byte cp.async copies into a three-stage ring of
//                      swizzled tiles, four warps on mma.sync (bf16 in, fp32
//                      accumulate) with an online softmax each, merged at the end
//   tok_attn_kernel    the same for fp32 or head_dim 64: 32 tokens at a time
//                      through shared memory, fp32 arithmetic (expf)
#include "mma_sync.cuh"

namespace msa {

namespace {

constexpr int kScoreChunk = 1024;  // positions per score CTA (256 threads x 4)
constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kTokChunk = 32;      // tokens gathered per attention step
constexpr int kCandCap = 16384;    // candidates of the sampled selection (keys + positions: 128 KB)

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

// Warp 0 of a radix-select pass: walking the 256 bins of `hist` from the top,
// the digit d at which the count reaches `remaining`, and the count of the
// bins above d (bin 0 when the bins never reach it). Lane l holds bins
// 255 - 8l down to 248 - 8l.
__device__ __forceinline__ void pick_digit(const unsigned* hist, unsigned remaining, unsigned* s_d,
                                           unsigned* s_cum) {
  const int lane = threadIdx.x & 31;
  unsigned v[8], sum = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[i] = hist[255 - 8 * lane - i];
    sum += v[i];
  }
  unsigned incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  const unsigned reach = __ballot_sync(0xffffffffu, incl >= remaining);
  const int at = reach ? __ffs(reach) - 1 : 31;
  if (lane == at) {
    unsigned cum = incl - sum;
    int d = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      d = 255 - 8 * lane - i;
      if (cum + v[i] >= remaining || d == 0) break;
      cum += v[i];
    }
    *s_d = (unsigned)d;
    *s_cum = cum;
  }
}

// Row r of a token-variant call: its sequence b and position t. Without cu_q
// there is one row per sequence, at seq_lens[r] - 1 (decode); with cu_q the
// rows cu_q[b] .. cu_q[b+1]-1 of sequence b sit at its last n_b positions
// (prefill, chunked prefill). false: the sequence's length is not valid.
__device__ __forceinline__ bool token_row(int r, const int32_t* __restrict__ cu_q, int batch,
                                          const int32_t* __restrict__ seq_lens, int max_blocks,
                                          int B, int& b, int& t) {
  if (!cu_q) {
    b = r;
    t = seq_lens[r] - 1;
    return t >= 0 && t < max_blocks * B;
  }
  int lo = 0, hi = batch;  // cu_q[lo] <= r < cu_q[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (cu_q[mid] <= r) lo = mid; else hi = mid;
  }
  b = lo;
  const int n_b = cu_q[lo + 1] - cu_q[lo];
  const int L = seq_lens[lo];
  t = L - n_b + (r - cu_q[lo]);
  // r past cu_q[batch] (more rows than the offsets describe) has no position
  return n_b <= L && L <= max_blocks * B && t >= 0 && r - cu_q[lo] < n_b;
}

}  // namespace

// Scores of the earlier positions. A warp takes 32 consecutive positions; in
// each step its lanes read two whole indexer-key rows (2 x D elements, one
// 16-byte chunk per lane, 512 contiguous bytes for d 128), lane l holding chunk
// l % (D / VEC) of row l / (D / VEC). Each lane keeps its chunk of qbar (the
// indexer heads summed left to right, fp32) in registers, computes an fp32 fma
// chain over its chunk, and the lanes of a row add their partial sums by a
// butterfly of shuffles.
template <typename T, int D>
__global__ void __launch_bounds__(256) tok_score_kernel(
    const T* __restrict__ qi, const T* __restrict__ ki_pages, const int32_t* __restrict__ page_table,
    const int32_t* __restrict__ seq_lens, const int32_t* __restrict__ cu_q, int batch,
    uint32_t* status, int hi, int B, int num_pages, int max_blocks, int max_len,
    float* __restrict__ scores) {
  constexpr int VEC = 16 / sizeof(T);       // elements per 16-byte chunk
  constexpr int CPR = D / VEC;              // chunks per row (16 for bf16 d 128)
  constexpr int RPI = 32 / CPR;             // rows per warp step
  static_assert(32 % CPR == 0, "a row's chunks stay inside one warp");
  __shared__ __align__(16) float qbar_s[D];
  const int r = blockIdx.y;  // the query row
  int b, t;                  // its sequence and position: positions 0 .. t-1 are scored
  if (!token_row(r, cu_q, batch, seq_lens, max_blocks, B, b, t)) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(status, MSA_DEV_BAD_LENGTH);
    return;
  }
  const int u_cta = blockIdx.x * kScoreChunk;
  if (u_cta >= t) return;
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    const T* p = qi + (size_t)r * hi * D + i;
    float s = to_f32(p[0]);
    for (int h = 1; h < hi; ++h) s = __fadd_rn(s, to_f32(p[(size_t)h * D]));
    qbar_s[i] = s;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = lane % CPR, sub = lane / CPR;
  float qc[VEC];
#pragma unroll
  for (int x = 0; x < VEC; ++x) qc[x] = qbar_s[c * VEC + x];
  // warp w takes positions [u_cta + 32 m + ...) for m = w, w + 8, ...
  for (int u0 = u_cta + 32 * warp; u0 < min(t, u_cta + kScoreChunk); u0 += 32 * 8) {
    float res = -INFINITY;                   // lane j < 32: the score of position u0 + j
#pragma unroll 4
    for (int step = 0; step < 32 / RPI; ++step) {
      const int u = u0 + step * RPI + sub;
      float part = 0.f;
      bool ok = false;
      if (u < t) {
        const int pg = page_table[(size_t)b * max_blocks + u / B];
        if (pg >= 0 && pg < num_pages) {
          ok = true;
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(
              ki_pages + ((size_t)pg * B + u % B) * D + c * VEC));
          const T* e = reinterpret_cast<const T*>(&v);
#pragma unroll
          for (int x = 0; x < VEC; ++x) part = __fmaf_rn(qc[x], to_f32(e[x]), part);
        } else if (c == 0) {
          report(status, MSA_DEV_BAD_PAGE);
        }
      }
#pragma unroll
      for (int o = CPR / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      // lane (step * RPI + r) keeps the score of row r of this step
      const float row_score = ok ? part : -INFINITY;
#pragma unroll
      for (int r = 0; r < RPI; ++r) {
        const float v = __shfl_sync(0xffffffffu, row_score, r * CPR);
        if (lane == step * RPI + r) res = v;
      }
    }
    if (u0 + lane < t && MSA_IN_BOUNDS(u0 + lane, max_len, status))
      scores[(size_t)r * max_len + u0 + lane] = res;
  }
}

__global__ void __launch_bounds__(kSelThreads) tok_select_kernel(
    const float* __restrict__ scores, const int32_t* __restrict__ seq_lens,
    const int32_t* __restrict__ cu_q, int batch, int max_blocks, int B, int max_len, int top_k,
    int32_t* __restrict__ tok_idx) {
  __shared__ unsigned hist[256];
  __shared__ unsigned whist[256 * kSelWarps];  // per-warp histograms
  __shared__ unsigned warp_tot[33];
  __shared__ unsigned s_prefix, s_remaining;
  const int r = blockIdx.x, tid = threadIdx.x;
  int32_t* out = tok_idx + (size_t)r * top_k;
  int b, t;
  if (!token_row(r, cu_q, batch, seq_lens, max_blocks, B, b, t)) {  // reported by the score kernel
    for (int i = tid; i < top_k; i += kSelThreads) out[i] = -1;
    return;
  }
  const int n = t;  // candidates: the earlier positions 0 .. t-1
  const int keep = min(top_k - 1, n);
  if (keep == n) {
    for (int i = tid; i < top_k; i += kSelThreads) out[i] = i < n ? i : (i == n ? t : -1);
    return;
  }
  const float* sc = scores + (size_t)r * max_len;

  // Sampled selection (long rows, keep <= kCandCap / 4). A regular sample of
  // kSelThreads scores, sorted, gives a key tau that about (rk / kSelThreads)
  // of all keys reach, rk set to 1.5 x the sample rank of the keep-th largest
  // plus 16; every key >= tau is a candidate. When the candidates number at
  // least keep (so the keep largest are among them) and fit in shared memory,
  // the selection below runs on them alone, in position order; otherwise the
  // full radix select further down runs. Either way the result is the exact
  // rule: the keep largest keys, ties to the lower position.
  if (keep <= kCandCap / 4 && n >= 8 * kSelThreads) {
    extern __shared__ __align__(16) unsigned char cand_smem[];
    unsigned* c_key = reinterpret_cast<unsigned*>(cand_smem);  // [kCandCap]
    int* c_pos = reinterpret_cast<int*>(c_key + kCandCap);      // [kCandCap]
    unsigned* samp = whist;                                     // [kSelThreads], reused
    samp[tid] = order_key(sc[(long long)tid * n / kSelThreads]);
    __syncthreads();
    for (int size = 2; size <= kSelThreads; size <<= 1) {  // bitonic sort, descending
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const int p = tid ^ stride;
        if (p > tid) {
          const unsigned a = samp[tid], c = samp[p];
          if (((tid & size) == 0) ? a < c : a > c) {
            samp[tid] = c;
            samp[p] = a;
          }
        }
        __syncthreads();
      }
    }
    const long long srank = ((long long)keep * kSelThreads + n - 1) / n;
    const unsigned tau = samp[(int)min((long long)kSelThreads - 1, srank + srank / 2 + 16)];
    // each thread a contiguous, 16-byte aligned run of positions, 8 vectors in flight
    const int per = (((n + kSelThreads - 1) / kSelThreads) + 3) & ~3;
    const int a0 = min(n, tid * per), a1 = min(n, a0 + per);
    unsigned cnt = 0u;
    for (int u = a0; u < a1; u += 32) {
      float4 f[8];
#pragma unroll
      for (int x = 0; x < 8; ++x)
        if (u + 4 * x < a1) f[x] = *reinterpret_cast<const float4*>(sc + u + 4 * x);
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const float fv[4] = {f[x].x, f[x].y, f[x].z, f[x].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          cnt += (u + 4 * x + e < a1 && order_key(fv[e]) >= tau) ? 1u : 0u;
      }
    }
    unsigned total;
    unsigned w = block_scan_1024(cnt, warp_tot, &total);
    if (total >= (unsigned)keep && total <= (unsigned)kCandCap) {  // the same in every thread
      for (int u = a0; u < a1; u += 32) {
        float4 f[8];
#pragma unroll
        for (int x = 0; x < 8; ++x)
          if (u + 4 * x < a1) f[x] = *reinterpret_cast<const float4*>(sc + u + 4 * x);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float fv[4] = {f[x].x, f[x].y, f[x].z, f[x].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const unsigned k = order_key(fv[e]);
            if (u + 4 * x + e < a1 && k >= tau && MSA_IN_BOUNDS(w, kCandCap, nullptr)) {
              c_key[w] = k;
              c_pos[w] = u + 4 * x + e;
              ++w;
            }
          }
        }
      }
      __syncthreads();
      // radix select of the keep-th largest candidate key
      unsigned prefix = 0u, pmask = 0u, remaining = (unsigned)keep;
      for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256 * kSelWarps; i += kSelThreads) whist[i] = 0u;
        __syncthreads();
        unsigned* wh = whist + (tid / 32) * 256;
        for (int i = tid; i < (int)total; i += kSelThreads) {
          const unsigned k = c_key[i];
          if ((k & pmask) == prefix) atomicAdd(&wh[(k >> shift) & 255u], 1u);
        }
        __syncthreads();
        for (int i = tid; i < 256; i += kSelThreads) {
          unsigned c = 0u;
          for (int ww = 0; ww < kSelWarps; ++ww) c += whist[ww * 256 + i];
          hist[i] = c;
        }
        __syncthreads();
        if (tid < 32) pick_digit(hist, remaining, &s_prefix, &s_remaining);
        __syncthreads();
        prefix |= s_prefix << shift;
        remaining -= s_remaining;
        pmask |= 255u << shift;
        __syncthreads();
      }
      const unsigned T_key = prefix;
      // ordered selection over the candidates (already in position order)
      const int cper = ((int)total + kSelThreads - 1) / kSelThreads;
      const int c0 = min((int)total, tid * cper), c1 = min((int)total, c0 + cper);
      unsigned eq = 0u;
      for (int i = c0; i < c1; ++i) eq += c_key[i] == T_key;
      unsigned tot;
      const unsigned eq_before = block_scan_1024(eq, warp_tot, &tot);
      unsigned sel = 0u;
      {
        unsigned e2 = eq_before;
        for (int i = c0; i < c1; ++i) {
          const unsigned k = c_key[i];
          sel += (k > T_key || (k == T_key && e2 < remaining)) ? 1u : 0u;
          e2 += k == T_key;
        }
      }
      unsigned pos = block_scan_1024(sel, warp_tot, &tot);
      {
        unsigned e2 = eq_before;
        for (int i = c0; i < c1; ++i) {
          const unsigned k = c_key[i];
          const bool s2 = k > T_key || (k == T_key && e2 < remaining);
          e2 += k == T_key;
          if (s2 && pos < (unsigned)keep) out[pos++] = c_pos[i];
        }
      }
      for (int i = keep + tid; i < top_k; i += kSelThreads) out[i] = (i == keep) ? t : -1;
      return;
    }
    __syncthreads();  // the sample buffer is reused by the full select
  }

  // radix select: the key of the keep-th largest score, and how many keys equal
  // to it are kept (the lowest positions among them)
  unsigned prefix = 0u, pmask = 0u, remaining = (unsigned)keep;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256 * kSelWarps; i += kSelThreads) whist[i] = 0u;
    __syncthreads();
    // each warp counts into its own histogram: the keys sit in a few bins (the
    // top byte holds the sign and the high exponent bits), and one shared
    // histogram would serialise every warp's atomics on them
    unsigned* wh = whist + (tid / 32) * 256;
    for (int u0 = 4 * tid; u0 < n; u0 += 4 * kSelThreads) {
      float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
      if (u0 + 3 < n) {
        f = *reinterpret_cast<const float4*>(sc + u0);
      } else {
        f.x = sc[u0];
        f.y = u0 + 1 < n ? sc[u0 + 1] : 0.f;
        f.z = u0 + 2 < n ? sc[u0 + 2] : 0.f;
      }
      const float fv[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const unsigned k = order_key(fv[x]);
        if (u0 + x < n && (k & pmask) == prefix) atomicAdd(&wh[(k >> shift) & 255u], 1u);
      }
    }
    __syncthreads();
    for (int i = tid; i < 256; i += kSelThreads) {
      unsigned c = 0u;
      for (int w = 0; w < kSelWarps; ++w) c += whist[w * 256 + i];
      hist[i] = c;
    }
    __syncthreads();
    if (tid < 32) pick_digit(hist, remaining, &s_prefix, &s_remaining);
    __syncthreads();
    prefix |= s_prefix << shift;
    remaining -= s_remaining;
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
    const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens,
    const int32_t* __restrict__ cu_q, int batch, uint32_t* status,
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

  const int g = blockIdx.x, r = blockIdx.y;
  const int tid = threadIdx.x;
  int b, t;
  if (!token_row(r, cu_q, batch, seq_lens, max_blocks, B, b, t)) {
    if (tid == 0) report(status, MSA_DEV_BAD_LENGTH);
    return;
  }
  for (int e = tid; e < G * D; e += blockDim.x) {
    qs[e] = to_f32(q[((size_t)r * hq + g * G) * D + e]);
    os[e] = 0.f;
  }
  if (tid < G) {
    m_s[tid] = -INFINITY;
    l_s[tid] = 0.f;
  }
  const int32_t* list = tok_idx + (size_t)r * top_k;
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
    out[((size_t)r * hq + g * G) * D + e] = from_f32<T>(l_s[h] > 0.f ? os[e] / l_s[h] : 0.f);
  }
  if (lse && tid < G)
    lse[(size_t)r * hq + g * G + tid] = l_s[tid] > 0.f ? m_s[tid] + logf(l_s[tid]) : -INFINITY;
}

constexpr int kTokTile = 64;    // tokens per stage of the tensor-core attention
constexpr int kTokStages = 3;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Attention of one (sequence, KV group) over the kept positions, G <= 16 query
// heads padded to 16 mma rows. Stage i holds tokens [64 i, 64 i + 64) of the
// list: their K and V rows (256 bytes each) copied into the 128-byte-swizzled
// two-half layout, an invalid slot (padding, an adjacent repeat, a bad page)
// zero-filled and masked. Warp w scores keys [16 w, 16 w + 16) of each stage.
__global__ void __launch_bounds__(128) tok_attn_tc_kernel(
    const bf16* __restrict__ q, const bf16* __restrict__ k_pages, const bf16* __restrict__ v_pages,
    const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens,
    const int32_t* __restrict__ cu_q, int batch, uint32_t* status,
    const int32_t* __restrict__ tok_idx, int top_k, int hq, int hkv, int B, int num_pages,
    int max_blocks, float scale_log2, bf16* __restrict__ out, float* __restrict__ lse) {
  using namespace warpmma;
  constexpr int D = 128;
  constexpr int TILE = kTokTile * D * 2;  // bytes of one K (or V) stage tile
  constexpr int KW = kTokTile / 4;        // keys per warp per stage
  constexpr int NT = KW / 8;              // n-tiles of 8 keys per warp
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ int s_row[kTokStages][kTokTile];  // K/V row of each slot, -1: none
  const int g = blockIdx.x, r = blockIdx.y;
  const int G = hq / hkv;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  int b, t;
  const bool len_ok = token_row(r, cu_q, batch, seq_lens, max_blocks, B, b, t);
  if (!len_ok && g == 0 && tid == 0) report(status, MSA_DEV_BAD_LENGTH);
  const int32_t* list = tok_idx + (size_t)r * top_k;
  const int nstage = len_ok ? (top_k + kTokTile - 1) / kTokTile : 0;

  // slot lookup for stage i (thread tid < 64: slot tid), then 16-byte copies:
  // 64 rows x 16 chunks x {K, V} = 2048 copies, 16 per thread
  auto issue = [&](int i) {
    const int st = i % kTokStages;
    if (tid < kTokTile) {
      const int sidx = i * kTokTile + tid;
      int row = -1;
      if (sidx < top_k) {
        const int u = list[sidx];
        if (u >= 0 && u <= t && !(sidx > 0 && list[sidx - 1] == u)) {
          const int pg = page_table[(size_t)b * max_blocks + u / B];
          if (pg >= 0 && pg < num_pages) row = (pg * hkv + g) * B + u % B;
          else report(status, MSA_DEV_BAD_PAGE);
        } else if (u > t) {
          report(status, MSA_DEV_BAD_INDEX);
        }
      }
      s_row[st][tid] = row;
    }
    __syncthreads();
    const uint32_t kt = smem_u32(smem + st * 2 * TILE), vt = kt + TILE;
#pragma unroll
    for (int x = 0; x < (kTokTile * 16) / 128; ++x) {
      const int e = x * 128 + tid, r = e / 16, c = e % 16;
      const int row = s_row[st][r];
      const size_t off = (size_t)(row < 0 ? 0 : row) * D + c * 8;
      cp_async16(tile_chunk(kt, kTokTile, r, c), k_pages + off, row >= 0);
      cp_async16(tile_chunk(vt, kTokTile, r, c), v_pages + off, row >= 0);
    }
  };

  // query fragments (rows >= G are zero)
  uint32_t qa[8][4];
  {
    const int r0 = lane / 4, r1 = r0 + 8, c = 2 * (lane % 4);
    const bf16* qb = q + ((size_t)r * hq + (size_t)g * G) * D;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int k0 = ks * 16 + c;
      qa[ks][0] = r0 < G ? *reinterpret_cast<const uint32_t*>(qb + r0 * D + k0) : 0u;
      qa[ks][1] = r1 < G ? *reinterpret_cast<const uint32_t*>(qb + r1 * D + k0) : 0u;
      qa[ks][2] = r0 < G ? *reinterpret_cast<const uint32_t*>(qb + r0 * D + k0 + 8) : 0u;
      qa[ks][3] = r1 < G ? *reinterpret_cast<const uint32_t*>(qb + r1 * D + k0 + 8) : 0u;
    }
  }
  for (int i = 0; i < kTokStages - 1; ++i) {
    if (i < nstage) issue(i);
    cp_async_commit();
  }

  float o[16][4];
#pragma unroll
  for (int nd = 0; nd < 16; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  for (int i = 0; i < nstage; ++i) {
    // refill the stage freed by stage i-1 with stage i+2, then wait for stage i
    if (i + kTokStages - 1 < nstage) issue(i + kTokStages - 1);
    cp_async_commit();
    cp_async_wait<kTokStages - 1>();
    __syncthreads();
    const int st = i % kTokStages;
    const uint32_t kt = smem_u32(smem + st * 2 * TILE), vt = kt + TILE;

    float s[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
      const int key0 = warp * KW + nt * 8;
#pragma unroll
      for (int ks = 0; ks < 8; ks += 2) {
        const int key = key0 + (lane & 7);
        const int chunk = 2 * ks + (lane >> 3);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(tile_chunk(kt, kTokTile, key, chunk), b0, b1, b2, b3);
        mma_bf16_16816(s[nt], qa[ks], b0, b1);
        mma_bf16_16816(s[nt], qa[ks + 1], b2, b3);
      }
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int kc = warp * KW + nt * 8 + 2 * (lane % 4);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool ok = s_row[st][kc + (e & 1)] >= 0;
        s[nt][e] = ok ? s[nt][e] * scale_log2 : -INFINITY;
      }
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float ms0 = mn0 == -INFINITY ? 0.f : mn0, ms1 = mn1 == -INFINITY ? 0.f : mn1;
    const float a0 = exp2f(m0 - ms0), a1 = exp2f(m1 - ms1);
    m0 = mn0;
    m1 = mn1;
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      // weights rounded to bf16 once: the row sum and P*V use the same values
#pragma unroll
      for (int e = 0; e < 4; ++e)
        s[nt][e] = __bfloat162float(__float2bfloat16_rn(exp2f(s[nt][e] - (e < 2 ? ms0 : ms1))));
      ps0 += s[nt][0] + s[nt][1];
      ps1 += s[nt][2] + s[nt][3];
    }
    l0 = l0 * a0 + ps0;
    l1 = l1 * a1 + ps1;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      o[nd][0] *= a0;
      o[nd][1] *= a0;
      o[nd][2] *= a1;
      o[nd][3] *= a1;
    }
#pragma unroll
    for (int kk = 0; kk < NT / 2; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
      const int kb = warp * KW + 16 * kk;
      const int key = kb + (lane & 7) + 8 * ((lane >> 3) & 1);
#pragma unroll
      for (int nd = 0; nd < 16; nd += 2) {
        const int chunk = nd + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(tile_chunk(vt, kTokTile, key, chunk), b0, b1, b2, b3);
        mma_bf16_16816(o[nd], pa, b0, b1);
        mma_bf16_16816(o[nd + 1], pa, b2, b3);
      }
    }
    __syncthreads();  // every warp is done with this stage before it is refilled
  }
  cp_async_wait<0>();

  // merge the four warps: quad-sum l, then max/scale across warps in smem
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  __syncthreads();
  float* red_o = reinterpret_cast<float*>(smem);         // [4][16][D]
  float* red_m = red_o + 4 * 16 * D;                      // [4][16]
  float* red_l = red_m + 4 * 16;                          // [4][16]
  const int r0 = lane / 4, r1 = r0 + 8;
  if (lane % 4 == 0) {
    red_m[warp * 16 + r0] = m0;
    red_m[warp * 16 + r1] = m1;
    red_l[warp * 16 + r0] = l0;
    red_l[warp * 16 + r1] = l1;
  }
#pragma unroll
  for (int nd = 0; nd < 16; ++nd) {
    const int c = nd * 8 + 2 * (lane % 4);
    red_o[(warp * 16 + r0) * D + c] = o[nd][0];
    red_o[(warp * 16 + r0) * D + c + 1] = o[nd][1];
    red_o[(warp * 16 + r1) * D + c] = o[nd][2];
    red_o[(warp * 16 + r1) * D + c + 1] = o[nd][3];
  }
  __syncthreads();
  for (int hh = 0; hh < G; ++hh) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, red_m[w * 16 + hh]);
    float acc = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float f = exp2f(red_m[w * 16 + hh] - M);
        acc += f * red_o[(w * 16 + hh) * D + tid];
        lsum += f * red_l[w * 16 + hh];
      }
    }
    const size_t head = (size_t)r * hq + (size_t)g * G + hh;
    out[head * D + tid] = __float2bfloat16_rn(lsum > 0.f ? acc / lsum : 0.f);
    if (lse && tid == 0) lse[head] = lsum > 0.f ? (M + log2f(lsum)) * 0.6931471805599453f : -INFINITY;
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// one fp32 score per (row, position)
size_t tokens_ws(const msa_paged_kv_t* kv, int num_rows) {
  return (size_t)num_rows * kv->max_blocks_per_seq * kv->block_size * sizeof(float);
}

template <typename T, int D>
static cudaError_t launch_tok_select(const msa_paged_kv_t* kv, const void* ki_pages, const void* qi,
                                     int hi, int top_k, int32_t* tok_idx, void* ws,
                                     const int32_t* cu_q, int rows, cudaStream_t st) {
  const int max_len = kv->max_blocks_per_seq * kv->block_size;
  float* scores = (float*)ws;
  dim3 grid((max_len + kScoreChunk - 1) / kScoreChunk, rows);
  tok_score_kernel<T, D><<<grid, 256, 0, st>>>((const T*)qi, (const T*)ki_pages, kv->page_table,
                                               kv->seq_lens, cu_q, kv->batch, kv->status_word, hi,
                                               kv->block_size, kv->num_pages,
                                               kv->max_blocks_per_seq, max_len, scores);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t cand = (size_t)kCandCap * 8;
  e = cudaFuncSetAttribute(tok_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cand);
  if (e != cudaSuccess) return e;
  tok_select_kernel<<<rows, kSelThreads, cand, st>>>(scores, kv->seq_lens, cu_q, kv->batch,
                                                     kv->max_blocks_per_seq, kv->block_size,
                                                     max_len, top_k, tok_idx);
  return cudaGetLastError();
}

cudaError_t select_tokens(const msa_paged_kv_t* kv, const void* ki_pages, const void* qi, int hi,
                          int top_k, int32_t* tok_idx, void* ws, const int32_t* cu_q, int rows,
                          cudaStream_t st) {
  const bool bf = kv->dtype == MSA_DTYPE_BF16;
  if (kv->head_dim == 128)
    return bf ? launch_tok_select<bf16, 128>(kv, ki_pages, qi, hi, top_k, tok_idx, ws, cu_q, rows, st)
              : launch_tok_select<float, 128>(kv, ki_pages, qi, hi, top_k, tok_idx, ws, cu_q, rows, st);
  return bf ? launch_tok_select<bf16, 64>(kv, ki_pages, qi, hi, top_k, tok_idx, ws, cu_q, rows, st)
            : launch_tok_select<float, 64>(kv, ki_pages, qi, hi, top_k, tok_idx, ws, cu_q, rows, st);
}

template <typename T, int D>
static cudaError_t launch_tok_attn(const msa_paged_kv_t* kv, const void* q, const int32_t* tok_idx,
                                   int top_k, float scale, void* out, float* lse,
                                   const int32_t* cu_q, int rows, cudaStream_t st) {
  const int G = kv->num_q_heads / kv->num_kv_heads;
  const size_t smem = ((size_t)2 * G * D + (size_t)kTokChunk * (D + 1) + (size_t)kTokChunk * D +
                       (size_t)G * kTokChunk) * 4;
  auto kern = tok_attn_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(kv->num_kv_heads, rows);
  kern<<<grid, 128, smem, st>>>((const T*)q, (const T*)kv->k_pages, (const T*)kv->v_pages,
                                 kv->page_table, kv->seq_lens, cu_q, kv->batch, kv->status_word,
                                 tok_idx, top_k, kv->num_q_heads, kv->num_kv_heads, kv->block_size,
                                 kv->num_pages, kv->max_blocks_per_seq, scale, (T*)out, lse);
  return cudaGetLastError();
}

cudaError_t attn_tokens(const msa_paged_kv_t* kv, const void* q, const int32_t* tok_idx, int top_k,
                        float scale, void* out, float* lse, const int32_t* cu_q, int rows,
                        cudaStream_t st) {
  const bool bf = kv->dtype == MSA_DTYPE_BF16;
  if (bf && kv->head_dim == 128) {
    const size_t red = (size_t)4 * 16 * 128 * 4 + 2 * 4 * 16 * 4;
    const size_t ring = (size_t)kTokStages * 2 * kTokTile * 128 * 2;
    const size_t smem = (ring > red ? ring : red) + 1024;
    cudaError_t e = cudaFuncSetAttribute(tok_attn_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(kv->num_kv_heads, rows);
    tok_attn_tc_kernel<<<grid, 128, smem, st>>>(
        (const bf16*)q, (const bf16*)kv->k_pages, (const bf16*)kv->v_pages, kv->page_table,
        kv->seq_lens, cu_q, kv->batch, kv->status_word, tok_idx, top_k, kv->num_q_heads,
        kv->num_kv_heads, kv->block_size, kv->num_pages, kv->max_blocks_per_seq,
        scale * 1.4426950408889634f, (bf16*)out, lse);
    return cudaGetLastError();
  }
  if (kv->head_dim == 128)
    return bf ? launch_tok_attn<bf16, 128>(kv, q, tok_idx, top_k, scale, out, lse, cu_q, rows, st)
              : launch_tok_attn<float, 128>(kv, q, tok_idx, top_k, scale, out, lse, cu_q, rows, st);
  return bf ? launch_tok_attn<bf16, 64>(kv, q, tok_idx, top_k, scale, out, lse, cu_q, rows, st)
            : launch_tok_attn<float, 64>(kv, q, tok_idx, top_k, scale, out, lse, cu_q, rows, st);
}

}  // namespace msa
