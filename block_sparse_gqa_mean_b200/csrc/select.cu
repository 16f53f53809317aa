// Exp-free per-group top-k block selection.
//
// "MiniMax Sparse Attention" (staik.se), method paragraph: a light index
// branch scores the key-value blocks and keeps a top-k subset for each GQA
// group independently; results paragraph: the top-k needs no exponentials.
// "Art of Focus: Ling 2.0 ...", "Summarizing the Breakthrough": the heads of a
// GQA group share one selection. Scoring reads only the fp32 block centroids
// of the block cache, never the keys.
//
// For a query row at position t and KV group g:
//   qbar     = sum of the group's query heads (fp32)
//   score_j  = qbar . c_j for complete past blocks j < t / B
//   selected = own block t / B plus the best k-1 under (score desc, index asc)
// Output: ascending block indices, -1 padded; optional scores (+inf own, -inf pad).
//
// Two kernels:
//  * select_rows   - many rows per sequence (prefill / chunked prefill). A CTA
//                    takes 32 consecutive rows of one sequence and one group,
//                    streams the candidate centroids in chunks of 64 through
//                    shared memory, scores them with a register-tiled fp32 fma
//                    micro-kernel and keeps per-thread sorted top lists that
//                    are merged at the end.
//  * select_decode - one row per sequence with thousands of candidates. Pass 1
//                    splits the candidates into chunks of 64 across CTAs
//                    (thread per candidate, bitonic sort of the chunk in shared
//                    memory, keep k-1); pass 2 merges the sorted chunk lists
//                    with a warp-wide tournament.
#include "common.cuh"

namespace msa {

namespace {

constexpr int kRows = 32;       // rows per select_rows CTA
constexpr int kChunk = 64;      // candidates per shared-memory chunk (select_rows)
constexpr int kDecChunk = 64;   // candidates per select_decode pass-1 CTA
constexpr int kMaxChunksPerLane = 8;  // pass 2: chunk lists per lane (256 chunks)

// qbar[i..i+VEC) = q_{gG}[i] + q_{gG+1}[i] + ... (left to right over the heads)
// for VEC = 16 / sizeof(T) consecutive coordinates. All G head loads are
// issued before the sums, as 16-byte vectors.
template <typename T>
__device__ __forceinline__ void load_qbar_vec(const T* __restrict__ qrow, int G, int g, int D, int i,
                                              float* out) {
  constexpr int VEC = 16 / sizeof(T);
  uint4 v[16];
  const T* p = qrow + (size_t)g * G * D + i;
#pragma unroll
  for (int h = 0; h < 16; ++h)
    if (h < G) v[h] = *reinterpret_cast<const uint4*>(p + (size_t)h * D);
  float acc[VEC];
  {
    const T* e = reinterpret_cast<const T*>(&v[0]);
#pragma unroll
    for (int x = 0; x < VEC; ++x) acc[x] = to_f32(e[x]);
  }
#pragma unroll
  for (int h = 1; h < 16; ++h) {
    if (h < G) {
      const T* e = reinterpret_cast<const T*>(&v[h]);
#pragma unroll
      for (int x = 0; x < VEC; ++x) acc[x] = __fadd_rn(acc[x], to_f32(e[x]));
    }
  }
#pragma unroll
  for (int x = 0; x < VEC; ++x) out[x] = acc[x];
}

// Sorted insertion into a descending list of N keys (L[N-1] smallest).
template <int N>
__device__ __forceinline__ void insert_key(uint64_t (&L)[N], uint64_t key) {
  if (key <= L[N - 1]) return;
#pragma unroll
  for (int s = N - 1; s > 0; --s) {
    const uint64_t prev = L[s - 1];
    L[s] = key > prev ? prev : (key > L[s] ? key : L[s]);
  }
  L[0] = key > L[0] ? key : L[0];
}

// Write the selection of one (row, group): `n` chosen past blocks given as
// keys (any order, 0 = empty), plus the own block, ascending, -1 padded.
__device__ void write_selection(const uint64_t* keys, int n, int own, int top_k, int32_t* idx_out,
                                float* score_out) {
  int cnt = 0;
  for (int a = 0; a < n; ++a) cnt += keys[a] != 0ull;
  for (int a = 0; a < n; ++a) {
    if (keys[a] == 0ull) continue;
    const int ja = key_block(keys[a]);
    int rank = 0;
    for (int c = 0; c < n; ++c)
      if (keys[c] != 0ull && key_block(keys[c]) < ja) ++rank;
    idx_out[rank] = ja;
    if (score_out) score_out[rank] = key_score(keys[a]);
  }
  idx_out[cnt] = own;
  if (score_out) score_out[cnt] = __int_as_float(0x7f800000);
  for (int s = cnt + 1; s < top_k; ++s) {
    idx_out[s] = -1;
    if (score_out) score_out[s] = __int_as_float(0xff800000);
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// select_rows
// ---------------------------------------------------------------------------
template <typename T, int D, int KMAX>
__global__ void __launch_bounds__(256) select_rows_kernel(
    const T* __restrict__ q, const int32_t* __restrict__ cu_q, const float* __restrict__ centroids,
    const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens, uint32_t* status,
    int hq, int hkv, int B, int num_pages, int max_blocks, int top_k, int32_t* __restrict__ idx,
    float* __restrict__ score) {
  constexpr int SUBS = 256 / kRows;  // 8 threads per row in the selection phase
  constexpr int CP = D + 4;          // padded centroid row (bank spread)
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* qbar = reinterpret_cast<float*>(smem_raw);                  // [kRows][D]
  float* cent = qbar + kRows * D;                                     // [kChunk][CP]
  float* sc = cent + kChunk * CP;                                     // [kRows][kChunk]
  uint64_t* lists = reinterpret_cast<uint64_t*>(sc + kRows * kChunk); // [kRows][SUBS][KMAX]
  __shared__ int s_page[kChunk];

  const int b = blockIdx.y, g = blockIdx.z;
  const int G = hq / hkv;
  const int row0 = cu_q[b];
  const int n_rows = cu_q[b + 1] - row0;
  const int r_lo = blockIdx.x * kRows;
  if (r_lo >= n_rows) return;
  const int nr = min(kRows, n_rows - r_lo);
  const int L = seq_lens[b];
  if (n_rows > L || L > max_blocks * B) {
    if (threadIdx.x == 0) report(status, MSA_DEV_BAD_LENGTH);
    return;
  }
  const int tid = threadIdx.x;

  // qbar for the tile's rows
  {
    constexpr int VEC = 16 / sizeof(T);
    for (int e = tid; e < kRows * (D / VEC); e += 256) {
      const int r = e / (D / VEC), i = (e % (D / VEC)) * VEC;
      float* dst = &qbar[r * D + i];
      if (r < nr) {
        load_qbar_vec<T>(q + (size_t)(row0 + r_lo + r) * hq * D, G, g, D, i, dst);
      } else {
#pragma unroll
        for (int x = 0; x < VEC; ++x) dst[x] = 0.f;
      }
    }
  }
  const int t_first = row_position(L, n_rows, r_lo);
  const int t_last = row_position(L, n_rows, r_lo + nr - 1);
  const int ncand = t_last / B;  // candidates of the last row; earlier rows use a prefix

  // selection state: thread (row sr, sub ss) keeps candidates j = ss (mod SUBS)
  const int sr = tid / SUBS, ss = tid % SUBS;
  const int my_t = row_position(L, n_rows, r_lo + sr);
  const int my_nc = (sr < nr) ? my_t / B : 0;
  uint64_t top[KMAX];
#pragma unroll
  for (int s = 0; s < KMAX; ++s) top[s] = 0ull;

  // score micro-tile: thread (tr, tc) -> rows 2tr, 2tr+1 and candidates tc + 16m, m < 4
  const int tr = tid / 16, tc = tid % 16;
  (void)t_first;

  for (int c0 = 0; c0 < ncand; c0 += kChunk) {
    const int nc = min(kChunk, ncand - c0);
    __syncthreads();  // previous chunk fully consumed (also orders qbar writes)
    if (tid < kChunk) {
      int pg = -1;
      if (tid < nc) {
        pg = page_table[(size_t)b * max_blocks + c0 + tid];
        if (pg < 0 || pg >= num_pages) {
          report(status, MSA_DEV_BAD_PAGE);
          pg = -1;
        }
      }
      s_page[tid] = pg;
    }
    __syncthreads();
    for (int e = tid; e < kChunk * (D / 4); e += 256) {
      const int jj = e / (D / 4), i4 = (e % (D / 4)) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (jj < nc && s_page[jj] >= 0)
        v = *reinterpret_cast<const float4*>(centroids + ((size_t)s_page[jj] * hkv + g) * D + i4);
      *reinterpret_cast<float4*>(&cent[jj * CP + i4]) = v;
    }
    __syncthreads();
    {
      float acc[2][4];
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int m = 0; m < 4; ++m) acc[a][m] = 0.f;
      const float* q0 = qbar + (2 * tr) * D;
      const float* q1 = q0 + D;
#pragma unroll 4
      for (int i = 0; i < D; i += 4) {
        const float4 a0 = *reinterpret_cast<const float4*>(q0 + i);
        const float4 a1 = *reinterpret_cast<const float4*>(q1 + i);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float4 cv = *reinterpret_cast<const float4*>(cent + (tc + 16 * m) * CP + i);
          acc[0][m] = __fmaf_rn(a0.x, cv.x, acc[0][m]);
          acc[0][m] = __fmaf_rn(a0.y, cv.y, acc[0][m]);
          acc[0][m] = __fmaf_rn(a0.z, cv.z, acc[0][m]);
          acc[0][m] = __fmaf_rn(a0.w, cv.w, acc[0][m]);
          acc[1][m] = __fmaf_rn(a1.x, cv.x, acc[1][m]);
          acc[1][m] = __fmaf_rn(a1.y, cv.y, acc[1][m]);
          acc[1][m] = __fmaf_rn(a1.z, cv.z, acc[1][m]);
          acc[1][m] = __fmaf_rn(a1.w, cv.w, acc[1][m]);
        }
      }
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int m = 0; m < 4; ++m) sc[(2 * tr + a) * kChunk + tc + 16 * m] = acc[a][m];
    }
    __syncthreads();
    if (sr < nr) {
      for (int jj = ss; jj < nc; jj += SUBS) {
        const int j = c0 + jj;
        if (j >= my_nc || s_page[jj] < 0) continue;
        insert_key<KMAX>(top, sel_key(sc[sr * kChunk + jj], j));
      }
    }
  }

  // merge the SUBS lists of each row pairwise (3 levels). Two descending lists
  // A, B: max(A[i], B[N-1-i]) holds the top N as a bitonic sequence, which a
  // half-cleaner network sorts back into descending order.
  uint64_t* my_list = lists + ((size_t)sr * SUBS + ss) * KMAX;
#pragma unroll
  for (int s = 0; s < KMAX; ++s) my_list[s] = top[s];
  __syncthreads();
#pragma unroll
  for (int w = 1; w < SUBS; w <<= 1) {
    if ((ss & (2 * w - 1)) == 0) {
      const uint64_t* other = my_list + (size_t)w * KMAX;
#pragma unroll
      for (int s = 0; s < KMAX; ++s) {
        const uint64_t o = other[KMAX - 1 - s];
        top[s] = top[s] > o ? top[s] : o;
      }
#pragma unroll
      for (int stride = KMAX / 2; stride >= 1; stride >>= 1) {
#pragma unroll
        for (int s = 0; s < KMAX; ++s) {
          if ((s & stride) == 0) {
            const uint64_t a = top[s], c = top[s + stride];
            top[s] = a > c ? a : c;
            top[s + stride] = a > c ? c : a;
          }
        }
      }
#pragma unroll
      for (int s = 0; s < KMAX; ++s) my_list[s] = top[s];
    }
    __syncthreads();
  }
  if (ss == 0 && sr < nr) {
    const int keep = min(top_k - 1, my_nc);
#pragma unroll
    for (int s = 0; s < KMAX; ++s) my_list[s] = (s < keep) ? top[s] : 0ull;
    const size_t out = ((size_t)(row0 + r_lo + sr) * hkv + g) * top_k;
    write_selection(my_list, min(keep, KMAX), my_t / B, top_k, idx + out, score ? score + out : nullptr);
  }
}

// ---------------------------------------------------------------------------
// select_decode
// ---------------------------------------------------------------------------
// Bitonic sort of n (power of two) keys in shared memory, descending.
__device__ void bitonic_desc(uint64_t* k, int n) {
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      __syncthreads();
      for (int t = threadIdx.x; t < n / 2; t += blockDim.x) {
        const int lo = 2 * t - (t & (stride - 1));
        const int hi = lo + stride;
        const bool desc = ((lo & size) == 0);
        const uint64_t a = k[lo], c = k[hi];
        if (desc ? (a < c) : (a > c)) {
          k[lo] = c;
          k[hi] = a;
        }
      }
    }
  }
  __syncthreads();
}

template <typename T, int D>
__global__ void __launch_bounds__(kDecChunk) select_decode_pass1(
    const T* __restrict__ q, const float* __restrict__ centroids,
    const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens, uint32_t* status,
    int hq, int hkv, int B, int num_pages, int max_blocks, int kw, int nchunks,
    uint64_t* __restrict__ ws) {
  constexpr int CP = D + 4;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* cent = reinterpret_cast<float*>(smem_raw);  // [kDecChunk][CP]
  __shared__ float qbar[D];
  __shared__ uint64_t keys[kDecChunk];
  __shared__ int s_page[kDecChunk];
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = hq / hkv;
  const int L = seq_lens[b];
  uint64_t* out = ws + (((size_t)b * hkv + g) * nchunks + c) * kw;
  if (L < 1 || L > max_blocks * B) {
    if (c == 0 && g == 0 && threadIdx.x == 0) report(status, MSA_DEV_BAD_LENGTH);
    for (int s = threadIdx.x; s < kw; s += blockDim.x) out[s] = 0ull;
    return;
  }
  const int ncand = (L - 1) / B;
  const int j0 = c * kDecChunk;
  const int nc = max(0, min(kDecChunk, ncand - j0));
  if (nc == 0) {
    for (int s = threadIdx.x; s < kw; s += blockDim.x) out[s] = 0ull;
    return;
  }
  const int tid = threadIdx.x;
  {
    constexpr int VEC = 16 / sizeof(T);
    for (int i = tid * VEC; i < D; i += blockDim.x * VEC)
      load_qbar_vec<T>(q + (size_t)b * hq * D, G, g, D, i, &qbar[i]);
  }
  {
    int pg = -1;
    if (tid < nc) {
      pg = page_table[(size_t)b * max_blocks + j0 + tid];
      if (pg < 0 || pg >= num_pages) {
        report(status, MSA_DEV_BAD_PAGE);
        pg = -1;
      }
    }
    s_page[tid] = pg;
  }
  __syncthreads();
  // stage the chunk's centroids: 16-byte async copies, one candidate row per 32 threads
  for (int e = tid; e < nc * (D / 4); e += blockDim.x) {
    const int jj = e / (D / 4), i4 = (e % (D / 4)) * 4;
    float* dst = &cent[jj * CP + i4];
    if (s_page[jj] >= 0) {
      const float* src = centroids + ((size_t)s_page[jj] * hkv + g) * D + i4;
      const uint32_t saddr = (uint32_t)__cvta_generic_to_shared(dst);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(saddr), "l"(src));
    }
  }
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
  __syncthreads();
  uint64_t key = 0ull;
  if (tid < nc && s_page[tid] >= 0) {
    const float* cr = cent + tid * CP;
    float s = 0.f;
#pragma unroll 8
    for (int i = 0; i < D; i += 4) {
      const float4 cv = *reinterpret_cast<const float4*>(cr + i);
      s = __fmaf_rn(qbar[i], cv.x, s);
      s = __fmaf_rn(qbar[i + 1], cv.y, s);
      s = __fmaf_rn(qbar[i + 2], cv.z, s);
      s = __fmaf_rn(qbar[i + 3], cv.w, s);
    }
    key = sel_key(s, j0 + tid);
  }
  keys[tid] = key;
  bitonic_desc(keys, kDecChunk);
  for (int s = tid; s < kw; s += blockDim.x) out[s] = keys[s];
}

// Pass 2: one warp per (sequence, group) merges the chunk lists, each already
// sorted by pass 1, with a tournament: every round the lanes offer the heads
// of their chunks, the warp maximum is taken and its chunk advances.
__global__ void __launch_bounds__(32) select_decode_pass2(
    const uint64_t* __restrict__ ws, const int32_t* __restrict__ seq_lens, int hkv, int B,
    int max_blocks, int kw, int nchunks, int top_k, int32_t* __restrict__ idx,
    float* __restrict__ score) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint64_t* lists = reinterpret_cast<uint64_t*>(smem_raw);  // [nch][kw]
  __shared__ uint64_t chosen[256];
  const int g = blockIdx.x, b = blockIdx.y, lane = threadIdx.x;
  const int L = seq_lens[b];
  const size_t outo = ((size_t)b * hkv + g) * top_k;
  if (L < 1 || L > max_blocks * B) return;  // reported by pass 1
  const int own = (L - 1) / B;
  const int ncand = own;
  const int keep = min(top_k - 1, ncand);
  const int nch = (ncand + kDecChunk - 1) / kDecChunk;
  const uint64_t* src = ws + ((size_t)b * hkv + g) * nchunks * kw;
  const int total = nch * kw;
  for (int i0 = 0; i0 < total; i0 += 8 * 32) {  // eight independent loads per lane in flight
    uint64_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * 32 + lane;
      v[u] = i < total ? src[i] : 0ull;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u * 32 + lane;
      if (i < total) lists[i] = v[u];
    }
  }
  __syncwarp();
  int ptr[kMaxChunksPerLane];
  uint64_t head[kMaxChunksPerLane];
#pragma unroll
  for (int s = 0; s < kMaxChunksPerLane; ++s) {
    const int c = lane + 32 * s;
    ptr[s] = 0;
    head[s] = (c < nch) ? lists[(size_t)c * kw] : 0ull;
  }
  int cnt = 0;
  for (; cnt < keep; ++cnt) {
    uint64_t best = 0ull;
#pragma unroll
    for (int s = 0; s < kMaxChunksPerLane; ++s) best = head[s] > best ? head[s] : best;
    uint64_t wb = best;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)wb, o);
      const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(wb >> 32), o);
      const uint64_t other = ((uint64_t)hi << 32) | lo;
      wb = other > wb ? other : wb;
    }
    if (wb == 0ull) break;  // fewer real candidates than requested (bad pages)
#pragma unroll
    for (int s = 0; s < kMaxChunksPerLane; ++s) {
      if (head[s] == wb) {  // keys are unique: exactly one lane, one chunk
        const int c = lane + 32 * s;
        const int nxt = ++ptr[s];
        head[s] = (nxt < kw) ? lists[(size_t)c * kw + nxt] : 0ull;
      }
    }
    if (lane == 0) chosen[cnt] = wb;
  }
  __syncwarp();
  // ascending output: rank by block index
  for (int a = lane; a < cnt; a += 32) {
    const uint64_t ka = chosen[a];
    const int ja = key_block(ka);
    int rank = 0;
    for (int c2 = 0; c2 < cnt; ++c2)
      if (key_block(chosen[c2]) < ja) ++rank;
    idx[outo + rank] = ja;
    if (score) score[outo + rank] = key_score(ka);
  }
  if (lane == 0) {
    idx[outo + cnt] = own;
    if (score) score[outo + cnt] = __int_as_float(0x7f800000);
  }
  for (int s = cnt + 1 + lane; s < top_k; s += 32) {
    idx[outo + s] = -1;
    if (score) score[outo + s] = __int_as_float(0xff800000);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int kmax_for(int top_k) { return top_k - 1 <= 16 ? 16 : (top_k - 1 <= 32 ? 32 : 64); }

static size_t rows_smem(int D, int kmax) {
  return (size_t)kRows * D * 4 + (size_t)kChunk * (D + 4) * 4 + (size_t)kRows * kChunk * 4 +
         (size_t)kRows * (256 / kRows) * kmax * 8;
}

template <typename T, int D, int KMAX>
static cudaError_t launch_rows(const msa_paged_kv_t* kv, const void* q, const int32_t* cu_q,
                               int max_rows, int top_k, int32_t* idx, float* score,
                               cudaStream_t st) {
  const size_t smem = rows_smem(D, KMAX);
  auto kern = select_rows_kernel<T, D, KMAX>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((max_rows + kRows - 1) / kRows, kv->batch, kv->num_kv_heads);
  kern<<<grid, 256, smem, st>>>((const T*)q, cu_q, kv->centroids, kv->page_table, kv->seq_lens,
                                 kv->status_word, kv->num_q_heads, kv->num_kv_heads,
                                 kv->block_size, kv->num_pages, kv->max_blocks_per_seq, top_k, idx,
                                 score);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t rows_dispatch_k(const msa_paged_kv_t* kv, const void* q, const int32_t* cu_q,
                                   int max_rows, int top_k, int32_t* idx, float* score,
                                   cudaStream_t st) {
  switch (kmax_for(top_k)) {
    case 16: return launch_rows<T, D, 16>(kv, q, cu_q, max_rows, top_k, idx, score, st);
    case 32: return launch_rows<T, D, 32>(kv, q, cu_q, max_rows, top_k, idx, score, st);
    default: return launch_rows<T, D, 64>(kv, q, cu_q, max_rows, top_k, idx, score, st);
  }
}

cudaError_t select_rows(const msa_paged_kv_t* kv, const void* q, const int32_t* cu_q, int max_rows,
                        int top_k, int32_t* idx, float* score, cudaStream_t st) {
  const bool bf = kv->dtype == MSA_DTYPE_BF16;
  if (kv->head_dim == 128)
    return bf ? rows_dispatch_k<bf16, 128>(kv, q, cu_q, max_rows, top_k, idx, score, st)
              : rows_dispatch_k<float, 128>(kv, q, cu_q, max_rows, top_k, idx, score, st);
  return bf ? rows_dispatch_k<bf16, 64>(kv, q, cu_q, max_rows, top_k, idx, score, st)
            : rows_dispatch_k<float, 64>(kv, q, cu_q, max_rows, top_k, idx, score, st);
}

bool select_rows_supported(int top_k) { return top_k - 1 <= 64; }

// decode selection merges at most 32 * kMaxChunksPerLane chunk lists of
// kDecChunk candidates
bool select_decode_supported(const msa_paged_kv_t* kv) {
  return kv->max_blocks_per_seq <= 32 * kMaxChunksPerLane * kDecChunk;
}

static int decode_nchunks(const msa_paged_kv_t* kv) {
  return (kv->max_blocks_per_seq + kDecChunk - 1) / kDecChunk;
}
static int decode_kw(int top_k) { return top_k - 1 < kDecChunk ? (top_k - 1 < 1 ? 1 : top_k - 1) : kDecChunk; }

size_t select_decode_ws(const msa_paged_kv_t* kv, int top_k) {
  return (size_t)kv->batch * kv->num_kv_heads * decode_nchunks(kv) * decode_kw(top_k) * 8;
}

template <typename T, int D>
static cudaError_t launch_decode_sel(const msa_paged_kv_t* kv, const void* q, int top_k,
                                     int32_t* idx, float* score, void* ws, cudaStream_t st) {
  const int nch = decode_nchunks(kv), kw = decode_kw(top_k);
  const size_t smem = (size_t)kDecChunk * (D + 4) * 4;
  auto k1 = select_decode_pass1<T, D>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 g1(nch, kv->num_kv_heads, kv->batch);
  k1<<<g1, kDecChunk, smem, st>>>((const T*)q, kv->centroids, kv->page_table, kv->seq_lens,
                                   kv->status_word, kv->num_q_heads, kv->num_kv_heads,
                                   kv->block_size, kv->num_pages, kv->max_blocks_per_seq, kw, nch,
                                   (uint64_t*)ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(kv->num_kv_heads, kv->batch);
  const size_t smem2 = (size_t)nch * kw * 8;
  e = cudaFuncSetAttribute(select_decode_pass2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem2);
  if (e != cudaSuccess) return e;
  select_decode_pass2<<<g2, 32, smem2, st>>>((const uint64_t*)ws, kv->seq_lens, kv->num_kv_heads,
                                          kv->block_size, kv->max_blocks_per_seq, kw, nch, top_k,
                                          idx, score);
  return cudaGetLastError();
}

cudaError_t select_decode(const msa_paged_kv_t* kv, const void* q, int top_k, int32_t* idx,
                          float* score, void* ws, cudaStream_t st) {
  const bool bf = kv->dtype == MSA_DTYPE_BF16;
  if (kv->head_dim == 128)
    return bf ? launch_decode_sel<bf16, 128>(kv, q, top_k, idx, score, ws, st)
              : launch_decode_sel<float, 128>(kv, q, top_k, idx, score, ws, st);
  return bf ? launch_decode_sel<bf16, 64>(kv, q, top_k, idx, score, ws, st)
            : launch_decode_sel<float, 64>(kv, q, top_k, idx, score, ws, st);
}

}  // namespace msa
