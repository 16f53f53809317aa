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
//                    cuts the candidates into chunks of 64 and streams whole
//                    pages of the block cache (every group of a candidate in
//                    one bulk copy) through persistent CTAs with a producer
//                    warp, thread per (candidate, group), a register bitonic
//                    sort per group and chunk, keep k-1; pass 2 merges the
//                    sorted chunk lists with a warp-wide tournament.
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "tma.cuh"

namespace msa {

namespace {

constexpr int kRows = 32;       // rows per select_rows CTA
constexpr int kChunk = 64;      // candidates per shared-memory chunk (select_rows)
constexpr int kDecChunk = 64;   // candidates per select_decode pass-1 CTA
constexpr int kMaxChunksPerLane = 8;  // pass 2: chunk lists per lane (256 chunks)
constexpr int kPass1Threads = 128;  // decode pass 1: consumer threads (plus one producer warp)

// decode pass 1: candidates per step, a power of two <= 32 with SC * hkv <= 128
__host__ __device__ inline int pass1_sc(int hkv) {
  int sc = 32;
  while (sc > 1 && sc * hkv > kPass1Threads) sc >>= 1;
  return sc;
}
// one stage: SC padded page copies (the item's groups of each candidate); 128-byte multiple
__host__ __device__ inline int pass1_stage_bytes(int hg, int D) {
  const int page = hg * D * 4;
  return (pass1_sc(hg) * (page + 16) + 127) & ~127;
}

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

__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, m);
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), m);
  return ((uint64_t)hi << 32) | lo;
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

// Write the selection of one (row, group) from the `lanes` threads that
// share it (consecutive lanes of one warp, `part` = this thread's index among
// them): `keys` holds the chosen past blocks, descending, non-zero keys first
// (a zero key is an empty slot). Output: those blocks ascending, then the own
// block, then -1. Each thread ranks keys part, part + lanes, ... by counting
// the keys with a lower block index.
__device__ void write_selection(const uint64_t* keys, int n, int own, int top_k, int part,
                                int lanes, int32_t* idx_out, float* score_out) {
  int cnt = 0;
  while (cnt < n && keys[cnt] != 0ull) ++cnt;
  for (int a = part; a < cnt; a += lanes) {
    const int ja = key_block(keys[a]);
    int rank = 0;
    for (int c = 0; c < cnt; ++c) rank += key_block(keys[c]) < ja;
    idx_out[rank] = ja;
    if (score_out) score_out[rank] = key_score(keys[a]);
  }
  for (int s = cnt + part; s < top_k; s += lanes) {
    idx_out[s] = s == cnt ? own : -1;
    if (score_out) score_out[s] = __int_as_float(s == cnt ? 0x7f800000 : 0xff800000);
  }
}

}  // namespace

// ---------------------------------------------------------------------------
// select_rows
// ---------------------------------------------------------------------------
template <typename T, int D, int KMAX>
__global__ void __launch_bounds__(256, KMAX <= 16 ? 3 : 1) select_rows_kernel(
    const T* __restrict__ q, const int32_t* __restrict__ cu_q, const float* __restrict__ centroids,
    const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens, uint32_t* status,
    int hq, int hkv, int B, int num_pages, int max_blocks, int top_k, int32_t* __restrict__ idx,
    float* __restrict__ score) {
  constexpr int SUBS = 256 / kRows;  // 8 threads per row in the selection phase
  constexpr int CP = D + 4;          // padded centroid row (bank spread)
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* qbar = reinterpret_cast<float*>(smem_raw);                  // [kRows][D]
  float* cent = qbar + kRows * D;                                     // [kChunk][CP]
  float* sc = cent + kChunk * CP;                                     // [kRows][kChunk]
  // the merge lists reuse the chunk buffers once every chunk is scored
  uint64_t* lists = reinterpret_cast<uint64_t*>(cent);                // [kRows][SUBS][KMAX]
  __shared__ int s_page[kChunk];

  const int b = blockIdx.y, g = blockIdx.z;
  const int G = hq / hkv;
  const int row0 = cu_q[b];
  const int n_rows = cu_q[b + 1] - row0;
  const int r_lo = blockIdx.x * kRows;
  // the sequence's rows lie inside q / idx, and the grid covers all of them
  if (blockIdx.x == 0 && threadIdx.x == 0) (void)MSA_RANGE_OK(n_rows, n_rows, gridDim.x * kRows, status);
  if (!MSA_RANGE_OK(row0, row0 + n_rows, cu_q[gridDim.y], status)) return;
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
  // Row threshold. The row keeps its best k-1 <= KMAX candidates, and its
  // SUBS threads hold SUBS * QK = KMAX keys at or above the smallest of their
  // QK-th best keys. A candidate below that key has k-1 better ones already
  // and can never be kept, so it is not inserted; every key of the final
  // selection still reaches its thread's list, and the selection is
  // unchanged. Refreshed after every chunk (0 until each thread holds QK keys).
  constexpr int QK = KMAX / SUBS;
  uint64_t row_thr = 0ull;

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
    // the chunk's candidates above the thresholds, one bit each, then the
    // inserts: a warp runs as many insert rounds as its busiest thread has
    // survivors, not one per candidate
    uint32_t live = 0u;
    if (sr < nr) {
      const uint64_t thr = row_thr > top[KMAX - 1] ? row_thr : top[KMAX - 1];
#pragma unroll
      for (int m = 0; m < kChunk / SUBS; ++m) {
        const int jj = ss + m * SUBS, j = c0 + jj;
        if (jj < nc && j < my_nc && s_page[jj] >= 0 && sel_key(sc[sr * kChunk + jj], j) > thr)
          live |= 1u << m;
      }
    }
    while (live) {
      const int m = __ffs(live) - 1;
      live &= live - 1u;
      const int jj = ss + m * SUBS;
      insert_key<KMAX>(top, sel_key(sc[sr * kChunk + jj], c0 + jj));
    }
    // refresh the row threshold: the minimum over the row's SUBS threads (SUBS
    // consecutive lanes of one warp) of their QK-th best key
    uint64_t kth = top[QK - 1];
#pragma unroll
    for (int o = 1; o < SUBS; o <<= 1) {
      const uint64_t x = shfl_xor_u64(kth, o);
      kth = x < kth ? x : kth;
    }
    row_thr = kth;
  }

  // merge the SUBS lists of each row pairwise (3 levels). Two descending lists
  // A, B: max(A[i], B[N-1-i]) holds the top N as a bitonic sequence, which a
  // half-cleaner network sorts back into descending order.
  uint64_t* my_list = lists + ((size_t)sr * SUBS + ss) * KMAX;
  __syncthreads();  // the last chunk's scores are read: the lists may overwrite them
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
  const int keep = min(top_k - 1, my_nc);
  if (ss == 0 && sr < nr) {
#pragma unroll
    for (int s = 0; s < KMAX; ++s) my_list[s] = (s < keep) ? top[s] : 0ull;
  }
  __syncwarp();  // the row's SUBS threads are consecutive lanes of one warp
  if (sr < nr) {
    const size_t out = ((size_t)(row0 + r_lo + sr) * hkv + g) * top_k;
    write_selection(lists + (size_t)sr * SUBS * KMAX, min(keep, KMAX), my_t / B, top_k, ss, SUBS,
                    idx + out, score ? score + out : nullptr);
  }
}

// ---------------------------------------------------------------------------
// select_decode
// ---------------------------------------------------------------------------

// Pass 1 of decode selection. An item is (sequence b, chunk c of 64 candidate
// blocks, subset gs of hg consecutive KV groups); items are numbered over the
// non-empty chunks and taken round-robin by the persistent CTAs (CTA i takes
// items i, i + grid, ...; the items are equal in size but for each sequence's
// last chunk). The block cache keeps all groups of a page together, so one
// bulk copy brings one candidate for the item's hg groups (hg * D fp32, 2 KB
// for 4 groups of d 128). An item is streamed in KPL steps of SC = 64 / KPL
// candidates through an NST-stage ring of shared memory.
//   * warp 4 (producer) reads the page-table entries one step ahead and per
//     step issues the page copies, completing on the stage's `full` mbarrier;
//     with an item's first step it also copies the item's raw query rows (its
//     hg groups' G heads each) into `qraw`, completing on `qfull`;
//   * warps 0-3 (consumers): at the start of an item they sum each group's
//     query heads into qbar (fp32, left to right over the heads: the same order
//     as every other selection path), then thread t scores candidate t % SC of
//     each step for group gs * hg + t / SC with the canonical fp32 fma chain,
//     keeps the key in register slot `step`, and the warp releases the stage
//     on `empty`. After the item's last step the SC lanes of a group hold its
//     64 keys (KPL each) and sort them with a bitonic network (in-register
//     strides below KPL, shuffles above); element e of the sorted order is
//     rank e.
template <typename T, int D, int KPL, int NST>
__global__ void __launch_bounds__(kPass1Threads + 32, 1) select_decode_pass1(
    const T* __restrict__ q, const float* __restrict__ centroids,
    const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens, uint32_t* status,
    int batch, int hq, int hkv, int hg, int B, int num_pages, int max_blocks, int kw, int nchunks,
    int cand_lo, int cand_hi, uint64_t* __restrict__ ws) {
  constexpr int SC = kDecChunk / KPL;         // candidates per step = lanes per group
  constexpr int NCW = kPass1Threads / 32;     // consumer warps
  constexpr int NW = NCW + 1;
  constexpr int kNoCand = -0x7fffffff - 1;
  static_assert(SC >= 1 && SC <= 32, "a group's lanes stay inside one warp");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full[NST];
  __shared__ __align__(8) uint64_t empty[NST];
  __shared__ __align__(8) uint64_t qfull, qempty, qready;
  __shared__ int s_item[NST][3];  // (b, c, gs) of the step held by each stage
  __shared__ uint32_t s_valid[NST];  // bit k: candidate k of the step was copied
  __shared__ int wsum[NW];
  const int G = hq / hkv;
  const int hsplit = hkv / hg;                 // items per (sequence, chunk)
  const uint32_t page_bytes = (uint32_t)hg * D * 4;  // the item's groups of one page
  const uint32_t q_bytes = (uint32_t)hg * G * D * sizeof(T);  // the item's raw query rows
  const int pstride = (int)page_bytes + 16;   // padded: conflict-free float4 reads
  const int stage_bytes = pass1_stage_bytes(hg, D);
  T* qraw = reinterpret_cast<T*>(smem_raw + (size_t)NST * stage_bytes);
  float* qbar2 = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(qraw) + q_bytes);  // [2][hg][D]
  int* pre = reinterpret_cast<int*>(qbar2 + 2 * hg * D);                                       // [batch + 1]
  int* ncs = pre + batch + 1;                                                                  // [batch]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCW);
    }
    mbar_init(&qfull, 1);
    mbar_init(&qempty, NCW);
    mbar_init(&qready, kPass1Threads);
    mbar_fence_init();
  }
  pdl_wait();
  // candidates and chunk counts per sequence -> prefix sums pre[b]
  int carry = 0;
  for (int base = 0; base < batch; base += NW * 32) {
    const int b = base + tid;
    int n = 0;
    if (b < batch) {
      const int L = seq_lens[b];
      int nc = 0;
      if (L < 1 || L > max_blocks * B) {
        if (blockIdx.x == 0) report(status, MSA_DEV_BAD_LENGTH);
      } else {
        // candidates: complete past blocks in [cand_lo, cand_hi)
        nc = max(0, min((L - 1) / B, cand_hi) - cand_lo);
        n = (nc + kDecChunk - 1) / kDecChunk * hsplit;
      }
      ncs[b] = nc;
    }
    int v = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += t;
    }
    if (lane == 31) wsum[warp] = v;
    __syncthreads();
    int before = 0, all = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      before += w < warp ? wsum[w] : 0;
      all += wsum[w];
    }
    if (b < batch) pre[b + 1] = carry + before + v;
    carry += all;
    __syncthreads();
  }
  if (tid == 0) pre[0] = 0;
  __syncthreads();
  const int total_items = pre[batch];

  if (warp == NCW) {
    // ------------------------------ producer ------------------------------
    int cur_b = 0, cur_c = 0, cur_gs = 0;
    // locate item `it` (sets cur_*); returns this lane's page entry for step `sub`
    auto fetch = [&](int it, int sub) {
      int lo = 0, hi = batch;  // pre[lo] <= it < pre[hi]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] <= it) lo = mid; else hi = mid;
      }
      cur_b = lo;
      const int r = it - pre[lo];
      cur_c = r / hsplit;
      cur_gs = r - cur_c * hsplit;
      const int j = cur_c * kDecChunk + sub * SC + lane;
      return (lane < SC && j < ncs[lo]) ? page_table[(size_t)lo * max_blocks + cand_lo + j]
                                        : kNoCand;
    };
    int it = (int)blockIdx.x < total_items ? (int)blockIdx.x : -1, sub = 0;
    int pg = it >= 0 ? fetch(it, 0) : kNoCand;
    int n = 0, items = 0;
    for (;; ++n) {
      const int s = n % NST;
      if (n >= NST &&
          !__all_sync(0xffffffffu, mbar_wait(&empty[s], (uint32_t)((n / NST) - 1) & 1u))) {
        if (lane == 0) report(status, MSA_DEV_TIMEOUT);
        break;
      }
      if (it < 0) {  // no items left: an empty stage tells the consumers to stop
        if (lane == 0) {
          s_item[s][0] = -1;
          mbar_expect_tx(&full[s], 0u);
        }
        ++n;
        break;
      }
      if (sub == 0) {
        // the item's query rows, once the consumers are done with the last item's
        if (items > 0 &&
            !__all_sync(0xffffffffu, mbar_wait(&qempty, (uint32_t)(items - 1) & 1u))) {
          if (lane == 0) report(status, MSA_DEV_TIMEOUT);
          break;
        }
        if (lane == 0) {
          mbar_expect_tx(&qfull, q_bytes);
          bulk_load_1d(qraw, q + ((size_t)cur_b * hq + (size_t)cur_gs * hg * G) * D, q_bytes,
                       &qfull);
        }
        ++items;
      }
      bool valid = false;
      if (pg != kNoCand) {
        if (pg < 0 || pg >= num_pages) report(status, MSA_DEV_BAD_PAGE);
        else valid = MSA_RANGE_OK((size_t)lane * pstride, (size_t)lane * pstride + page_bytes,
                                  stage_bytes, status);
      }
      const uint32_t vb = __ballot_sync(0xffffffffu, valid);
      unsigned char* st = smem_raw + (size_t)s * stage_bytes;
      if (lane == 0) {
        s_valid[s] = vb;
        s_item[s][0] = cur_b;
        s_item[s][1] = cur_c;
        s_item[s][2] = cur_gs;
        mbar_expect_tx(&full[s], (uint32_t)__popc(vb) * page_bytes);
      }
      __syncwarp();
      if (valid)
        bulk_load_1d(st + (size_t)lane * pstride,
                     centroids + ((size_t)pg * hkv + (size_t)cur_gs * hg) * D, page_bytes, &full[s]);
      if (++sub == KPL) {
        sub = 0;
        it += gridDim.x;
        if (it >= total_items) it = -1;
      }
      pg = it >= 0 ? fetch(it, sub) : kNoCand;
    }
    // every copy issued has landed before the CTA may end
    for (int m = n - NST < 0 ? 0 : n - NST; m < n; ++m)
      (void)mbar_wait(&full[m % NST], (uint32_t)(m / NST) & 1u);
    if (items > 0) (void)mbar_wait(&qfull, (uint32_t)(items - 1) & 1u);
    return;
  }

  // ------------------------------- consumers -------------------------------
  const int my_g = tid / SC, my_k = tid - (tid / SC) * SC;
  const bool active = my_g < hg;
  int n = 0, items = 0;
#pragma unroll 1
  for (;;) {
    uint64_t keys[KPL];
    int b = 0, c = 0, gs = 0;
    bool done = false;
    const float* qbar = qbar2 + (items & 1) * hg * D;
#pragma unroll
    for (int sub = 0; sub < KPL; ++sub, ++n) {
      const int s = n % NST;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (uint32_t)(n / NST) & 1u))) {
        if (lane == 0) report(status, MSA_DEV_TIMEOUT);
        return;
      }
      b = s_item[s][0];
      if (b < 0) {  // the producer ran out of items (only at an item boundary)
        done = true;
        break;
      }
      c = s_item[s][1];
      gs = s_item[s][2];
      if (sub == 0) {
        // the item's qbar: each group's G heads summed left to right in fp32
        if (!__all_sync(0xffffffffu, mbar_wait(&qfull, (uint32_t)items & 1u))) {
          if (lane == 0) report(status, MSA_DEV_TIMEOUT);
          return;
        }
        float* qb_w = qbar2 + (items & 1) * hg * D;
        for (int x = tid; x < hg * D; x += kPass1Threads) {
          const int gl = x / D, i = x - gl * D;
          const T* src = qraw + (size_t)gl * G * D + i;
          float a = to_f32(src[0]);
          for (int h = 1; h < G; ++h) a = __fadd_rn(a, to_f32(src[(size_t)h * D]));
          qb_w[x] = a;
        }
        // every consumer has its qbar (a bounded mbarrier wait, not bar.sync:
        // a consumer that gave up on a wait must not leave the others stuck),
        // and the raw rows may be replaced
        mbar_arrive(&qready);
        if (!__all_sync(0xffffffffu, mbar_wait(&qready, (uint32_t)items & 1u))) {
          if (lane == 0) report(status, MSA_DEV_TIMEOUT);
          return;
        }
        if (lane == 0) mbar_arrive(&qempty);
        ++items;
      }
      uint64_t key = 0ull;
      if (active && ((s_valid[s] >> my_k) & 1u)) {
        const unsigned char* st = smem_raw + (size_t)s * stage_bytes;
        const float4* cr = reinterpret_cast<const float4*>(st + (size_t)my_k * pstride +
                                                           (size_t)my_g * D * 4);
        const float4* qb = reinterpret_cast<const float4*>(qbar + (size_t)my_g * D);
        float acc = 0.f;
#pragma unroll
        for (int x = 0; x < D / 4; ++x) {
          const float4 cv = cr[x];
          const float4 qv = qb[x];
          acc = __fmaf_rn(qv.x, cv.x, acc);
          acc = __fmaf_rn(qv.y, cv.y, acc);
          acc = __fmaf_rn(qv.z, cv.z, acc);
          acc = __fmaf_rn(qv.w, cv.w, acc);
        }
        key = sel_key(acc, cand_lo + c * kDecChunk + sub * SC + my_k);
      }
      keys[sub] = key;
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (done) break;
    // bitonic sort (descending) of the group's 64 keys: element e = my_k * KPL + r
#pragma unroll
    for (int size = 2; size <= kDecChunk; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        if (stride >= KPL) {
#pragma unroll
          for (int r = 0; r < KPL; ++r) {
            const int e = my_k * KPL + r;
            const uint64_t o = shfl_xor_u64(keys[r], stride / KPL);
            const bool take_max = ((e & stride) == 0) == ((e & size) == 0);
            keys[r] = take_max ? (keys[r] > o ? keys[r] : o) : (keys[r] < o ? keys[r] : o);
          }
        } else {
#pragma unroll
          for (int r = 0; r < KPL; ++r) {
            if ((r & stride) == 0) {
              const int e = my_k * KPL + r;
              const uint64_t x0 = keys[r], x1 = keys[r + stride];
              const bool desc = (e & size) == 0;
              const bool swap = desc ? (x0 < x1) : (x0 > x1);
              keys[r] = swap ? x1 : x0;
              keys[r + stride] = swap ? x0 : x1;
            }
          }
        }
      }
    }
    if (active && MSA_IN_BOUNDS(b, batch, status) && MSA_IN_BOUNDS(c, nchunks, status)) {
      uint64_t* out = ws + (((size_t)b * hkv + gs * hg + my_g) * nchunks + c) * kw;
#pragma unroll
      for (int r = 0; r < KPL; ++r) {
        const int e = my_k * KPL + r;
        if (e < kw) out[e] = keys[r];
      }
    }
  }
  pdl_release();
}

__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int src) {
  const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)v, src);
  const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(v >> 32), src);
  return ((uint64_t)hi << 32) | lo;
}

// Top 32 of two descending lists held one key per lane (lane l = rank l):
// the elementwise max of one list and the other reversed is bitonic and holds
// the top 32 of both; five half-cleaner steps sort it, descending.
__device__ __forceinline__ uint64_t warp_merge_top32(uint64_t a, uint64_t b, int lane) {
  const uint64_t r = shfl_u64(b, 31 - lane);
  uint64_t x = a > r ? a : r;
#pragma unroll
  for (int st = 16; st > 0; st >>= 1) {
    const uint64_t o = shfl_xor_u64(x, st);
    x = ((lane & st) == 0) ? (x > o ? x : o) : (x < o ? x : o);
  }
  return x;
}

// Top 64 of two descending lists held two keys per lane (x[0] = rank l,
// x[1] = rank l + 32): reverse + max is bitonic; the stride-32 step is inside
// the lane, strides 16..1 are shuffles on each register.
__device__ __forceinline__ void warp_merge_top64(uint64_t (&a)[2], const uint64_t (&b)[2],
                                                 int lane) {
  const uint64_t r0 = shfl_u64(b[1], 31 - lane), r1 = shfl_u64(b[0], 31 - lane);
  uint64_t x0 = a[0] > r0 ? a[0] : r0, x1 = a[1] > r1 ? a[1] : r1;
  const uint64_t hi = x0 > x1 ? x0 : x1, lo = x0 > x1 ? x1 : x0;
  x0 = hi;
  x1 = lo;
#pragma unroll
  for (int st = 16; st > 0; st >>= 1) {
    const uint64_t o0 = shfl_xor_u64(x0, st), o1 = shfl_xor_u64(x1, st);
    const bool up = (lane & st) == 0;
    x0 = up ? (x0 > o0 ? x0 : o0) : (x0 < o0 ? x0 : o0);
    x1 = up ? (x1 > o1 ? x1 : o1) : (x1 < o1 ? x1 : o1);
  }
  a[0] = x0;
  a[1] = x1;
}

template <int NK>
__device__ __forceinline__ void warp_merge_top(uint64_t (&a)[NK], const uint64_t (&b)[NK], int lane) {
  if constexpr (NK == 1) a[0] = warp_merge_top32(a[0], b[0], lane);
  else warp_merge_top64(a, b, lane);
}

// Pass 2 for kw <= 32 * NK: a CTA of four warps per (sequence, group). A chunk
// list is held NK keys per lane (rank lane + 32 r in register r; coalesced
// loads); each warp loads LG lists at once and merges them as a balanced tree
// into its running top 32·NK, warp 0 merges the four warps' lists, and a
// bitonic sort on the block index (NK elements per lane) gives the ascending
// output.
// The same kernel merges (a) the chunk lists of one sequence's candidates in
// [cand_lo, cand_hi) (nlists = 0: one list per chunk of 64 candidates, list c
// of (b, g) at ws + ((b * hkv + g) * nchunks + c) * kw), or (b) nlists lists
// gathered from the ranks of a context-sharded decode (list c of (b, g) at
// ws + ((c * batch + b) * hkv + g) * kw). With keys_out it writes the best
// min(k-1, candidates) keys of each (b, g), descending, 0 padded to top_k - 1,
// instead of the ascending block list.
template <int NK, int LG>
__global__ void __launch_bounds__(128) select_decode_merge(
    const uint64_t* __restrict__ ws, const int32_t* __restrict__ seq_lens, int batch, int hkv,
    int B, int max_blocks, int kw, int nchunks, int top_k, int nlists, int cand_lo, int cand_hi,
    int32_t* __restrict__ idx, float* __restrict__ score, uint64_t* __restrict__ keys_out) {
  __shared__ uint64_t part[4][32 * NK];
  pdl_wait();
  const int g = blockIdx.x, b = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int L = seq_lens[b];
  const size_t outo = ((size_t)b * hkv + g) * top_k;
  if (L < 1 || L > max_blocks * B) return;  // reported by pass 1
  const int own = (L - 1) / B;
  const int ncand = max(0, min(own, cand_hi) - cand_lo);
  const int keep = min(top_k - 1, ncand);
  const int nch = nlists > 0 ? nlists : (ncand + kDecChunk - 1) / kDecChunk;
  const uint64_t* src = nlists > 0 ? ws + ((size_t)b * hkv + g) * kw
                                   : ws + ((size_t)b * hkv + g) * nchunks * kw;
  const size_t lstride = nlists > 0 ? (size_t)batch * hkv * kw : (size_t)kw;
  uint64_t acc[NK];
#pragma unroll
  for (int r = 0; r < NK; ++r) acc[r] = 0ull;
  for (int c0 = warp * LG; c0 < nch; c0 += 4 * LG) {
    uint64_t l[LG][NK];
#pragma unroll
    for (int u = 0; u < LG; ++u) {
      const int c = c0 + u;
#pragma unroll
      for (int r = 0; r < NK; ++r) {
        const int i = lane + 32 * r;
        l[u][r] = (c < nch && i < kw) ? src[(size_t)c * lstride + i] : 0ull;
      }
    }
#pragma unroll
    for (int w = 1; w < LG; w <<= 1) {
#pragma unroll
      for (int u = 0; u < LG; u += 2 * w) warp_merge_top<NK>(l[u], l[u + w], lane);
    }
    warp_merge_top<NK>(acc, l[0], lane);
  }
#pragma unroll
  for (int r = 0; r < NK; ++r) part[warp][lane + 32 * r] = acc[r];
  __syncthreads();
  if (warp != 0) return;
  uint64_t m0[NK], m1[NK], m2[NK], m3[NK];
#pragma unroll
  for (int r = 0; r < NK; ++r) {
    m0[r] = part[0][lane + 32 * r];
    m1[r] = part[1][lane + 32 * r];
    m2[r] = part[2][lane + 32 * r];
    m3[r] = part[3][lane + 32 * r];
  }
  warp_merge_top<NK>(m0, m1, lane);
  warp_merge_top<NK>(m2, m3, lane);
  warp_merge_top<NK>(m0, m2, lane);
  if (keys_out) {  // the best keys themselves, descending
    uint64_t* ko = keys_out + ((size_t)b * hkv + g) * (top_k - 1);
#pragma unroll
    for (int r = 0; r < NK; ++r) {
      const int e = lane + 32 * r;
      if (e < top_k - 1) ko[e] = e < keep ? m0[r] : 0ull;
    }
    pdl_release();
    return;
  }
  // element e = lane + 32 r holds rank e; sort the first `keep` by block index
  int blk[NK];
  float sc[NK];
  int cnt = 0;
#pragma unroll
  for (int r = 0; r < NK; ++r) {
    const bool real = lane + 32 * r < keep && m0[r] != 0ull;
    cnt += __popc(__ballot_sync(0xffffffffu, real));  // fewer if pages were bad
    blk[r] = real ? key_block(m0[r]) : 0x7fffffff;
    sc[r] = key_score(m0[r]);
  }
#pragma unroll
  for (int size = 2; size <= 32 * NK; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (stride == 32) {  // NK == 2, size 64: both elements in this lane, ascending
        if (blk[0] > blk[NK - 1]) {
          const int tb = blk[0];
          const float ts = sc[0];
          blk[0] = blk[NK - 1];
          sc[0] = sc[NK - 1];
          blk[NK - 1] = tb;
          sc[NK - 1] = ts;
        }
        continue;
      }
#pragma unroll
      for (int r = 0; r < NK; ++r) {
        const int e = lane + 32 * r;
        const int ob = __shfl_xor_sync(0xffffffffu, blk[r], stride);
        const float os = __shfl_xor_sync(0xffffffffu, sc[r], stride);
        const bool take_min = ((e & stride) == 0) == ((e & size) == 0);
        if (take_min ? (ob < blk[r]) : (ob > blk[r])) {
          blk[r] = ob;
          sc[r] = os;
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < NK; ++r) {
    const int e = lane + 32 * r;
    if (e < cnt) {
      idx[outo + e] = blk[r];
      if (score) score[outo + e] = sc[r];
    }
  }
  if (lane == 0) {
    idx[outo + cnt] = own;
    if (score) score[outo + cnt] = __int_as_float(0x7f800000);
  }
  for (int s = cnt + 1 + lane; s < top_k; s += 32) {
    idx[outo + s] = -1;
    if (score) score[outo + s] = __int_as_float(0xff800000);
  }
  pdl_release();
}

// Pass 2: one warp per (sequence, group) merges the chunk lists, each already
// sorted by pass 1, with a tournament: every round the lanes offer the heads
// of their chunks, the warp maximum is taken (high then low 32 bits, keys are
// unique) and its chunk advances.
__global__ void __launch_bounds__(32) select_decode_pass2(
    const uint64_t* __restrict__ ws, const int32_t* __restrict__ seq_lens, int hkv, int B,
    int max_blocks, int kw, int nchunks, int top_k, int32_t* __restrict__ idx,
    float* __restrict__ score) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  uint64_t* lists = reinterpret_cast<uint64_t*>(smem_raw);  // [nch][kw]
  __shared__ uint64_t chosen[256];
  pdl_wait();
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
  for (int i0 = 0; i0 < total; i0 += 32 * 32) {  // up to 32 loads per lane in flight
    uint64_t v[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      const int i = i0 + u * 32 + lane;
      v[u] = i < total ? src[i] : 0ull;
    }
#pragma unroll
    for (int u = 0; u < 32; ++u) {
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
  const int lane_chunks = (nch + 31) / 32;
  for (; cnt < keep; ++cnt) {
    uint64_t best = head[0];
#pragma unroll
    for (int s = 1; s < kMaxChunksPerLane; ++s)
      if (s < lane_chunks) best = head[s] > best ? head[s] : best;
    const uint32_t bhi = (uint32_t)(best >> 32), blo = (uint32_t)best;
    const uint32_t whi = __reduce_max_sync(0xffffffffu, bhi);
    const uint32_t wlo = __reduce_max_sync(0xffffffffu, bhi == whi ? blo : 0u);
    const uint64_t wb = ((uint64_t)whi << 32) | wlo;
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
  pdl_release();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int kmax_for(int top_k) { return top_k - 1 <= 16 ? 16 : (top_k - 1 <= 32 ? 32 : 64); }

static size_t rows_smem(int D, int kmax) {
  const size_t chunk = (size_t)kChunk * (D + 4) * 4 + (size_t)kRows * kChunk * 4;
  const size_t lists = (size_t)kRows * (256 / kRows) * kmax * 8;
  return (size_t)kRows * D * 4 + (chunk > lists ? chunk : lists);
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

static int decode_nchunks(const msa_paged_kv_t* kv) {
  return (kv->max_blocks_per_seq + kDecChunk - 1) / kDecChunk;
}
static int decode_kw(int top_k) { return top_k - 1 < kDecChunk ? (top_k - 1 < 1 ? 1 : top_k - 1) : kDecChunk; }

static int device_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// KV groups per pass-1 item: the largest divisor of hkv up to 8 that still
// makes about two items per SM (from the page-table width, an upper bound of
// the chunks); a small batch gets fewer groups per item, hence more items
// (one 1M-token sequence: 2 of 8 groups, 512 items instead of 128).
static int pass1_groups(const msa_paged_kv_t* kv) {
  const int hkv = kv->num_kv_heads;
  const long chunks = (long)kv->batch * decode_nchunks(kv);
  const long target = 2L * device_sms();
  int smallest = hkv;
  for (int d = hkv < 8 ? hkv : 8; d >= 1; --d) {
    if (hkv % d) continue;
    if (chunks * (hkv / d) >= target) return d;
    if (d >= 2) smallest = d;
  }
  return hkv == 1 ? 1 : smallest;
}
static size_t pass1_smem(const msa_paged_kv_t* kv, int nst) {
  const int hg = pass1_groups(kv), D = kv->head_dim;
  const size_t esz = kv->dtype == MSA_DTYPE_BF16 ? 2 : 4;
  const size_t G = (size_t)(kv->num_q_heads / kv->num_kv_heads);
  return (size_t)nst * pass1_stage_bytes(hg, D) + (size_t)hg * G * D * esz +
         (size_t)2 * hg * D * 4 + (size_t)(2 * kv->batch + 1) * 4;
}
constexpr size_t kSmemLimit = 227 * 1024 - 1024;  // dynamic + static, per CTA
// three stages where they fit (steps of up to 8 candidates), else two
static int pass1_stages(const msa_paged_kv_t* kv) {
  const int kpl = kDecChunk / pass1_sc(pass1_groups(kv));
  if (kpl <= 8 && pass1_smem(kv, 3) <= kSmemLimit) return 3;
  return pass1_smem(kv, 2) <= kSmemLimit ? 2 : 0;
}

// decode selection merges at most 32 * kMaxChunksPerLane chunk lists of
// kDecChunk candidates
bool select_decode_supported(const msa_paged_kv_t* kv) {
  return kv->batch <= 65535 && kv->max_blocks_per_seq <= 32 * kMaxChunksPerLane * kDecChunk &&
         kv->num_kv_heads <= kPass1Threads / 2 && pass1_stages(kv) > 0;
}

// workspace: chunk lists [batch][hkv][nchunks][kw] u64
static size_t decode_lists_bytes(const msa_paged_kv_t* kv, int top_k) {
  const size_t b = (size_t)kv->batch * kv->num_kv_heads * decode_nchunks(kv) * decode_kw(top_k) * 8;
  return (b + 255) & ~(size_t)255;
}
size_t select_decode_ws(const msa_paged_kv_t* kv, int top_k) {
  return decode_lists_bytes(kv, top_k) + 256;
}

// Resident pass-1 CTAs on the whole device, cached per (device, smem size).
static int pass1_slots(const void* fn, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, size_t>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  const auto key = std::make_tuple(dev, fn, smem);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int per_sm = 0, sms = 148;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kPass1Threads + 32, smem) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int slots = per_sm * (sms > 0 ? sms : 148);
  cache.emplace(key, slots);
  return slots;
}

template <typename T, int D, int KPL, int NST>
static cudaError_t launch_pass1(const msa_paged_kv_t* kv, const void* q, int kw, int nch,
                                uint64_t* lists, int cand_lo, int cand_hi, cudaStream_t st) {
  const size_t smem = pass1_smem(kv, NST);
  auto k1 = select_decode_pass1<T, D, KPL, NST>;
  cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int hg = pass1_groups(kv);
  const long upper = (long)kv->batch * nch * (kv->num_kv_heads / hg);
  const int grid = (int)std::max(1L, std::min<long>(upper, pass1_slots((const void*)k1, smem)));
  return launch_pdl(k1, dim3(grid), dim3(kPass1Threads + 32), smem, st, (const T*)q,
                    (const float*)kv->centroids, (const int32_t*)kv->page_table,
                    (const int32_t*)kv->seq_lens, kv->status_word, kv->batch, kv->num_q_heads,
                    kv->num_kv_heads, hg, kv->block_size, kv->num_pages, kv->max_blocks_per_seq, kw,
                    nch, cand_lo, cand_hi, lists);
}

template <typename T, int D, int NST>
static cudaError_t pass1_dispatch_k(const msa_paged_kv_t* kv, const void* q, int kw, int nch,
                                    uint64_t* lists, int lo, int hi, cudaStream_t st) {
  switch (kDecChunk / pass1_sc(pass1_groups(kv))) {
    case 2: return launch_pass1<T, D, 2, NST>(kv, q, kw, nch, lists, lo, hi, st);
    case 4: return launch_pass1<T, D, 4, NST>(kv, q, kw, nch, lists, lo, hi, st);
    case 8: return launch_pass1<T, D, 8, NST>(kv, q, kw, nch, lists, lo, hi, st);
    case 16: return launch_pass1<T, D, 16, 2>(kv, q, kw, nch, lists, lo, hi, st);
    default: return launch_pass1<T, D, 32, 2>(kv, q, kw, nch, lists, lo, hi, st);
  }
}

// Merge launch: kw <= 32 and <= 64 keys per list use the merge tree; longer
// lists (only for the per-sequence chunk lists) use the tournament.
static cudaError_t launch_merge(const msa_paged_kv_t* kv, const uint64_t* lists, int kw, int nch,
                                int top_k, int nlists, int lo, int hi, int32_t* idx, float* score,
                                uint64_t* keys_out, cudaStream_t st) {
  dim3 g2(kv->num_kv_heads, kv->batch);
  const int32_t* sl = kv->seq_lens;
  const int hkv = kv->num_kv_heads, B = kv->block_size, mb = kv->max_blocks_per_seq;
  const int nl = nlists > 0 ? nlists : nch;
  // lists per warp and round: enough that the four warps take them in one round
  const int lg = nl <= 32 ? 8 : (nl <= 64 ? 16 : 32);
  if (kw <= 32) {
    auto k = lg == 8 ? select_decode_merge<1, 8>
                     : (lg == 16 ? select_decode_merge<1, 16> : select_decode_merge<1, 32>);
    return launch_pdl(k, g2, dim3(128), 0, st, lists, sl, kv->batch, hkv, B, mb, kw, nch, top_k,
                      nlists, lo, hi, idx, score, keys_out);
  }
  auto k = lg == 8 ? select_decode_merge<2, 8> : select_decode_merge<2, 16>;
  return launch_pdl(k, g2, dim3(128), 0, st, lists, sl, kv->batch, hkv, B, mb, kw, nch, top_k,
                    nlists, lo, hi, idx, score, keys_out);
}

template <typename T, int D>
static cudaError_t launch_decode_sel(const msa_paged_kv_t* kv, const void* q, int top_k,
                                     int32_t* idx, float* score, void* ws, int lo, int hi,
                                     uint64_t* keys_out, cudaStream_t st) {
  const int nch = decode_nchunks(kv), kw = decode_kw(top_k);
  uint64_t* lists = (uint64_t*)ws;
  cudaError_t e = pass1_stages(kv) == 3
                      ? pass1_dispatch_k<T, D, 3>(kv, q, kw, nch, lists, lo, hi, st)
                      : pass1_dispatch_k<T, D, 2>(kv, q, kw, nch, lists, lo, hi, st);
  if (e != cudaSuccess) return e;
  if (top_k - 1 <= 64)
    return launch_merge(kv, lists, kw, nch, top_k, 0, lo, hi, idx, score, keys_out, st);
  const size_t smem2 = (size_t)nch * kw * 8;
  e = cudaFuncSetAttribute(select_decode_pass2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem2);
  if (e != cudaSuccess) return e;
  dim3 g2(kv->num_kv_heads, kv->batch);
  return launch_pdl(select_decode_pass2, g2, dim3(32), smem2, st, (const uint64_t*)lists,
                    (const int32_t*)kv->seq_lens, kv->num_kv_heads, kv->block_size,
                    kv->max_blocks_per_seq, kw, nch, top_k, idx, score);
}

static cudaError_t decode_sel_any(const msa_paged_kv_t* kv, const void* q, int top_k, int32_t* idx,
                                  float* score, void* ws, int lo, int hi, uint64_t* keys_out,
                                  cudaStream_t st) {
  const bool bf = kv->dtype == MSA_DTYPE_BF16;
  if (kv->head_dim == 128)
    return bf ? launch_decode_sel<bf16, 128>(kv, q, top_k, idx, score, ws, lo, hi, keys_out, st)
              : launch_decode_sel<float, 128>(kv, q, top_k, idx, score, ws, lo, hi, keys_out, st);
  return bf ? launch_decode_sel<bf16, 64>(kv, q, top_k, idx, score, ws, lo, hi, keys_out, st)
            : launch_decode_sel<float, 64>(kv, q, top_k, idx, score, ws, lo, hi, keys_out, st);
}

cudaError_t select_decode(const msa_paged_kv_t* kv, const void* q, int top_k, int32_t* idx,
                          float* score, void* ws, cudaStream_t st) {
  return decode_sel_any(kv, q, top_k, idx, score, ws, 0, 0x7fffffff, nullptr, st);
}

// Context-sharded decode: this rank's best keys among candidates [lo, hi).
cudaError_t select_decode_range(const msa_paged_kv_t* kv, const void* q, int top_k, int lo, int hi,
                                uint64_t* keys_out, void* ws, cudaStream_t st) {
  return decode_sel_any(kv, q, top_k, nullptr, nullptr, ws, lo, hi, keys_out, st);
}

// Context-sharded decode: the global selection from nlists gathered key lists.
cudaError_t select_merge_lists(const msa_paged_kv_t* kv, const uint64_t* keys, int nlists,
                               int top_k, int32_t* idx, float* score, cudaStream_t st) {
  return launch_merge(kv, keys, top_k - 1, 0, top_k, nlists, 0, 0x7fffffff, idx, score, nullptr,
                      st);
}

}  // namespace msa
