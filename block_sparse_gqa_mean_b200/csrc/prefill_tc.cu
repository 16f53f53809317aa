// Sparse prefill attention on the 5th-generation tensor cores (tcgen05, TMEM).
//
// "MiniMax Sparse Attention" (staik.se), method and results paragraphs: exact
// blockwise sparse attention over the selected blocks, made fast by keeping
// the tensor cores busy; "Gated Sparse Attention: An Architectural Evolution
// for Long-Context LLMs", section 4: sparse patterns are mapped onto dense
// block matrix operations and the kernels skip the work that is masked out.
//
// Work unit: a query tile of TM = 128 / G consecutive tokens of one sequence
// and one KV group, i.e. 128 query rows (token-major, the group's G heads per
// token). The tile's tokens select their blocks independently, so the tile
// walks the UNION of their selections (built by prefill_plan_kernel,
// ascending, each entry carrying one bit per token). Per union block the CTA
// computes S = Q K^T for all 128 rows on the tensor cores and the softmax
// gives zero weight to the rows of tokens that did not select the block.
//
// CTA layout (192 threads): warp 0 issues TMA loads of K and V tiles (two
// 64-column boxes each, 128-byte swizzle, no multicast) into a ring of
// stages; warp 1 owns the TMEM allocation and issues tcgen05.mma from one
// thread; warps 2..5 are the softmax warps, one TMEM lane (query row) per
// thread.
//   TMEM columns : Q (bf16 pairs, 64) | P0 | P1 (bf16 pairs, 64 each) |
//                  S (fp32, 128) | O (fp32, 128)
// The row sums l are kept in the softmax threads' registers, summed over the
// same bf16-rounded weights that P V uses (an extra row-sum MMA was measured
// to cost the tensor pipe more than the adds cost the softmax).
//   S = Q K^T    : M=128, N=B, K=128, A = Q (TMEM), B = K tile (K-major SW128)
//   O += P V     : M=128, N=128, K=B, A = P (TMEM), B = V tile (MN-major SW128)
// The softmax reads S into registers at once and releases it, so the tensor
// cores compute S for block e+1 while the exponentials of block e run; P is
// double-buffered and the softmax reference max moves lazily (only when a
// row's max grows by more than 2^8), so writing P never waits for the P V in
// flight and O is rescaled in TMEM only rarely.
#include "tc.cuh"

namespace msa {

namespace {

constexpr int kD = 128;
constexpr float kLog2e = 1.4426950408889634f;

}  // namespace

// ---------------------------------------------------------------------------
// Token order. The query rows of a sequence are taken in windows of kWin rows;
// per window and KV group the tokens are dealt into the window's tiles (TM
// tokens each) greedily: a tile starts from the lowest-indexed token not yet
// placed and grows by the tokens whose usable blocks add the fewest new blocks
// to the tile's union (two per step; ties: the lower index). Tokens that
// selected the same blocks then share a tile, so the union a tile walks
// shrinks (on the prefill workload from 64 to 54 blocks per 16-token tile;
// taking one token per step gives 53.6, two 53.9). perm[window][g][p] is the
// window offset of the p-th token of the new order; the attention is the same
// for any order, only the work changes.
// ---------------------------------------------------------------------------
constexpr int kWin = 128;

constexpr int kClusterK = 16;  // block lists of up to 16 entries are clustered (in registers)

// one CTA per region (window, group), a thread per token
__global__ void __launch_bounds__(kWin) prefill_cluster_kernel(
    const int32_t* __restrict__ cu_q, const int32_t* __restrict__ seq_lens,
    const int32_t* __restrict__ block_idx, int hkv, int B, int max_blocks, int top_k, int TM,
    int wps, uint8_t* __restrict__ perm) {
  extern __shared__ uint32_t cur[];  // union bitmap of the tile being built
  __shared__ unsigned s_red[2 * (kWin / 32)];
  const int region = blockIdx.x;
  const int g = region % hkv;
  const int w = (region / hkv) % wps;
  const int b = region / (hkv * wps);
  const int tid = threadIdx.x;
  const int row0 = cu_q[b];
  const int n_rows = cu_q[b + 1] - row0;
  const int r_lo = w * kWin;
  if (r_lo >= n_rows) return;
  const int nw = min(kWin, n_rows - r_lo);
  uint8_t* pw = perm + (size_t)region * kWin;
  const int L = seq_lens[b];
  if (n_rows > L || L > max_blocks * B || top_k > kClusterK) {  // identity order
    if (tid < nw) pw[tid] = (uint8_t)tid;
    return;
  }
  const int t0 = L - n_rows + r_lo;
  int my[kClusterK];
#pragma unroll
  for (int s = 0; s < kClusterK; ++s) {
    int j = -1;
    if (tid < nw && s < top_k) {
      j = block_idx[((size_t)(row0 + r_lo + tid) * hkv + g) * top_k + s];
      if (j > (t0 + tid) / B) j = -1;
    }
    my[s] = j;
  }
  const int rw = ((t0 + nw - 1) / B + 1 + 31) / 32;  // bitmap words of blocks 0 .. last own block
  bool placed = tid >= nw;
  // Each step places the two tokens with the smallest growth against the
  // tile's current union (one when the tile or the window has one slot left);
  // the seed step places the lowest unplaced token alone.
  for (int p = 0; p < nw;) {
    const bool seed = (p % TM) == 0;
    if (seed) {
      for (int i = tid; i < rw; i += kWin) cur[i] = 0u;
      __syncthreads();
    }
    const int take = seed ? 1 : min(2, min(TM - p % TM, nw - p));
    unsigned key = 0xffffffffu;
    if (!placed) {
      unsigned grow = 0;
      if (!seed) {
#pragma unroll
        for (int s = 0; s < kClusterK; ++s)
          if (my[s] >= 0) grow += ((cur[my[s] >> 5] >> (my[s] & 31)) & 1u) ^ 1u;
      }
      key = (grow << 8) | (unsigned)tid;  // unique: the thread index is in the low bits
    }
    const unsigned m1 = __reduce_min_sync(0xffffffffu, key);
    const unsigned m2 = __reduce_min_sync(0xffffffffu, key == m1 ? 0xffffffffu : key);
    if ((tid & 31) == 0) {
      s_red[2 * (tid >> 5)] = m1;
      s_red[2 * (tid >> 5) + 1] = m2;
    }
    __syncthreads();
    unsigned b1 = 0xffffffffu, b2 = 0xffffffffu;  // every thread: the two smallest of the warps'
#pragma unroll
    for (int k = 0; k < 2 * (kWin / 32); ++k) {
      const unsigned v = s_red[k];
      if (v < b1) {
        b2 = b1;
        b1 = v;
      } else if (v < b2) {
        b2 = v;
      }
    }
    const int best1 = (int)(b1 & 0xffu);
    const int best2 = (take == 2 && b2 != 0xffffffffu) ? (int)(b2 & 0xffu) : -1;
    if (tid == 0) {
      pw[p] = (uint8_t)best1;
      if (best2 >= 0) pw[p + 1] = (uint8_t)best2;
    }
    if (tid == best1 || tid == best2) {
      placed = true;
#pragma unroll
      for (int s = 0; s < kClusterK; ++s)
        if (my[s] >= 0) atomicOr(&cur[my[s] >> 5], 1u << (my[s] & 31));
    }
    __syncthreads();
    p += best2 >= 0 ? 2 : 1;
  }
}

// ---------------------------------------------------------------------------
// Planning: for each query tile (TM tokens in the window order above), the
// union of the tokens' selections, ascending, each block with a 32-bit mask:
// bit i is set when the tile's token i selected the block.
// ---------------------------------------------------------------------------
constexpr int kPlanWindow = 4096;

__global__ void __launch_bounds__(128) prefill_plan_kernel(
    const int32_t* __restrict__ cu_q, const int32_t* __restrict__ seq_lens,
    const int32_t* __restrict__ block_idx, uint32_t* status, int hkv, int B, int max_blocks,
    int top_k, int TM, int units_per_seq, int wps, const uint8_t* __restrict__ perm, int ecap,
    int2* __restrict__ entries, int* __restrict__ counts) {
  __shared__ uint32_t bm[kPlanWindow];
  __shared__ int warp_tot[4];
  __shared__ int s_base;
  const int tile = blockIdx.x;  // unit index
  const int g = tile % hkv;
  const int tt = (tile / hkv) % units_per_seq;
  const int b = tile / (hkv * units_per_seq);
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int row0 = cu_q[b];
  const int n_rows = cu_q[b + 1] - row0;
  const int r_lo = tt * TM;
  // the sequence's rows lie inside q / block_idx, and the tiles cover all of them
  if (tt == 0 && g == 0 && tid == 0)
    (void)MSA_RANGE_OK(n_rows, n_rows, units_per_seq * TM, status);
  if (r_lo >= n_rows ||
      !MSA_RANGE_OK(row0, row0 + n_rows, cu_q[gridDim.x / (hkv * units_per_seq)], status)) {
    if (tid == 0) counts[tile] = 0;
    return;
  }
  const int w = r_lo / kWin;                      // window, and the tile's first order position
  const int p0 = r_lo % kWin;
  const int nw = min(kWin, n_rows - w * kWin);
  const int nr = min(TM, nw - p0);
  const uint8_t* pw = perm + ((size_t)(b * wps + w) * hkv + g) * kWin;
  const int L = seq_lens[b];
  if (n_rows > L || L > max_blocks * B) {
    if (tid == 0) {
      counts[tile] = 0;
      report(status, MSA_DEV_BAD_LENGTH);
    }
    return;
  }
  const int t_win = L - n_rows + w * kWin;       // position of the window's first row
  const int own_max = (t_win + nw - 1) / B;
  const int R = own_max + 1;
  int2* out = entries + (size_t)tile * ecap;
  if (tid == 0) s_base = 0;
  for (int w0 = 0; w0 < R; w0 += kPlanWindow) {
    const int W = min(kPlanWindow, R - w0);
    for (int i = tid; i < W; i += 128) bm[i] = 0u;
    __syncthreads();
    for (int it = tid; it < nr * top_k; it += 128) {
      const int i = it / top_k, s = it % top_k;
      const int o = pw[p0 + i];                     // the token's offset in its window
      if (!MSA_IN_BOUNDS(o, nw, status)) continue;
      const int j = block_idx[((size_t)(row0 + w * kWin + o) * hkv + g) * top_k + s];
      if (j < 0) continue;
      const int own_i = (t_win + o) / B;
      if (j > own_i) {
        report(status, MSA_DEV_BAD_INDEX);
        continue;
      }
      if (j >= w0 && j < w0 + W) atomicOr(&bm[j - w0], 1u << i);
    }
    __syncthreads();
    // compaction: thread tid scans words [tid*per, (tid+1)*per)
    const int per = (W + 127) / 128;
    const int a0 = min(W, tid * per), a1 = min(W, a0 + per);
    int cnt = 0;
    for (int a = a0; a < a1; ++a) cnt += bm[a] != 0u;
    int incl = cnt;
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int off = s_base + incl - cnt;
    for (int w = 0; w < warp; ++w) off += warp_tot[w];
    for (int a = a0; a < a1; ++a)
      if (bm[a] != 0u) {
        if (MSA_IN_BOUNDS(off, ecap, status)) out[off] = make_int2(w0 + a, (int)bm[a]);
        ++off;
      }
    __syncthreads();
    if (tid == 0) s_base += warp_tot[0] + warp_tot[1] + warp_tot[2] + warp_tot[3];
    __syncthreads();
  }
  if (tid == 0) counts[tile] = MSA_RANGE_OK(s_base, s_base, ecap, status) ? s_base : 0;
}

// ---------------------------------------------------------------------------
// Attention
// ---------------------------------------------------------------------------
constexpr float kRescaleLog2 = 8.f;  // lazy rescale threshold (log2 units)


// 2 NP scores -> NP bf16 pairs P = exp2(s * c - m) and their fp32 sum (of the
// rounded values) added into lsum2 (two partial sums). One pair in four on
// the FMA pipe, the rest on MUFU.
template <int NP>
__device__ __forceinline__ void exp_pack(const float* s, uint64_t sl2, uint64_t neg_m,
                                         uint32_t (&pv)[NP], uint64_t& lsum2) {
#pragma unroll
  for (int xx = 0; xx < NP; ++xx) {
    const uint64_t arg = f2_fma(f2_pack(s[2 * xx], s[2 * xx + 1]), sl2, neg_m);
    if ((xx & 3) == 0) {
      float p0, p1;
      exp2_poly_pair(arg, p0, p1);
      pv[xx] = pack_bf16(p0, p1);
    } else {
      pv[xx] = pack_bf16(fast_exp2(__uint_as_float((uint32_t)arg)),
                         fast_exp2(__uint_as_float((uint32_t)(arg >> 32))));
    }
    // the rounded pair, widened back to fp32, into the row sum
    lsum2 = f2_add(lsum2, ((uint64_t)(pv[xx] & 0xffff0000u) << 32) | (uint64_t)(pv[xx] << 16));
  }
}

// 16 lanes x 2N columns in two halves: thread t < 16 reads lane (base + t),
// columns 0..N-1 of the address; thread t >= 16 reads lane (base + t - 16),
// columns N..2N-1.
__device__ __forceinline__ void tc_ld16x2(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tc_ld16x2(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,"
      "%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,"
      "%61,%62,%63}, [%64], 64;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]),
        "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]),
        "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]),
        "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]),
        "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
}

// 16 lanes x 2N columns in two halves: thread t < 16 writes lane (base + t),
// columns 0..N-1; thread t >= 16 writes lane (base + t - 16), columns N..2N-1.
__device__ __forceinline__ void tc_st16x2(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], 16, {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tc_st16x2(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], 32, {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

template <int B, int G>
__global__ void __launch_bounds__(192, 1) prefill_tc_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const bf16* __restrict__ q, const int32_t* __restrict__ cu_q,
    const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens, uint32_t* status,
    int hq, int hkv, int num_pages, int max_blocks, int units_per_seq, int wps,
    const uint8_t* __restrict__ perm, int ecap,
    const int2* __restrict__ entries, const int* __restrict__ counts, float scale_log2,
    bf16* __restrict__ out, float* __restrict__ lse, gate_t gate) {
  constexpr int TM = 128 / G;              // tokens per query tile (128 rows)
  constexpr int NST = (B == 128) ? 3 : 4;  // K+V stages
  constexpr int TILE = B * kD * 2;         // bytes of a K (or V) tile
  constexpr int STAGE = 2 * TILE;
  constexpr uint32_t IDESC_S = idesc_bf16(128, B, false);
  constexpr uint32_t IDESC_O = idesc_bf16(128, kD, true);
  // TMEM columns
  constexpr uint32_t COL_Q = 0;    // Q, 64 columns (bf16 pairs), A operand of S = Q K^T
  constexpr uint32_t COL_P = 64;   // two P buffers of 64 columns (bf16 pairs)
  constexpr uint32_t COL_S = 192;  // S, 128 columns (fp32)
  constexpr uint32_t COL_O = 320;  // O, 128 columns (fp32)

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* stages = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t kv_full[NST], kv_empty[NST];
  __shared__ __align__(8) uint64_t s_full, s_free, p_full[2], o_done[2], q_ready, fin;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;

  const int unit = blockIdx.x;
  const int g = unit % hkv;
  const int pu = (unit / hkv) % units_per_seq;
  const int b = unit / (hkv * units_per_seq);
  int n_e = counts[unit];
  if (!MSA_RANGE_OK(n_e, n_e, ecap, status)) n_e = 0;
  const int2* ent = entries + (size_t)unit * ecap;
  const int row0 = cu_q[b];
  const int n_rows = cu_q[b + 1] - row0;
  const int r_lo = pu * TM;
  const int wdw = r_lo / kWin;                    // window of the tile, and its first order position
  const int p0 = r_lo % kWin;
  const int nw = min(kWin, n_rows - wdw * kWin);
  const int nr = min(TM, nw - p0);
  const uint8_t* pw = perm + ((size_t)(b * wps + wdw) * hkv + g) * kWin;
  const int L = seq_lens[b];
  const int t_win = L - n_rows + wdw * kWin;      // position of the window's first row
  const int row_win = row0 + wdw * kWin;          // global row of the window's first row
  // window offset of the tile's token ti (the order table is the library's own)
  auto tok_off = [&](int ti) {
    const int o = pw[p0 + ti];
    return MSA_IN_BOUNDS(o, nw, status) ? o : 0;
  };
  if (n_e == 0) {
    // no token of the tile took a block (or the tile lies past the sequence's
    // rows): its rows attend to nothing, A = 0. Uniform exit before any sync.
    if (threadIdx.x >= 64) {
      const int r = threadIdx.x - 64, ti = r / G, h = r % G;
      if (ti < nr) {
        const size_t head = ((size_t)row_win + tok_off(ti)) * hq + (size_t)g * G + h;
        for (int c = 0; c < kD; ++c)
          out[head * kD + c] = __float2bfloat16_rn(gate_apply<bf16>(gate, head, c, kD, 0.f));
        if (lse) lse[head] = -INFINITY;
      }
    }
    return;
  }

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(&s_full, 1);
    mbar_init(&s_free, 128);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&p_full[x], 128);
      mbar_init(&o_done[x], 1);
    }
    mbar_init(&q_ready, 128);
    mbar_init(&fin, 1);
    s_abort = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(&s_tmem))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued = 0;
      for (int e = 0; e < n_e && !s_abort; ++e) {
        const int st = e % NST;
        if (!mbar_wait(&kv_empty[st], ((e / NST) & 1) ^ 1)) {
          report(status, MSA_DEV_TIMEOUT);
          s_abort = 1;
          break;
        }
        const int j = ent[e].x;
        int pg = MSA_IN_BOUNDS(j, max_blocks, status) ? page_table[(size_t)b * max_blocks + j] : 0;
        if (pg < 0 || pg >= num_pages) {
          report(status, MSA_DEV_BAD_PAGE);
          pg = 0;  // keep the pipeline in step; the result of this unit is unspecified
        }
        const int y = (pg * hkv + g) * B;
        unsigned char* kt = stages + st * STAGE;
        mbar_expect_tx(&kv_full[st], STAGE);
        tma_load_2d(kt, &tm_k, &kv_full[st], 0, y);
        tma_load_2d(kt + TILE / 2, &tm_k, &kv_full[st], 64, y);
        tma_load_2d(kt + TILE, &tm_v, &kv_full[st], 0, y);
        tma_load_2d(kt + TILE + TILE / 2, &tm_v, &kv_full[st], 64, y);
        ++issued;
      }
      // every copy issued must have landed before the CTA may exit (bounded)
      for (int e = max(0, issued - NST); e < issued; ++e)
        if (!mbar_wait(&kv_full[e % NST], (e / NST) & 1)) report(status, MSA_DEV_TIMEOUT);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (one thread) ----------------
    if (lane == 0) {
      bool ok = mbar_wait(&q_ready, 0);
      tc_fence_after();
      // S_e = Q K_e^T, once block e is loaded and the softmax has read S_{e-1}
      auto issue_s = [&](int e) -> bool {
        const int st = e % NST;
        if (!mbar_wait(&kv_full[st], (e / NST) & 1)) return false;
        if (e >= 1 && !mbar_wait(&s_free, (e - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t kt = smem_u32(stages + st * STAGE);
#pragma unroll
        for (int ks = 0; ks < kD / 16; ++ks) {
          const uint32_t boff = (uint32_t)(ks >> 2) * (uint32_t)(TILE / 2) + (uint32_t)(ks & 3) * 32u;
          tc_mma_ts(tmem + COL_S, tmem + COL_Q + ks * 8, sdesc_sw128(kt + boff, 16, 1024),
                    IDESC_S, ks > 0);
        }
        tc_commit(&s_full);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int e = 0; e < n_e && ok && !s_abort; ++e) {
        if (e + 1 < n_e && !issue_s(e + 1)) { ok = false; break; }
        const int pb = e & 1;
        if (!mbar_wait(&p_full[pb], (e >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t vt = smem_u32(stages + (e % NST) * STAGE + TILE);
#pragma unroll
        for (int kk = 0; kk < B / 16; ++kk) {
          const uint32_t acc = (e > 0 || kk > 0) ? 1u : 0u;
          tc_mma_ts(tmem + COL_O, tmem + COL_P + pb * 64 + kk * 8,
                    sdesc_sw128(vt + (uint32_t)kk * 2048u, (uint32_t)(TILE / 2), 1024), IDESC_O, acc);
        }
        tc_commit(&o_done[pb]);
        tc_commit(&kv_empty[e % NST]);
      }
      if (!ok) {
        report(status, MSA_DEV_TIMEOUT);
        s_abort = 1;
      }
      // all MMAs issued by this thread complete before TMEM is released (bounded)
      tc_commit(&fin);
      if (!mbar_wait(&fin, 0)) report(status, MSA_DEV_TIMEOUT);
    }
  } else {
    // ---------------- softmax warps: a TMEM lane (query row) per thread ----------------
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;             // row within the tile == TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const int ti = r / G, h = r % G;               // token within the tile, head in the group
    const bool row_ok = ti < nr;
    const int o_tok = row_ok ? tok_off(ti) : 0;    // the token's offset in its window
    const int t = t_win + o_tok;                   // position of this row's token
    const size_t qrow = (size_t)row_win + o_tok;   // its global query row
    // Q row -> TMEM (bf16 pairs as 32-bit columns)
    {
      uint32_t qv[32];
      const uint4* src = reinterpret_cast<const uint4*>(
          q + (qrow * hq + (size_t)g * G + h) * kD);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = row_ok ? src[half * 8 + c] : make_uint4(0u, 0u, 0u, 0u);
          qv[4 * c + 0] = v.x;
          qv[4 * c + 1] = v.y;
          qv[4 * c + 2] = v.z;
          qv[4 * c + 3] = v.w;
        }
        tc_st32(lane_base + COL_Q + half * 32, qv);
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&q_ready);
    }
    // Online softmax with a lazily moved reference (log2 units): P = exp2(s*c - m_ref);
    // m_ref moves, and O, l are rescaled, only when a row's max exceeds m_ref by
    // more than kRescaleLog2, so the weights stay below 2^8 and writing P never
    // has to wait for the P*V in flight. Rows whose token did not select the
    // block get zero weights.
    //
    // A warp holds 32 rows = 32 / G tokens, split into two halves of 16 TMEM
    // lanes. When the block was selected only by tokens of one half, the warp
    // works on that half alone: a 16-lane access (16x32bx2) gives each of the
    // half's rows to two threads, 64 columns each (thread t: row 16*half +
    // t % 16, columns 64 * (t / 16) ..), so the exponentials of the block cost
    // half as much; the row's max and sum are combined over the thread pair,
    // and its state (m_ref, l_run) stays with the thread that owns the row.
    float m_ref = -INFINITY;
    float l_run = 0.f;  // row sum of the bf16-rounded weights P (the ones P V uses)
    const uint64_t sl2 = f2_pack(scale_log2, scale_log2);
    // the row this thread works on when only half hv (0, 1) of the warp is busy
    int ti_half[2], t_half[2];
    bool ok_half[2];
#pragma unroll
    for (int hv = 0; hv < 2; ++hv) {
      ti_half[hv] = (quarter * 32 + hv * 16 + (lane & 15)) / G;
      ok_half[hv] = ti_half[hv] < nr;
      t_half[hv] = t_win + (ok_half[hv] ? tok_off(ti_half[hv]) : 0);
    }
    const bool upper = lane >= 16;  // which 64 columns of the half-mode row
    int2 en_next = ent[0];
    for (int e = 0; e < n_e; ++e) {
      if (__any_sync(0xffffffffu, s_abort != 0)) break;
      const int2 en = en_next;
      if (e + 1 < n_e) en_next = ent[e + 1];      // prefetch the next plan entry
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full, e & 1))) {
        report(status, MSA_DEV_TIMEOUT);
        s_abort = 1;
        break;
      }
      tc_fence_after();
      const int j = en.x;
      const bool sel = row_ok && ((en.y >> ti) & 1);
      const uint32_t bal = __ballot_sync(0xffffffffu, sel);
      // 0: no row, 1: one half (hv), 2: both halves
      const int mode = (bal == 0u) ? 0 : (((bal & 0xffffu) != 0u) && ((bal >> 16) != 0u)) ? 2 : 1;
      const int hv = (bal & 0xffffu) ? 0 : 1;
      const bool owner = upper == (hv == 1);       // half mode: this thread's own row is the half's row
      // half-mode row of this thread and its visible keys
      const int kmax_h = (hv ? t_half[1] : t_half[0]) - j * B - (upper ? B / 2 : 0);
      const bool sel_h = (hv ? ok_half[1] : ok_half[0]) && ((en.y >> (hv ? ti_half[1] : ti_half[0])) & 1);
      const int kmax = t - j * B;  // full mode: visible keys of this thread's row: index <= kmax
      float s[B];
      if (mode == 2) {
#pragma unroll
        for (int c = 0; c < B / 32; ++c) {
          uint32_t v[32];
          tc_ld32(lane_base + COL_S + c * 32, v);
#pragma unroll
          for (int xx = 0; xx < 32; ++xx) s[c * 32 + xx] = __uint_as_float(v[xx]);
        }
        tc_wait_ld();
        tc_tie(s);
      } else if (mode == 1) {
        uint32_t v[B / 2];
        tc_ld16x2(lane_base + ((uint32_t)(hv * 16) << 16) + COL_S, v);
        tc_wait_ld();
        tc_tie(v);
#pragma unroll
        for (int xx = 0; xx < B / 2; ++xx) s[xx] = __uint_as_float(v[xx]);
      }
      tc_fence_before();
      mbar_arrive(&s_free);                        // S is in registers: the next S may start

      float mraw = -INFINITY;                      // max of the raw scores of this thread's row
      if (mode == 2) {
        if (__any_sync(0xffffffffu, kmax < B - 1)) {
          // a block that holds some row's own position: mask keys after it
#pragma unroll
          for (int c = 0; c < B; ++c) s[c] = (c <= kmax) ? s[c] : -INFINITY;
        }
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < B; c += 8) {
#pragma unroll
          for (int a = 0; a < 4; ++a) m4[a] = max3(m4[a], s[c + 2 * a], s[c + 2 * a + 1]);
        }
        mraw = max3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
      } else if (mode == 1) {
        if (__any_sync(0xffffffffu, kmax_h < B / 2 - 1)) {
#pragma unroll
          for (int c = 0; c < B / 2; ++c) s[c] = (c <= kmax_h) ? s[c] : -INFINITY;
        }
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < B / 2; c += 8) {
#pragma unroll
          for (int a = 0; a < 4; ++a) m4[a] = max3(m4[a], s[c + 2 * a], s[c + 2 * a + 1]);
        }
        const float mh = max3(m4[0], m4[1], fmaxf(m4[2], m4[3]));
        mraw = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, 16));  // both halves of the row
      }
      bool rescale = false;
      float alpha = 1.f;
      if (sel) {  // this thread's own row (in half mode its owner has the pair's max)
        const float mx = mraw * scale_log2;
        if (m_ref == -INFINITY) {
          m_ref = mx;                              // first block of this row: O and l are zero
        } else if (mx > m_ref + kRescaleLog2) {
          rescale = true;
          alpha = fast_exp2(m_ref - mx);
          m_ref = mx;
        }
      }
      if (__any_sync(0xffffffffu, rescale)) {
        // every P*V up to block e-1 must have completed before O is rescaled
        if (e > 0 && !__all_sync(0xffffffffu, mbar_wait(&o_done[(e - 1) & 1], ((e - 1) >> 1) & 1))) {
          report(status, MSA_DEV_TIMEOUT);
          s_abort = 1;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t v[32];
          tc_ld32(lane_base + COL_O + c * 32, v);
          tc_wait_ld();
          tc_tie(v);
#pragma unroll
          for (int xx = 0; xx < 32; ++xx) v[xx] = __float_as_uint(__uint_as_float(v[xx]) * alpha);
          tc_st32(lane_base + COL_O + c * 32, v);
        }
        l_run *= alpha;
      }
      // P buffer e&1 was last read by the P*V of block e-2. That P*V was issued
      // by the MMA thread before S_e, and the commit that signalled s_full for
      // S_e tracks every earlier MMA of that thread, so it has completed.
      const int pb = e & 1;
      // P = exp2(s*c - m_ref) rounded to bf16 (the tensor cores sum the same
      // rounded weights into l, so the output is an exact convex combination)
      const float m_own = sel ? m_ref : INFINITY;
      if (mode == 2) {
        const uint64_t neg_m = f2_pack(-m_own, -m_own);
        uint64_t lsum2 = 0ull;  // two fp32 partial sums
#pragma unroll
        for (int cc = 0; cc < B / 64; ++cc) {
          uint32_t pv[32];
          exp_pack<32>(s + 64 * cc, sl2, neg_m, pv, lsum2);
          tc_st32(lane_base + COL_P + pb * 64 + cc * 32, pv);
        }
        l_run += __uint_as_float((uint32_t)lsum2) + __uint_as_float((uint32_t)(lsum2 >> 32));
      } else if (mode == 1) {
        // the half's rows: m from the row's owner; the other half's rows: zero weights
        const float m_pair = __shfl_xor_sync(0xffffffffu, m_own, 16);
        const float m_use = owner ? m_own : m_pair;
        const float mu = sel_h ? m_use : INFINITY;
        const uint64_t neg_m = f2_pack(-mu, -mu);
        uint64_t lsum2 = 0ull;
        uint32_t pv[B / 4];
        exp_pack<B / 4>(s, sl2, neg_m, pv, lsum2);
        tc_st16x2(lane_base + ((uint32_t)(hv * 16) << 16) + COL_P + pb * 64, pv);
        uint32_t zero[B / 4];
#pragma unroll
        for (int xx = 0; xx < B / 4; ++xx) zero[xx] = 0u;
        tc_st16x2(lane_base + ((uint32_t)((1 - hv) * 16) << 16) + COL_P + pb * 64, zero);
        const float lh = __uint_as_float((uint32_t)lsum2) + __uint_as_float((uint32_t)(lsum2 >> 32));
        const float lp = __shfl_xor_sync(0xffffffffu, lh, 16);
        if (owner && sel) l_run += lh + lp;
      } else {
        uint32_t pv[32];
#pragma unroll
        for (int xx = 0; xx < 32; ++xx) pv[xx] = 0u;
#pragma unroll
        for (int cc = 0; cc < B / 64; ++cc) tc_st32(lane_base + COL_P + pb * 64 + cc * 32, pv);
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[pb]);
    }
    // epilogue: O / l -> bf16 once the last P*V has completed
    const bool go = !__any_sync(0xffffffffu, s_abort != 0);
    if (go && __all_sync(0xffffffffu, mbar_wait(&o_done[(n_e - 1) & 1], ((n_e - 1) >> 1) & 1))) {
      tc_fence_after();
      // a row that took no block (its token selected none) has an empty sum: A = 0
      const float l = (m_ref == -INFINITY) ? 0.f : l_run;
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      const size_t head = qrow * hq + (size_t)g * G + h;
      uint4* dst = reinterpret_cast<uint4*>(out + head * kD);
#pragma unroll
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t v[32];
        tc_ld32(lane_base + COL_O + c * 32, v);
        tc_wait_ld();
        tc_tie(v);
        if (row_ok && gate.g) {  // fused output gate: O = g A + (1 - g) X, one rounding
#pragma unroll
          for (int xx = 0; xx < 32; ++xx)
            v[xx] = __float_as_uint(gate_apply<bf16>(gate, head, c * 32 + xx, kD,
                                                     __uint_as_float(v[xx]) * inv));
#pragma unroll
          for (int xx = 0; xx < 32; xx += 8) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(v[xx]), __uint_as_float(v[xx + 1]));
            w.y = pack_bf16(__uint_as_float(v[xx + 2]), __uint_as_float(v[xx + 3]));
            w.z = pack_bf16(__uint_as_float(v[xx + 4]), __uint_as_float(v[xx + 5]));
            w.w = pack_bf16(__uint_as_float(v[xx + 6]), __uint_as_float(v[xx + 7]));
            dst[(c * 32 + xx) / 8] = w;
          }
        } else if (row_ok) {
#pragma unroll
          for (int xx = 0; xx < 32; xx += 8) {
            uint4 w;
            w.x = pack_bf16(__uint_as_float(v[xx]) * inv, __uint_as_float(v[xx + 1]) * inv);
            w.y = pack_bf16(__uint_as_float(v[xx + 2]) * inv, __uint_as_float(v[xx + 3]) * inv);
            w.z = pack_bf16(__uint_as_float(v[xx + 4]) * inv, __uint_as_float(v[xx + 5]) * inv);
            w.w = pack_bf16(__uint_as_float(v[xx + 6]) * inv, __uint_as_float(v[xx + 7]) * inv);
            dst[(c * 32 + xx) / 8] = w;
          }
        }
      }
      if (row_ok && lse)
        lse[qrow * hq + (size_t)g * G + h] =
            (l > 0.f) ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
    } else if (go) {
      report(status, MSA_DEV_TIMEOUT);
      s_abort = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
// units of one 128-row query tile (128 / G tokens) per CTA
static int plan_units(const msa_paged_kv_t* kv, int max_rows, int* ups) {
  const int TM = 128 / (kv->num_q_heads / kv->num_kv_heads);
  *ups = (max_rows + TM - 1) / TM;
  return kv->batch * (*ups) * kv->num_kv_heads;
}

static int windows_per_seq(int max_rows) { return (max_rows + kWin - 1) / kWin; }

// workspace: entries [units][ecap] int2 | counts [units] int | perm [batch][wps][hkv][kWin] u8
size_t prefill_ws(const msa_paged_kv_t* kv, int max_rows, int top_k) {
  int ups;
  const size_t units = plan_units(kv, max_rows, &ups);
  const int TM = 128 / (kv->num_q_heads / kv->num_kv_heads);
  const size_t ecap = (size_t)TM * top_k;
  const size_t perm = (size_t)kv->batch * windows_per_seq(max_rows) * kv->num_kv_heads * kWin;
  return units * ecap * sizeof(int2) + units * sizeof(int) + perm + 256;
}

bool prefill_tc_supported(const msa_paged_kv_t* kv) {
  const int G = kv->num_q_heads / kv->num_kv_heads;
  return kv->dtype == MSA_DTYPE_BF16 && kv->head_dim == 128 && (G == 8 || G == 16) &&
         (kv->block_size == 64 || kv->block_size == 128);
}

template <int B, int G>
static cudaError_t launch_tc(const msa_paged_kv_t* kv, const CUtensorMap& tk, const CUtensorMap& tv,
                             const void* q, const int32_t* cu_q, int units, int ups, int wps,
                             const uint8_t* perm, int ecap, const int2* entries, const int* counts,
                             float sl2, void* out, float* lse, gate_t gate, cudaStream_t st) {
  constexpr int NST = (B == 128) ? 3 : 4;
  const size_t smem = (size_t)NST * 2 * B * kD * 2 + 1024;
  auto kern = prefill_tc_kernel<B, G>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<units, 192, smem, st>>>(tk, tv, (const bf16*)q, cu_q, kv->page_table, kv->seq_lens,
                                 kv->status_word, kv->num_q_heads, kv->num_kv_heads, kv->num_pages,
                                 kv->max_blocks_per_seq, ups, wps, perm, ecap, entries, counts, sl2,
                                 (bf16*)out, lse, gate);
  return cudaGetLastError();
}

cudaError_t prefill_tc(const msa_paged_kv_t* kv, const void* q, const int32_t* cu_q, int max_rows,
                       const int32_t* idx, int top_k, float scale, void* out, float* lse, void* ws,
                       gate_t gate, cudaStream_t st) {
  const int G = kv->num_q_heads / kv->num_kv_heads, B = kv->block_size;
  const int TM = 128 / G;
  int ups;
  const int units = plan_units(kv, max_rows, &ups);
  const int wps = windows_per_seq(max_rows);
  const int ecap = TM * top_k;
  int2* entries = (int2*)ws;
  int* counts = (int*)(entries + (size_t)units * ecap);
  uint8_t* perm = (uint8_t*)(counts + units);
  const int hkv = kv->num_kv_heads, mb = kv->max_blocks_per_seq;
  const size_t cl_smem = ((size_t)(mb + 31) / 32) * 4;
  cudaError_t e = cudaFuncSetAttribute(prefill_cluster_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cl_smem);
  if (e != cudaSuccess) return e;
  prefill_cluster_kernel<<<kv->batch * wps * hkv, kWin, cl_smem, st>>>(
      cu_q, kv->seq_lens, idx, hkv, B, mb, top_k, TM, wps, perm);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  prefill_plan_kernel<<<units, 128, 0, st>>>(cu_q, kv->seq_lens, idx, kv->status_word, hkv, B, mb,
                                             top_k, TM, ups, wps, perm, ecap, entries, counts);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  CUtensorMap tk, tv;
  const uint64_t rows = (uint64_t)kv->num_pages * hkv * B;
  if (!make_tmap_bf16_2d(&tk, kv->k_pages, rows, kD, 64, B) ||
      !make_tmap_bf16_2d(&tv, kv->v_pages, rows, kD, 64, B))
    return cudaErrorInvalidValue;
  const float sl2 = scale * kLog2e;
  if (B == 128)
    return G == 8 ? launch_tc<128, 8>(kv, tk, tv, q, cu_q, units, ups, wps, perm, ecap, entries, counts, sl2, out, lse, gate, st)
                  : launch_tc<128, 16>(kv, tk, tv, q, cu_q, units, ups, wps, perm, ecap, entries, counts, sl2, out, lse, gate, st);
  return G == 8 ? launch_tc<64, 8>(kv, tk, tv, q, cu_q, units, ups, wps, perm, ecap, entries, counts, sl2, out, lse, gate, st)
                : launch_tc<64, 16>(kv, tk, tv, q, cu_q, units, ups, wps, perm, ecap, entries, counts, sl2, out, lse, gate, st);
}

}  // namespace msa
