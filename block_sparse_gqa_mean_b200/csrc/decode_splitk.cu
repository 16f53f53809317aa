// Sparse decode attention: split-k over the selected pages, then an LSE merge.
//
// "Art of Focus: Ling 2.0 ...", section "Summarizing the Breakthrough": during
// decode only the top-k relevant blocks are fetched, which removes the I/O of
// reading every key. "MiniMax Sparse Attention", method paragraph: exact
// attention over the selected blocks. The query at position t = seq_len-1 of
// each (sequence, KV group) has G heads; they attend to the tokens of the
// selected blocks (the own block up to t).
//
// Decode moves G flops per byte of K/V, so it is bound by HBM bandwidth. Each
// CTA takes one (sequence, KV group, split) and a contiguous share of the
// selected block list; it streams each block's K and V tile (page-contiguous,
// B x 128 bf16) into shared memory with 2-D TMA loads (128-byte swizzle, two
// 64-column boxes per tile, no multicast) through a two-stage mbarrier
// pipeline. Four warps split each tile's keys; each warp runs
// mma.sync m16n8k16 (bf16 in, fp32 accumulate) with the G query heads padded
// to 16 rows, keeps an online softmax per row, and the warps are merged in
// shared memory. The CTA writes its normalised partial (o, lse); a second
// kernel merges the splits by log-sum-exp and rounds to bf16.
#include "mma_sync.cuh"

namespace msa {

namespace {

constexpr int kD = 128;
constexpr float kLog2e = 1.4426950408889634f;
using namespace warpmma;
}  // namespace

template <int B>
__global__ void __launch_bounds__(128) decode_splitk_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const bf16* __restrict__ q, const int32_t* __restrict__ block_idx,
    const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens, uint32_t* status,
    int top_k, int hq, int hkv, int num_pages, int max_blocks, float scale_log2, int splits,
    int per_split, int block_lo, int block_hi, float* __restrict__ ws_o,
    float* __restrict__ ws_lse) {
  constexpr int NST = 2;                 // pipeline stages
  constexpr int TILE = B * kD * 2;       // bytes of one K (or V) tile
  constexpr int KW = B / 4;              // keys per warp per block
  constexpr int NT = KW / 8;             // n-tiles of 8 keys per warp
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full[NST];
  __shared__ int s_page[256];
  __shared__ int s_blk[256];
  __shared__ int s_n;
  __shared__ int s_abort;

  pdl_wait();
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = hq / hkv;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int L = seq_lens[b];
  const int t = L - 1;
  const bool len_ok = (L >= 1 && L <= max_blocks * B);

  // this split's slots: one thread each looks up block and page, then the
  // valid ones are compacted in slot order (per_split <= 256)
  __shared__ int s_wcnt[4];
  const int s0 = split * per_split;
  const int nslots = len_ok ? max(0, min(top_k, s0 + per_split) - s0) : 0;
  if (!len_ok && split == 0 && g == 0 && tid == 0) report(status, MSA_DEV_BAD_LENGTH);
  if (tid == 0) {
    s_n = 0;
    s_abort = 0;
    for (int s = 0; s < NST; ++s) mbar_init(&full[s], 1);
    mbar_fence_init();
  }
  const int32_t* sel = block_idx + ((size_t)b * hkv + g) * top_k + s0;
  for (int base = 0; base < nslots; base += 128) {
    int j = -1, pg = -1;
    bool ok = false;
    if (base + tid < nslots) {
      j = sel[base + tid];
      // a block repeated in the adjacent slot (rows are ascending) counts once
      if (j >= 0 && s0 + base + tid > 0 && sel[base + tid - 1] == j) j = -1;
      // context-sharded decode: blocks outside this rank's range are another's
      if (j >= 0 && j <= t / B && (j < block_lo || j >= block_hi)) j = -1;
      if (j >= 0) {
        if (j > t / B) {
          report(status, MSA_DEV_BAD_INDEX);
        } else {
          pg = page_table[(size_t)b * max_blocks + j];
          if (pg < 0 || pg >= num_pages) report(status, MSA_DEV_BAD_PAGE);
          else ok = true;
        }
      }
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, ok);
    if (lane == 0) s_wcnt[warp] = __popc(bal);
    __syncthreads();
    int pos = s_n + __popc(bal & ((1u << lane) - 1u));
    for (int w = 0; w < warp; ++w) pos += s_wcnt[w];
    if (ok && MSA_IN_BOUNDS(pos, 256, status)) {
      s_page[pos] = pg;
      s_blk[pos] = j;
    }
    __syncthreads();
    if (tid == 0) s_n += s_wcnt[0] + s_wcnt[1] + s_wcnt[2] + s_wcnt[3];
    __syncthreads();
  }
  __syncthreads();
  const int n = s_n;

  auto issue = [&](int i) {
    const int st = i % NST;
    unsigned char* kt = smem + st * 2 * TILE;
    unsigned char* vt = kt + TILE;
    const int y = (s_page[i] * hkv + g) * B;
    mbar_expect_tx(&full[st], 2 * TILE);
    tma_load_2d(kt, &tm_k, &full[st], 0, y);
    tma_load_2d(kt + TILE / 2, &tm_k, &full[st], 64, y);
    tma_load_2d(vt, &tm_v, &full[st], 0, y);
    tma_load_2d(vt + TILE / 2, &tm_v, &full[st], 64, y);
  };
  if (tid == 0)
    for (int i = 0; i < min(NST, n); ++i) issue(i);

  // query fragments (rows >= G are zero)
  uint32_t qa[8][4];
  {
    const int r0 = lane / 4, r1 = r0 + 8, c = 2 * (lane % 4);
    const bf16* qb = q + ((size_t)b * hq + (size_t)g * G) * kD;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int k0 = ks * 16 + c;
      qa[ks][0] = r0 < G ? *reinterpret_cast<const uint32_t*>(qb + r0 * kD + k0) : 0u;
      qa[ks][1] = r1 < G ? *reinterpret_cast<const uint32_t*>(qb + r1 * kD + k0) : 0u;
      qa[ks][2] = r0 < G ? *reinterpret_cast<const uint32_t*>(qb + r0 * kD + k0 + 8) : 0u;
      qa[ks][3] = r1 < G ? *reinterpret_cast<const uint32_t*>(qb + r1 * kD + k0 + 8) : 0u;
    }
  }

  float o[16][4];
#pragma unroll
  for (int nd = 0; nd < 16; ++nd) o[nd][0] = o[nd][1] = o[nd][2] = o[nd][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  for (int i = 0; i < n; ++i) {
    const int st = i % NST;
    if (!mbar_wait(&full[st], (i / NST) & 1)) {
      report(status, MSA_DEV_TIMEOUT);
      atomicExch(&s_abort, 1);
    }
    __syncthreads();
    if (s_abort) break;
    const uint32_t kt = smem_u32(smem + st * 2 * TILE);
    const uint32_t vt = kt + TILE;
    const int j = s_blk[i];
    const int kmax = t - j * B;  // keys with index <= kmax are visible

    // S = Q K^T for this warp's KW keys
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
        ldsm_x4(tile_chunk(kt, B, key, chunk), b0, b1, b2, b3);
        mma_bf16_16816(s[nt], qa[ks], b0, b1);
        mma_bf16_16816(s[nt], qa[ks + 1], b2, b3);
      }
    }
    // mask, scale into log2 units, row max
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int kc = warp * KW + nt * 8 + 2 * (lane % 4);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = kc + (e & 1);
        const float v = key <= kmax ? s[nt][e] * scale_log2 : -INFINITY;
        s[nt][e] = v;
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
      // weights rounded to bf16 here, once: the row sum and P*V use the same values
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
    // O += P V
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
        ldsm_x4_t(tile_chunk(vt, B, key, chunk), b0, b1, b2, b3);
        mma_bf16_16816(o[nd], pa, b0, b1);
        mma_bf16_16816(o[nd + 1], pa, b2, b3);
      }
    }
    __syncthreads();  // every warp is done with this stage
    if (tid == 0 && i + NST < n) issue(i + NST);
  }
  if (s_abort) {
    // let copies already in flight land before the CTA exits (bounded)
    if (tid == 0)
      for (int i = 0; i < n; ++i) (void)mbar_wait(&full[i % NST], (i / NST) & 1);
    __syncthreads();
  }

  // merge the four warps: quad-sum l, then max/scale across warps in smem
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  __syncthreads();  // stage buffers are free for reuse
  float* red_o = reinterpret_cast<float*>(smem);         // [4][16][kD]
  float* red_m = red_o + 4 * 16 * kD;                     // [4][16]
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
    red_o[(warp * 16 + r0) * kD + c] = o[nd][0];
    red_o[(warp * 16 + r0) * kD + c + 1] = o[nd][1];
    red_o[(warp * 16 + r1) * kD + c] = o[nd][2];
    red_o[(warp * 16 + r1) * kD + c + 1] = o[nd][3];
  }
  __syncthreads();
  // thread tid owns column tid of every head row
  for (int r = 0; r < G; ++r) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, red_m[w * 16 + r]);
    float acc = 0.f, lsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float f = exp2f(red_m[w * 16 + r] - M);
        acc += f * red_o[(w * 16 + r) * kD + tid];
        lsum += f * red_l[w * 16 + r];
      }
    }
    const int h = g * G + r;
    const size_t part = ((size_t)b * hq + h) * splits + split;
    ws_o[part * kD + tid] = lsum > 0.f ? acc / lsum : 0.f;
    if (tid == 0) ws_lse[part] = lsum > 0.f ? M + log2f(lsum) : -INFINITY;
  }
  pdl_release();
}

// Merge the split partials of each (sequence, head) by log-sum-exp.
template <typename T>
__global__ void __launch_bounds__(128) decode_combine_kernel(const float* __restrict__ ws_o,
                                                             const float* __restrict__ ws_lse,
                                                             int splits, T* __restrict__ out,
                                                             float* __restrict__ lse, gate_t gate) {
  pdl_wait();
  const size_t bh = blockIdx.x;
  const int tid = threadIdx.x;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, ws_lse[bh * splits + s]);
  float acc = 0.f, w = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < splits; ++s) {
      const float f = exp2f(ws_lse[bh * splits + s] - M);
      acc += f * ws_o[(bh * splits + s) * kD + tid];
      w += f;
    }
  }
  out[bh * kD + tid] = from_f32<T>(gate_apply<T>(gate, bh, tid, kD, w > 0.f ? acc / w : 0.f));
  if (lse && tid == 0) lse[bh] = (M + log2f(w)) * 0.6931471805599453f;
  pdl_release();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
int decode_splits(const msa_paged_kv_t* kv, int top_k, int num_sms) {
  // about eight CTAs per SM over the whole grid (three resident at a time),
  // so the HBM stream has bytes in flight and the last wave is short
  const int units = kv->batch * kv->num_kv_heads;
  int splits = (8 * num_sms + units - 1) / units;
  if (splits > top_k) splits = top_k;
  if (splits < 1) splits = 1;
  return splits;
}

size_t decode_ws(const msa_paged_kv_t* kv, int top_k, int num_sms) {
  const size_t parts = (size_t)kv->batch * kv->num_q_heads * decode_splits(kv, top_k, num_sms);
  return parts * kD * 4 + parts * 4 + 256;
}

static size_t decode_smem(int B) {
  const size_t stages = (size_t)2 * 2 * B * kD * 2;
  const size_t red = (size_t)4 * 16 * kD * 4 + 2 * 4 * 16 * 4;
  return (stages > red ? stages : red) + 1024;
}

static cudaError_t decode_splitk_any(const msa_paged_kv_t* kv, const void* q, const int32_t* idx,
                                     int top_k, float scale, void* out, bool f32_out, float* lse,
                                     void* ws, int num_sms, gate_t gate, int lo, int hi,
                                     cudaStream_t st) {
  const int B = kv->block_size;
  const int splits = decode_splits(kv, top_k, num_sms);
  const int per = (top_k + splits - 1) / splits;
  CUtensorMap tk, tv;
  const uint64_t rows = (uint64_t)kv->num_pages * kv->num_kv_heads * B;
  if (!make_tmap_bf16_2d(&tk, kv->k_pages, rows, kD, 64, B) ||
      !make_tmap_bf16_2d(&tv, kv->v_pages, rows, kD, 64, B))
    return cudaErrorInvalidValue;
  const size_t parts = (size_t)kv->batch * kv->num_q_heads * splits;
  float* ws_o = (float*)ws;
  float* ws_lse = ws_o + parts * kD;
  const size_t smem = decode_smem(B);
  dim3 grid(splits, kv->num_kv_heads, kv->batch);
  const float sl2 = scale * kLog2e;
  cudaError_t e;
  if (B == 64) {
    e = cudaFuncSetAttribute(decode_splitk_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(decode_splitk_kernel<64>, grid, dim3(128), smem, st, tk, tv, (const bf16*)q,
                   idx, (const int32_t*)kv->page_table, (const int32_t*)kv->seq_lens,
                   kv->status_word, top_k, kv->num_q_heads, kv->num_kv_heads, kv->num_pages,
                   kv->max_blocks_per_seq, sl2, splits, per, lo, hi, ws_o, ws_lse);
  } else {
    e = cudaFuncSetAttribute(decode_splitk_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(decode_splitk_kernel<128>, grid, dim3(128), smem, st, tk, tv, (const bf16*)q,
                   idx, (const int32_t*)kv->page_table, (const int32_t*)kv->seq_lens,
                   kv->status_word, top_k, kv->num_q_heads, kv->num_kv_heads, kv->num_pages,
                   kv->max_blocks_per_seq, sl2, splits, per, lo, hi, ws_o, ws_lse);
  }
  if (e != cudaSuccess) return e;
  if (f32_out)
    return launch_pdl(decode_combine_kernel<float>, dim3(kv->batch * kv->num_q_heads), dim3(128),
                      0, st, (const float*)ws_o, (const float*)ws_lse, splits, (float*)out, lse,
                      gate);
  return launch_pdl(decode_combine_kernel<bf16>, dim3(kv->batch * kv->num_q_heads), dim3(128), 0,
                    st, (const float*)ws_o, (const float*)ws_lse, splits, (bf16*)out, lse, gate);
}

cudaError_t decode_splitk(const msa_paged_kv_t* kv, const void* q, const int32_t* idx, int top_k,
                          float scale, void* out, float* lse, void* ws, int num_sms, gate_t gate,
                          cudaStream_t st) {
  return decode_splitk_any(kv, q, idx, top_k, scale, out, false, lse, ws, num_sms, gate, 0,
                           0x7fffffff, st);
}

// Context-sharded decode: this rank's normalised fp32 partial and its lse over
// the selected blocks in [lo, hi).
cudaError_t decode_splitk_range(const msa_paged_kv_t* kv, const void* q, const int32_t* idx,
                                int top_k, float scale, float* o_part, float* lse_part, void* ws,
                                int num_sms, int lo, int hi, cudaStream_t st) {
  return decode_splitk_any(kv, q, idx, top_k, scale, o_part, true, lse_part, ws, num_sms, gate_t{},
                           lo, hi, st);
}

// Log-sum-exp merge of num_parts normalised partials: o_parts [num_parts][rows][D]
// fp32, lse_parts [num_parts][rows] (natural log, -inf: no keys) -> out [rows][D]
// in T, lse [rows] (may be null).
template <typename T>
__global__ void __launch_bounds__(128) lse_merge_kernel(const float* __restrict__ o_parts,
                                                        const float* __restrict__ lse_parts,
                                                        int num_parts, int rows, int D,
                                                        T* __restrict__ out,
                                                        float* __restrict__ lse) {
  pdl_wait();
  const size_t r = blockIdx.x;
  float M = -INFINITY;
  for (int p = 0; p < num_parts; ++p) M = fmaxf(M, lse_parts[(size_t)p * rows + r]);
  float w = 0.f;
  if (M != -INFINITY)
    for (int p = 0; p < num_parts; ++p) w += expf(lse_parts[(size_t)p * rows + r] - M);
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    float acc = 0.f;
    if (M != -INFINITY)
      for (int p = 0; p < num_parts; ++p)
        acc += expf(lse_parts[(size_t)p * rows + r] - M) * o_parts[((size_t)p * rows + r) * D + i];
    out[r * D + i] = from_f32<T>(w > 0.f ? acc / w : 0.f);
  }
  if (lse && threadIdx.x == 0) lse[r] = w > 0.f ? M + logf(w) : -INFINITY;
  pdl_release();
}

cudaError_t lse_merge(const float* o_parts, const float* lse_parts, int num_parts, int rows, int D,
                      bool bf16_out, void* out, float* lse, cudaStream_t st) {
  if (bf16_out)
    return launch_pdl(lse_merge_kernel<bf16>, dim3(rows), dim3(128), 0, st, o_parts, lse_parts,
                      num_parts, rows, D, (bf16*)out, lse);
  return launch_pdl(lse_merge_kernel<float>, dim3(rows), dim3(128), 0, st, o_parts, lse_parts,
                    num_parts, rows, D, (float*)out, lse);
}

}  // namespace msa
