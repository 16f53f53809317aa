// Sparse decode attention: a stream-K split of the selected pages over one
// wave of resident CTAs, each (sequence, KV group) finished by the CTA that
// holds its first pages.
//
// "Art of Focus: Ling 2.0 ...", section "Summarizing the Breakthrough": during
// decode only the top-k relevant blocks are fetched, which removes the I/O of
// reading every key. "MiniMax Sparse Attention", method paragraph: exact
// attention over the selected blocks. The query at position t = seq_len-1 of
// each (sequence, KV group) has G heads; they attend to the tokens of the
// selected blocks (the own block up to t).
//
// Decode moves G flops per byte of K/V, so it is bound by HBM bandwidth. The
// work is the list of selection slots, unit u = (sequence b, group g) after
// unit, top_k slots each: W = batch * hkv * top_k. The grid is one wave of
// resident CTAs, C = min(W, CTAs per SM * SMs), and CTA c takes slots
// [c W / C, (c+1) W / C): every CTA streams the same number of slots, so no
// SM idles at the end of a partly filled last wave. A CTA walks its range as
// segments, one per unit it touches; per segment it looks up the blocks and
// pages of its slots, streams each block's K and V tile (page-contiguous,
// B x 128 bf16) into shared memory with 2-D TMA loads (128-byte swizzle, two
// 64-column boxes per tile, no multicast) through a two-stage mbarrier ring,
// and its four warps split each tile's keys, running mma.sync m16n8k16 (bf16
// in, fp32 accumulate) with the G query heads padded to 16 rows and an online
// softmax per row; the warps are merged in shared memory at the segment's
// end.
//   * A unit inside one CTA's range is finished there: output (rounded,
//     gated) and lse, with no partial written and no second kernel.
//   * A unit split over CTAs c0 < c1 < ... is finished by c0, whose range ends
//     with the unit's first slots; each later CTA holds a part of it as the
//     first segment of its range, writes that part's normalised (o, lse) to
//     its own workspace slot and publishes it with a release store of this
//     call's 64-bit tag into its flag. c0 reaches the unit last, waits for
//     those flags with acquire loads (bounded: about one second, then
//     MSA_DEV_TIMEOUT), merges the parts by log-sum-exp and clears the flags.
//     The parts are the first work of their CTAs and the grid is resident,
//     so the wait is short and cannot be circular.
// The tag is a fresh 64-bit value from a counter-based generator for every
// host call (a CUDA graph replays its captured tag, and the flags are cleared
// after each merge, so replays are safe too): the workspace needs no
// initialisation, and stale bytes could pass for a published flag only by
// matching the tag, a 2^-64 chance.
#include <algorithm>
#include <atomic>
#include <chrono>
#include <initializer_list>
#include <map>
#include <mutex>
#include <random>
#include <tuple>

#include "mma_sync.cuh"

namespace msa {

namespace {

constexpr int kD = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kStreamNST = 2;  // pipeline stages
using namespace warpmma;

// The CTA whose range holds slot x (the largest c with c W / C <= x).
__device__ __forceinline__ int cta_of_slot(long long x, int C, long long W) {
  return (int)(((x + 1) * C - 1) / W);
}

}  // namespace

template <int B, bool F32_OUT>
__global__ void __launch_bounds__(128, B == 64 ? 3 : 1) decode_streamk_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const bf16* __restrict__ q, const int32_t* __restrict__ block_idx,
    const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens, uint32_t* status,
    int batch, int top_k, int hq, int hkv, int num_pages, int max_blocks, float scale_log2,
    int block_lo, int block_hi, void* __restrict__ out, float* __restrict__ lse, gate_t gate,
    float* __restrict__ ws_o, float* __restrict__ ws_lse, uint64_t* __restrict__ flags,
    uint64_t tag) {
  constexpr int NST = kStreamNST;
  constexpr int TILE = B * kD * 2;       // bytes of one K (or V) tile
  constexpr int KW = B / 4;              // keys per warp per block
  constexpr int NT = KW / 8;             // n-tiles of 8 keys per warp
  // parts loaded at once by an owner's merge: a block-128 unit is typically
  // split over many CTAs (one CTA per SM fits), a block-64 unit over two or three
  constexpr int PB = B == 128 ? 16 : 4;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full[NST];
  __shared__ int s_page[256];
  __shared__ int s_blk[256];
  __shared__ int s_wcnt[4];
  __shared__ int s_n;
  __shared__ int s_abort;

  pdl_wait();
  const int G = hq / hkv;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int C = gridDim.x, c = blockIdx.x;
  const long long W = (long long)batch * hkv * top_k;
  const long long x0 = (long long)c * W / C, x1 = (long long)(c + 1) * W / C;
  if (tid == 0) {
    s_abort = 0;
    for (int s = 0; s < NST; ++s) mbar_init(&full[s], 1);
    mbar_fence_init();
  }
  int done = 0;  // tiles consumed by earlier segments: stage and phase of the next one

  for (long long x = x0; x < x1;) {
    const int u = (int)(x / top_k);
    const int s_begin = (int)(x - (long long)u * top_k);
    const int s_end = (int)min((long long)top_k, (long long)s_begin + (x1 - x));
    x += s_end - s_begin;
    const int b = u / hkv, g = u - (u / hkv) * hkv;
    const bool owner = s_begin == 0;  // the unit starts in this CTA's range
    const int L = seq_lens[b];
    const int t = L - 1;
    const bool len_ok = (L >= 1 && L <= max_blocks * B);
    if (!len_ok && owner && tid == 0) report(status, MSA_DEV_BAD_LENGTH);

    // the segment's slots: one thread each looks up block and page, then the
    // valid ones are compacted in slot order (a segment has <= top_k <= 256)
    __syncthreads();  // the previous segment is done with s_n, s_page and the stages
    if (tid == 0) s_n = 0;
    const int nslots = len_ok ? s_end - s_begin : 0;
    const int32_t* sel = block_idx + ((size_t)b * hkv + g) * top_k;
    for (int base = 0; base < nslots; base += 128) {
      int j = -1, pg = -1;
      bool ok = false;
      const int sl = s_begin + base + tid;
      if (base + tid < nslots) {
        j = sel[sl];
        // a block repeated in the adjacent slot (rows are ascending) counts once
        if (j >= 0 && sl > 0 && sel[sl - 1] == j) j = -1;
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
      const int st = (done + i) % NST;
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
      const int r0 = lane / 4, r1 = r0 + 8, cc = 2 * (lane % 4);
      const bf16* qb = q + ((size_t)b * hq + (size_t)g * G) * kD;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int k0 = ks * 16 + cc;
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

    int i = 0;
    for (; i < n; ++i) {
      const int st = (done + i) % NST;
      if (!mbar_wait(&full[st], (uint32_t)((done + i) / NST) & 1u)) {
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
      // let the copies still in flight (tiles i .. i+NST-1) land before the CTA exits (bounded)
      if (tid == 0)
        for (int k = i; k < min(n, i + NST); ++k)
          (void)mbar_wait(&full[(done + k) % NST], (uint32_t)((done + k) / NST) & 1u);
      __syncthreads();
      break;
    }
    done += n;

    // merge the four warps: quad-sum l, then max/scale across warps in smem
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    __syncthreads();  // stage buffers are free for reuse
    float* red_o = reinterpret_cast<float*>(smem);         // [4][16][kD]
    float* red_m = red_o + 4 * 16 * kD;                     // [4][16]
    float* red_l = red_m + 4 * 16;                          // [4][16]
    {
      const int r0 = lane / 4, r1 = r0 + 8;
      if (lane % 4 == 0) {
        red_m[warp * 16 + r0] = m0;
        red_m[warp * 16 + r1] = m1;
        red_l[warp * 16 + r0] = l0;
        red_l[warp * 16 + r1] = l1;
      }
#pragma unroll
      for (int nd = 0; nd < 16; ++nd) {
        const int cc = nd * 8 + 2 * (lane % 4);
        red_o[(warp * 16 + r0) * kD + cc] = o[nd][0];
        red_o[(warp * 16 + r0) * kD + cc + 1] = o[nd][1];
        red_o[(warp * 16 + r1) * kD + cc] = o[nd][2];
        red_o[(warp * 16 + r1) * kD + cc + 1] = o[nd][3];
      }
    }
    // an owner whose unit continues in later CTAs waits for their parts
    const int last = owner ? cta_of_slot((long long)u * top_k + top_k - 1, C, W) : c;
    const int np = last - c;  // later parts to merge (0 for a unit inside this range)
    // the flags are polled in parallel, one thread per part (acquire loads)
    int ok = 1;
    if (np > 0) {
      const uint64_t t0 = global_timer_ns();
      for (int k = tid; k < np && ok; k += 128) {
        if (!wait_flag(flags + c + 1 + k, tag, t0)) {
          report(status, MSA_DEV_TIMEOUT);
          ok = 0;
        }
      }
    }
    // every part this CTA merges is visible to all its threads after the barrier
    const int parts_ok = __syncthreads_and(ok);
    // the parts' lse (contiguous: CTAs c+1 .. last), staged after the warp buffers
    float* part_lse = red_l + 4 * 16;                       // [np][G]
    const bool merge = np > 0 && parts_ok;
    if (merge)
      for (int k = tid; k < np * G; k += 128) part_lse[k] = ws_lse[(size_t)(c + 1) * G + k];
    __syncthreads();
    // thread (row rq of a group of four rows, columns 4 cq .. 4 cq + 3)
    const int rq = tid / 32, cq = tid % 32, col = 4 * cq;
    for (int r = rq; r < G; r += 4) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) M = fmaxf(M, red_m[w * 16 + r]);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      float lsum = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float f = exp2f(red_m[w * 16 + r] - M);
          const float4 v = *reinterpret_cast<const float4*>(&red_o[(w * 16 + r) * kD + col]);
          acc.x += f * v.x;
          acc.y += f * v.y;
          acc.z += f * v.z;
          acc.w += f * v.w;
          lsum += f * red_l[w * 16 + r];
        }
      }
      // this segment's normalised part and its lse (log2 units)
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      const float4 o_part = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
      const float lse_part = lsum > 0.f ? M + log2f(lsum) : -INFINITY;
      if (!owner) {
        *reinterpret_cast<float4*>(&ws_o[((size_t)c * G + r) * kD + col]) = o_part;
        if (cq == 0) ws_lse[(size_t)c * G + r] = lse_part;
        continue;
      }
      // owner: log-sum-exp merge of its own part and the later CTAs' parts
      float Mx = lse_part;
      if (merge)
        for (int k = 0; k < np; ++k) Mx = fmaxf(Mx, part_lse[k * G + r]);
      float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
      float den = 0.f;
      if (Mx != -INFINITY) {
        const float f = exp2f(lse_part - Mx);
        num = make_float4(f * o_part.x, f * o_part.y, f * o_part.z, f * o_part.w);
        den = f;
        if (merge) {
          // PB parts' loads in flight at a time
          for (int k0 = 0; k0 < np; k0 += PB) {
            float4 pv[PB];
#pragma unroll
            for (int k = 0; k < PB; ++k)
              if (k0 + k < np)
                pv[k] = *reinterpret_cast<const float4*>(
                    &ws_o[((size_t)(c + 1 + k0 + k) * G + r) * kD + col]);
#pragma unroll
            for (int k = 0; k < PB; ++k) {
              if (k0 + k < np) {
                const float fc = exp2f(part_lse[(k0 + k) * G + r] - Mx);
                num.x += fc * pv[k].x;
                num.y += fc * pv[k].y;
                num.z += fc * pv[k].z;
                num.w += fc * pv[k].w;
                den += fc;
              }
            }
          }
        }
      }
      const float rden = den > 0.f ? 1.f / den : 0.f;  // no key: A = 0
      const float a[4] = {num.x * rden, num.y * rden, num.z * rden, num.w * rden};
      const size_t bh = (size_t)b * hq + (size_t)g * G + r;
      if constexpr (F32_OUT) {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + bh * kD + col) =
            make_float4(a[0], a[1], a[2], a[3]);
      } else {
        uint2 pk;
        pk.x = pack_bf16x2(gate_apply<bf16>(gate, bh, col, kD, a[0]),
                           gate_apply<bf16>(gate, bh, col + 1, kD, a[1]));
        pk.y = pack_bf16x2(gate_apply<bf16>(gate, bh, col + 2, kD, a[2]),
                           gate_apply<bf16>(gate, bh, col + 3, kD, a[3]));
        *reinterpret_cast<uint2*>(reinterpret_cast<bf16*>(out) + bh * kD + col) = pk;
      }
      if (lse && cq == 0) lse[bh] = den > 0.f ? (Mx + log2f(den)) * kLn2 : -INFINITY;
    }
    if (!owner) {
      // publish the part: every thread's stores, then the flag. The release
      // store is cumulative: the barrier orders the other threads' stores
      // before it, so the owner's acquire load sees all of them.
      __syncthreads();
      if (tid == 0) st_release_u64(flags + c, tag);
    } else if (np > 0 && tid == 0) {
      // the parts are merged: clear their flags for the next call
      for (int cc = c + 1; cc <= last; ++cc) flags[cc] = 0ull;
    }
  }
  pdl_release();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

// Resident CTAs of `fn` per SM at this shared-memory size, cached per device.
int resident_per_sm(const void* fn, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, size_t>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  const auto key = std::make_tuple(dev, fn, smem);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, 128, smem) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  cache.emplace(key, per_sm);
  return per_sm;
}

// A fresh nonzero 64-bit tag per call: SplitMix64 (Steele, Lea and Flood,
// "Fast splittable pseudorandom number generators", OOPSLA 2014) over a
// process-wide counter, seeded once from the system's entropy source and the
// clock.
uint64_t next_call_tag() {
  static const uint64_t seed = [] {
    std::random_device rd;
    return ((uint64_t)rd() << 32) ^ (uint64_t)rd() ^
           (uint64_t)std::chrono::steady_clock::now().time_since_epoch().count();
  }();
  static std::atomic<uint64_t> counter{0};
  uint64_t z = seed + 0x9e3779b97f4a7c15ull * (counter.fetch_add(1) + 1);
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
  z ^= z >> 31;
  return z | 1ull;  // 0 is the cleared flag
}

}  // namespace

// Upper bound of the grid: no more than four 128-thread CTAs of this kernel
// fit on an SM (its stage buffers alone take 64 KB of shared memory).
static int max_grid(int num_sms) { return 4 * num_sms; }

static size_t decode_smem(int B) {
  const size_t stages = (size_t)kStreamNST * 2 * B * kD * 2;
  const size_t red = (size_t)4 * 16 * kD * 4 + 2 * 4 * 16 * 4;
  return (stages > red ? stages : red) + 1024;
}

// workspace: per CTA one part, [grid][G][kD] fp32 o, [grid][G] fp32 lse, [grid] u64 flags
size_t decode_ws(const msa_paged_kv_t* kv, int top_k, int num_sms) {
  (void)top_k;
  const size_t G = (size_t)(kv->num_q_heads / kv->num_kv_heads);
  const size_t grid = (size_t)max_grid(num_sms);
  const size_t o = (grid * G * kD * 4 + 255) & ~(size_t)255;
  const size_t l = (grid * G * 4 + 255) & ~(size_t)255;
  return o + l + grid * 8 + 256;
}

template <int B, bool F32_OUT>
static cudaError_t launch_streamk(const msa_paged_kv_t* kv, const CUtensorMap& tk,
                                  const CUtensorMap& tv, const void* q, const int32_t* idx,
                                  int top_k, float sl2, void* out, float* lse, gate_t gate,
                                  void* ws, int num_sms, int lo, int hi, cudaStream_t st) {
  auto kern = decode_streamk_kernel<B, F32_OUT>;
  const size_t smem = decode_smem(B);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long W = (long long)kv->batch * kv->num_kv_heads * top_k;
  const long long resident = (long long)resident_per_sm((const void*)kern, smem) * num_sms;
  const int grid = (int)std::max(1LL, std::min({W, resident, (long long)max_grid(num_sms)}));
  const size_t G = (size_t)(kv->num_q_heads / kv->num_kv_heads);
  const size_t gmax = (size_t)max_grid(num_sms);
  float* ws_o = (float*)ws;
  float* ws_lse = (float*)((char*)ws + ((gmax * G * kD * 4 + 255) & ~(size_t)255));
  uint64_t* flags = (uint64_t*)((char*)ws_lse + ((gmax * G * 4 + 255) & ~(size_t)255));
  return launch_pdl(kern, dim3(grid), dim3(128), smem, st, tk, tv, (const bf16*)q, idx,
                    (const int32_t*)kv->page_table, (const int32_t*)kv->seq_lens, kv->status_word,
                    kv->batch, top_k, kv->num_q_heads, kv->num_kv_heads, kv->num_pages,
                    kv->max_blocks_per_seq, sl2, lo, hi, out, lse, gate, ws_o, ws_lse, flags,
                    next_call_tag());
}

static cudaError_t decode_splitk_any(const msa_paged_kv_t* kv, const void* q, const int32_t* idx,
                                     int top_k, float scale, void* out, bool f32_out, float* lse,
                                     void* ws, int num_sms, gate_t gate, int lo, int hi,
                                     cudaStream_t st) {
  const int B = kv->block_size;
  CUtensorMap tk, tv;
  const uint64_t rows = (uint64_t)kv->num_pages * kv->num_kv_heads * B;
  if (!make_tmap_bf16_2d(&tk, kv->k_pages, rows, kD, 64, B) ||
      !make_tmap_bf16_2d(&tv, kv->v_pages, rows, kD, 64, B))
    return cudaErrorInvalidValue;
  const float sl2 = scale * kLog2e;
  if (B == 64)
    return f32_out ? launch_streamk<64, true>(kv, tk, tv, q, idx, top_k, sl2, out, lse, gate, ws,
                                              num_sms, lo, hi, st)
                   : launch_streamk<64, false>(kv, tk, tv, q, idx, top_k, sl2, out, lse, gate, ws,
                                               num_sms, lo, hi, st);
  return f32_out ? launch_streamk<128, true>(kv, tk, tv, q, idx, top_k, sl2, out, lse, gate, ws,
                                             num_sms, lo, hi, st)
                 : launch_streamk<128, false>(kv, tk, tv, q, idx, top_k, sl2, out, lse, gate, ws,
                                              num_sms, lo, hi, st);
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
