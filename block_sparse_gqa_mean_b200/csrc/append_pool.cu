// KV append with the block-centroid pooling fused in.
//
// "Art of Focus: Ling 2.0 ...", section "Summarizing the Breakthrough": during
// prefill the tokens are aggregated into block representations kept in a block
// cache that uses the KV cache's page indexing, so decode can fetch block
// representations instead of re-reading every key. "Sparse Attention for
// Long-Context LLMs: Evolution and Practical Deployment", section 7.3: cache
// writes must stay consistent with the index. Here every write of a token
// re-pools the centroid of the block it lands in, in the same kernel.
//
// One CTA per (sequence, touched block, KV head). It stages the block's keys
// in shared memory - the rows already in the page and the new rows from the
// input are loaded together, 16-byte vectors, up to 16 per thread in flight,
// so a decode step's append costs one memory latency, not a store followed
// by a reload - writes the new key and value rows into the page, then every
// thread owns one coordinate and sums the keys present in the block in token
// order, in fp32, and divides by the count. The order does not depend on how
// the tokens arrived, so token-by-token appends and a one-shot build give
// equal bits.
#include "common.cuh"

namespace msa {

template <typename T, int D>
__global__ void __launch_bounds__(128) append_pool_kernel(
    const T* __restrict__ k_new, const T* __restrict__ v_new, const int32_t* __restrict__ cu_new,
    T* __restrict__ k_pages, T* __restrict__ v_pages, float* __restrict__ centroids,
    const int32_t* __restrict__ page_table, const int32_t* __restrict__ seq_lens,
    uint32_t* status, int hkv, int B, int num_pages, int max_blocks) {
  pdl_wait();
  const int lb = blockIdx.x;  // local block index among the blocks this append touches
  const int b = blockIdx.y;
  const int g = blockIdx.z;
  const int row0 = cu_new[b];
  const int n_new = cu_new[b + 1] - row0;
  const int L = seq_lens[b];
  if (n_new <= 0) return;
  if (n_new > L || L > max_blocks * B) {
    if (lb == 0 && g == 0 && threadIdx.x == 0) report(status, MSA_DEV_BAD_LENGTH);
    return;
  }
  const int t0 = L - n_new;           // first new position
  // the new rows lie inside k_new / v_new, and the grid (sized from the
  // caller's max_new) covers every block they touch
  if (!MSA_RANGE_OK(row0, row0 + n_new, cu_new[gridDim.y], status) ||
      !MSA_RANGE_OK(0, (t0 % B + n_new + B - 1) / B, gridDim.x, status))
    return;
  const int j = t0 / B + lb;          // logical block
  if (j * B >= L) return;             // beyond the last touched block
  const int page = page_table[(size_t)b * max_blocks + j];
  if (page < 0 || page >= num_pages) {
    if (g == 0 && threadIdx.x == 0) report(status, MSA_DEV_BAD_PAGE);
    return;
  }
  const int u_lo = max(t0, j * B);
  const int u_hi = min(L, (j + 1) * B);
  const size_t page_off = ((size_t)page * hkv + g) * B * D;
  [[maybe_unused]] const size_t pool = (size_t)num_pages * hkv * B * D;  // bounds-checked build
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* tile = reinterpret_cast<T*>(smem_raw);  // [n][D]

  // 1) the block's keys into shared memory, the new ones also into the page;
  //    the new values into the page. 16-byte chunks, CPR per row.
  constexpr int VEC = 16 / sizeof(T);
  constexpr int CPR = D / VEC;
  constexpr int NV = 16;                 // chunks in flight per thread
  const int n = u_hi - j * B;            // tokens in the block after the append
  const int total = n * CPR;
  const int first_new = (u_lo - j * B) * CPR;  // chunks before this one are in the page already
  auto new_src = [&](int c) {  // offset in k_new / v_new of chunk c of a new row
    const int r = c / CPR, col = (c % CPR) * VEC;
    return ((size_t)(row0 + (j * B + r - t0)) * hkv + g) * D + col;
  };
  // this thread's first value chunk is loaded before the keys, so its latency
  // overlaps theirs (a decode step has one new row: one chunk per thread at most)
  const int vc0 = first_new + (int)threadIdx.x;
  uint4 v_first = make_uint4(0u, 0u, 0u, 0u);
  if (vc0 < total) v_first = *reinterpret_cast<const uint4*>(v_new + new_src(vc0));
  for (int base = 0; base < total; base += NV * 128) {
    uint4 kv4[NV];
#pragma unroll
    for (int x = 0; x < NV; ++x) {
      const int c = base + x * 128 + (int)threadIdx.x;
      if (c < total) {
        if (c < first_new) {
          kv4[x] = reinterpret_cast<const uint4*>(k_pages + page_off)[c];
        } else {
          kv4[x] = *reinterpret_cast<const uint4*>(k_new + new_src(c));
        }
      }
    }
#pragma unroll
    for (int x = 0; x < NV; ++x) {
      const int c = base + x * 128 + (int)threadIdx.x;
      if (c < total && MSA_IN_BOUNDS(c, B * CPR, status)) {
        reinterpret_cast<uint4*>(tile)[c] = kv4[x];
        const size_t dst = page_off + (size_t)c * VEC;
        if (c >= first_new && MSA_RANGE_OK(dst, dst + VEC, pool, status))
          *reinterpret_cast<uint4*>(k_pages + dst) = kv4[x];
      }
    }
  }
  for (int c = vc0; c < total; c += blockDim.x) {
    const size_t dst = page_off + (size_t)c * VEC;
    const uint4 v = c == vc0 ? v_first : *reinterpret_cast<const uint4*>(v_new + new_src(c));
    if (MSA_RANGE_OK(dst, dst + VEC, pool, status)) *reinterpret_cast<uint4*>(v_pages + dst) = v;
  }
  __syncthreads();

  // 2) re-pool the block: mean over every token present, fixed token order
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    float s = 0.f;
    for (int u = 0; u < n; ++u) s = __fadd_rn(s, to_f32(tile[u * D + i]));
    centroids[((size_t)page * hkv + g) * D + i] = __fdiv_rn(s, (float)n);
  }
  pdl_release();
}

template <typename T, int D>
static cudaError_t launch_append(const msa_paged_kv_t* kv, const void* k_new, const void* v_new,
                                 const int32_t* cu_new, int max_new, cudaStream_t st) {
  const int B = kv->block_size;
  dim3 grid((max_new + B - 1) / B + 1, kv->batch, kv->num_kv_heads);
  const size_t smem = (size_t)B * D * sizeof(T);
  cudaError_t e = cudaFuncSetAttribute(append_pool_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(append_pool_kernel<T, D>, grid, dim3(128), smem, st, (const T*)k_new,
                    (const T*)v_new, cu_new, (T*)kv->k_pages, (T*)kv->v_pages, kv->centroids,
                    (const int32_t*)kv->page_table, (const int32_t*)kv->seq_lens, kv->status_word,
                    kv->num_kv_heads, B, kv->num_pages, kv->max_blocks_per_seq);
}

cudaError_t append_pool(const msa_paged_kv_t* kv, const void* k_new, const void* v_new,
                        const int32_t* cu_new, int max_new, cudaStream_t st) {
  const bool bf = kv->dtype == MSA_DTYPE_BF16;
  if (kv->head_dim == 128)
    return bf ? launch_append<bf16, 128>(kv, k_new, v_new, cu_new, max_new, st)
              : launch_append<float, 128>(kv, k_new, v_new, cu_new, max_new, st);
  return bf ? launch_append<bf16, 64>(kv, k_new, v_new, cu_new, max_new, st)
            : launch_append<float, 64>(kv, k_new, v_new, cu_new, max_new, st);
}

}  // namespace msa
