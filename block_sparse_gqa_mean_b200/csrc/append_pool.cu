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
// One CTA per (sequence, touched block, KV head). It copies the new rows of
// that block into the page (16-byte vector copies), stages the block's keys
// in shared memory, then every thread owns one coordinate and sums the keys
// present in the block in token order, in fp32, and divides by the count. The order does not depend on how the tokens
// arrived, so token-by-token appends and a one-shot build give equal bits.
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

  // 1) copy the new rows of this block: 16-byte chunks, D/8 (bf16) or D/4 (fp32) per row
  constexpr int VEC = 16 / sizeof(T);
  constexpr int CPR = D / VEC;  // chunks per row
  const int nrows = u_hi - u_lo;
  for (int c = threadIdx.x; c < nrows * CPR; c += blockDim.x) {
    const int r = c / CPR, col = (c % CPR) * VEC;
    const int u = u_lo + r;
    const size_t src = ((size_t)(row0 + (u - t0)) * hkv + g) * D + col;
    const size_t dst = page_off + (size_t)(u - j * B) * D + col;
    if (!MSA_RANGE_OK(dst, dst + VEC, (size_t)num_pages * hkv * B * D, status)) continue;
    *reinterpret_cast<uint4*>(k_pages + dst) = *reinterpret_cast<const uint4*>(k_new + src);
    *reinterpret_cast<uint4*>(v_pages + dst) = *reinterpret_cast<const uint4*>(v_new + src);
  }
  __syncthreads();

  // 2) re-pool the block: mean over every token present, fixed token order.
  //    The block's keys are staged in shared memory with 16-byte loads first.
  extern __shared__ __align__(16) unsigned char smem_raw[];
  T* tile = reinterpret_cast<T*>(smem_raw);  // [n][D]
  const int n = u_hi - j * B;
  for (int c = threadIdx.x; c < n * CPR; c += blockDim.x)
    if (MSA_IN_BOUNDS(c, B * CPR, status))
      reinterpret_cast<uint4*>(tile)[c] =
          reinterpret_cast<const uint4*>(k_pages + page_off)[c];
  __syncthreads();
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
