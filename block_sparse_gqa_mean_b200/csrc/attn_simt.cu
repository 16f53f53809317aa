// Exact attention over the selected blocks, CUDA-core (SIMT) form.
//
// "MiniMax Sparse Attention" (staik.se), method paragraph: after selection the
// main branch runs exact attention over the selected blocks only; "Sparse
// Attention + Linear Backbones", section 5.5: softmax(q k_sel^T / sqrt(d)) v_sel.
// For row r at position t, head h of group g:
//   U = tokens u of the blocks listed in block_idx[r][g] with u <= t,
//   o = sum_{u in U} softmax_u(scale * q.k_u) v_u,  lse = log sum exp(scale * q.k_u).
//
// This kernel serves the fp32 cache (accuracy path) and any shape the tensor-
// core kernels do not cover. One CTA per (row, KV group) holds the G query
// heads of the group, streams each selected block's K and V rows through
// shared memory and keeps an online softmax (running max, running sum) per
// head. Accumulation is fp32 with expf.
#include "common.cuh"

namespace msa {

template <typename T, int D>
__global__ void __launch_bounds__(128) attn_simt_kernel(
    const T* __restrict__ q, const int32_t* __restrict__ cu_q, const T* __restrict__ k_pages,
    const T* __restrict__ v_pages, const int32_t* __restrict__ page_table,
    const int32_t* __restrict__ seq_lens, uint32_t* status, const int32_t* __restrict__ block_idx,
    int top_k, int hq, int hkv, int B, int num_pages, int max_blocks, float scale,
    T* __restrict__ out, float* __restrict__ lse, gate_t gate) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int G = hq / hkv;
  float* qs = reinterpret_cast<float*>(smem_raw);  // [G][D]
  float* os = qs + G * D;                          // [G][D]
  float* ks = os + G * D;                          // [B][D+1]
  float* vs = ks + B * (D + 1);                    // [B][D]
  float* ps = vs + B * D;                          // [G][B]
  __shared__ float m_s[16], l_s[16], a_s[16];

  const int b = blockIdx.y, g = blockIdx.z;
  int row, t;
  const int L = seq_lens[b];
  if (cu_q) {
    const int r0 = cu_q[b], n = cu_q[b + 1] - r0;
    // the sequence's rows lie inside q / out, and the grid covers all of them
    if (blockIdx.x == 0) (void)MSA_RANGE_OK(n, n, gridDim.x, status);
    if (!MSA_RANGE_OK(r0, r0 + n, cu_q[gridDim.y], status)) return;
    if ((int)blockIdx.x >= n) return;
    row = r0 + blockIdx.x;
    if (n > L || L > max_blocks * B) {
      if (threadIdx.x == 0) report(status, MSA_DEV_BAD_LENGTH);
      return;
    }
    t = row_position(L, n, blockIdx.x);
  } else {
    row = b;
    if (L < 1 || L > max_blocks * B) {
      if (threadIdx.x == 0) report(status, MSA_DEV_BAD_LENGTH);
      return;
    }
    t = L - 1;
  }
  const int tid = threadIdx.x;
  for (int e = tid; e < G * D; e += blockDim.x) {
    qs[e] = to_f32(q[((size_t)row * hq + g * G) * D + e]);
    os[e] = 0.f;
  }
  if (tid < G) {
    m_s[tid] = -INFINITY;
    l_s[tid] = 0.f;
  }
  const int own = t / B;
  const int32_t* sel = block_idx + ((size_t)row * hkv + g) * top_k;
  for (int s = 0; s < top_k; ++s) {
    const int j = sel[s];
    if (j < 0 || (s > 0 && j == sel[s - 1])) continue;  // a repeated block counts once
    if (j > own) {
      if (tid == 0) report(status, MSA_DEV_BAD_INDEX);
      continue;
    }
    const int page = page_table[(size_t)b * max_blocks + j];
    if (page < 0 || page >= num_pages) {
      if (tid == 0) report(status, MSA_DEV_BAD_PAGE);
      continue;
    }
    const int nk = min(B, t + 1 - j * B);
    const size_t base = ((size_t)page * hkv + g) * B * D;
    if (!MSA_RANGE_OK(base, base + (size_t)nk * D, (size_t)num_pages * hkv * B * D, status))
      continue;
    __syncthreads();  // previous block's K/V/P fully consumed
    for (int e = tid; e < nk * D; e += blockDim.x) {
      const int kk = e / D, i = e % D;
      ks[kk * (D + 1) + i] = to_f32(k_pages[base + e]);
      vs[e] = to_f32(v_pages[base + e]);
    }
    __syncthreads();
    for (int e = tid; e < G * nk; e += blockDim.x) {
      const int h = e / nk, kk = e % nk;
      const float* qh = qs + h * D;
      const float* kr = ks + kk * (D + 1);
      float acc = 0.f;
      for (int i = 0; i < D; ++i) acc = fmaf(qh[i], kr[i], acc);
      ps[h * B + kk] = acc * scale;
    }
    __syncthreads();
    // per-head online-softmax update, one warp per head
    for (int h = tid / 32; h < G; h += blockDim.x / 32) {
      const int lane = tid % 32;
      float mx = -INFINITY;
      for (int kk = lane; kk < nk; kk += 32) mx = fmaxf(mx, ps[h * B + kk]);
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_new = fmaxf(m_s[h], mx);
      float sum = 0.f;
      for (int kk = lane; kk < nk; kk += 32) {
        const float p = expf(ps[h * B + kk] - m_new);
        ps[h * B + kk] = p;
        sum += p;
      }
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        const float alpha = expf(m_s[h] - m_new);  // 0 when m_s = -inf
        a_s[h] = alpha;
        l_s[h] = l_s[h] * alpha + sum;
        m_s[h] = m_new;
      }
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += blockDim.x) {
      const int h = e / D, i = e % D;
      const float* ph = ps + h * B;
      float acc = os[e] * a_s[h];
      for (int kk = 0; kk < nk; ++kk) acc = fmaf(ph[kk], vs[kk * D + i], acc);
      os[e] = acc;
    }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += blockDim.x) {
    const int h = e / D;
    out[((size_t)row * hq + g * G) * D + e] = from_f32<T>(
        gate_apply<T>(gate, (size_t)row * hq + g * G + h, e - h * D, D,
                      l_s[h] > 0.f ? os[e] / l_s[h] : 0.f));  // no key: A = 0
  }
  if (lse && tid < G) lse[(size_t)row * hq + g * G + tid] = m_s[tid] + logf(l_s[tid]);
}

template <typename T, int D>
static cudaError_t launch_simt(const msa_paged_kv_t* kv, const void* q, const int32_t* cu_q,
                               int grid_rows, const int32_t* idx, int top_k, float scale,
                               void* out, float* lse, gate_t gate, cudaStream_t st) {
  const int G = kv->num_q_heads / kv->num_kv_heads, B = kv->block_size;
  const size_t smem = ((size_t)2 * G * D + (size_t)B * (D + 1) + (size_t)B * D + (size_t)G * B) * 4;
  auto kern = attn_simt_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(grid_rows, kv->batch, kv->num_kv_heads);
  kern<<<grid, 128, smem, st>>>((const T*)q, cu_q, (const T*)kv->k_pages, (const T*)kv->v_pages,
                                 kv->page_table, kv->seq_lens, kv->status_word, idx, top_k,
                                 kv->num_q_heads, kv->num_kv_heads, B, kv->num_pages,
                                 kv->max_blocks_per_seq, scale, (T*)out, lse, gate);
  return cudaGetLastError();
}

// grid_rows: max rows per sequence (prefill, cu_q != NULL) or 1 (decode, cu_q == NULL)
cudaError_t attn_simt(const msa_paged_kv_t* kv, const void* q, const int32_t* cu_q, int grid_rows,
                      const int32_t* idx, int top_k, float scale, void* out, float* lse,
                      gate_t gate, cudaStream_t st) {
  const bool bf = kv->dtype == MSA_DTYPE_BF16;
  if (kv->head_dim == 128)
    return bf ? launch_simt<bf16, 128>(kv, q, cu_q, grid_rows, idx, top_k, scale, out, lse, gate, st)
              : launch_simt<float, 128>(kv, q, cu_q, grid_rows, idx, top_k, scale, out, lse, gate, st);
  return bf ? launch_simt<bf16, 64>(kv, q, cu_q, grid_rows, idx, top_k, scale, out, lse, gate, st)
            : launch_simt<float, 64>(kv, q, cu_q, grid_rows, idx, top_k, scale, out, lse, gate, st);
}

}  // namespace msa
