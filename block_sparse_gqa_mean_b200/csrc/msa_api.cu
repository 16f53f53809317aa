// C-ABI entry points of libmsa: host-side validation, kernel dispatch and
// workspace sizing. See include/msa.h for the contract of each call.
#include <cudaTypedefs.h>

#include <mutex>

#include "tma.cuh"

namespace msa {

// kernels (defined in the other translation units)
cudaError_t append_pool(const msa_paged_kv_t*, const void*, const void*, const int32_t*, int,
                        cudaStream_t);
cudaError_t select_rows(const msa_paged_kv_t*, const void*, const int32_t*, int, int, int32_t*,
                        float*, cudaStream_t);
bool select_rows_supported(int top_k);
bool select_decode_supported(const msa_paged_kv_t*);
size_t select_decode_ws(const msa_paged_kv_t*, int top_k);
cudaError_t select_decode(const msa_paged_kv_t*, const void*, int, int32_t*, float*, void*,
                          cudaStream_t);
cudaError_t attn_simt(const msa_paged_kv_t*, const void*, const int32_t*, int, const int32_t*, int,
                      float, void*, float*, gate_t, cudaStream_t);
size_t decode_ws(const msa_paged_kv_t*, int top_k, int num_sms);
cudaError_t decode_splitk(const msa_paged_kv_t*, const void*, const int32_t*, int, float, void*,
                          float*, void*, int, gate_t, cudaStream_t);
size_t tokens_ws(const msa_paged_kv_t*, int num_rows);
cudaError_t select_tokens(const msa_paged_kv_t*, const void*, const void*, int, int, int32_t*, void*,
                          const int32_t*, int, cudaStream_t);
cudaError_t attn_tokens(const msa_paged_kv_t*, const void*, const int32_t*, int, float, void*,
                        float*, const int32_t*, int, cudaStream_t);
cudaError_t select_decode_range(const msa_paged_kv_t*, const void*, int, int, int, uint64_t*, void*,
                                cudaStream_t);
cudaError_t select_merge_lists(const msa_paged_kv_t*, const uint64_t*, int, int, int32_t*, float*,
                               cudaStream_t);
cudaError_t decode_splitk_range(const msa_paged_kv_t*, const void*, const int32_t*, int, float,
                                float*, float*, void*, int, int, int, cudaStream_t);
cudaError_t lse_merge(const float*, const float*, int, int, int, bool, void*, float*, cudaStream_t);
cudaError_t selftest_wait(int which, uint32_t* status, cudaStream_t st);
bool prefill_tc_supported(const msa_paged_kv_t*);
size_t prefill_ws(const msa_paged_kv_t*, int max_rows, int top_k);
cudaError_t prefill_tc(const msa_paged_kv_t*, const void*, const int32_t*, int, const int32_t*,
                       int, float, void*, float*, void*, gate_t, cudaStream_t);

// ---------------------------------------------------------------------------
// tensor maps (driver entry point resolved once through the runtime)
// ---------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                       uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// validation helpers
// ---------------------------------------------------------------------------
static bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

static msa_status_t check_kv(const msa_paged_kv_t* kv) {
  if (!kv) return MSA_ERR_INVALID_ARG;
  if (kv->dtype != MSA_DTYPE_BF16 && kv->dtype != MSA_DTYPE_F32) return MSA_ERR_UNSUPPORTED;
  if (kv->num_q_heads <= 0 || kv->num_kv_heads <= 0 || kv->batch <= 0 || kv->num_pages <= 0 ||
      kv->max_blocks_per_seq <= 0)
    return MSA_ERR_INVALID_ARG;
  if (kv->num_q_heads % kv->num_kv_heads != 0) return MSA_ERR_INVALID_ARG;
  if (kv->num_q_heads / kv->num_kv_heads > 16) return MSA_ERR_UNSUPPORTED;
  if (kv->head_dim != 64 && kv->head_dim != 128) return MSA_ERR_UNSUPPORTED;
  if (kv->block_size != 64 && kv->block_size != 128) return MSA_ERR_UNSUPPORTED;
  if ((uint64_t)kv->num_pages * kv->num_kv_heads * kv->block_size >= (1ull << 31))
    return MSA_ERR_UNSUPPORTED;
  if ((uint64_t)kv->max_blocks_per_seq * kv->block_size >= (1ull << 31)) return MSA_ERR_UNSUPPORTED;
  if (!kv->k_pages || !kv->v_pages || !kv->centroids || !kv->page_table || !kv->seq_lens ||
      !kv->status_word)
    return MSA_ERR_INVALID_ARG;
  if (!aligned(kv->k_pages, 16) || !aligned(kv->v_pages, 16) || !aligned(kv->centroids, 16) ||
      !aligned(kv->page_table, 4) || !aligned(kv->seq_lens, 4) || !aligned(kv->status_word, 4))
    return MSA_ERR_INVALID_ARG;
  return MSA_OK;
}

static int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

static bool use_decode_splitk(const msa_paged_kv_t* kv) {
  return kv->dtype == MSA_DTYPE_BF16 && kv->head_dim == 128;
}

static msa_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

// Host-side checks of the decode attention arguments other than the
// workspace; every decode attention entry point runs them before anything else.
msa_status_t check_decode_args(const msa_paged_kv_t* kv, const void* q, const int32_t* block_idx,
                               int32_t top_k, float softmax_scale, const void* out,
                               const float* lse) {
  msa_status_t s = check_kv(kv);
  if (s != MSA_OK) return s;
  if (top_k < 1 || top_k > 256) return MSA_ERR_UNSUPPORTED;
  if (!q || !block_idx || !out || !aligned(q, 16) || !aligned(out, 16) || !aligned(block_idx, 4) ||
      (lse && !aligned(lse, 4)) || !(softmax_scale > 0.f))
    return MSA_ERR_INVALID_ARG;
  return MSA_OK;
}

}  // namespace msa

using namespace msa;

extern "C" {

int32_t msa_version(void) { return 1000; }

int32_t msa_build_flags(void) { return kDebugBounds ? MSA_BUILD_DEBUG_BOUNDS : 0; }

msa_status_t msa_selftest_bounded_wait(int32_t which, uint32_t* status_word,
                                       msa_stream_t stream) {
  if (!status_word || !aligned(status_word, 4) || (which != 0 && which != 1))
    return MSA_ERR_INVALID_ARG;
  return from_cuda(selftest_wait(which, status_word, (cudaStream_t)stream));
}

const char* msa_status_string(msa_status_t s) {
  switch (s) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MSA_ERR_WORKSPACE: return "workspace too small";
    case MSA_ERR_CUDA: return "CUDA launch error";
  }
  return "unknown status";
}

size_t msa_workspace_size(msa_op_t op, const msa_paged_kv_t* kv, int32_t num_rows,
                          int32_t max_rows_per_seq, int32_t top_k) {
  if (check_kv(kv) != MSA_OK || top_k < 1) return 0;
  if (op == MSA_OP_SELECT_TOKENS)  // token top-K is not bounded by 256
    return tokens_ws(kv, max_rows_per_seq <= 1 ? kv->batch : (num_rows > 0 ? num_rows : 0));
  if (top_k > 256) return 0;
  switch (op) {
    case MSA_OP_SELECT:
      return max_rows_per_seq <= 1 ? select_decode_ws(kv, top_k) : 0;
    case MSA_OP_PREFILL:
      return prefill_tc_supported(kv) && max_rows_per_seq > 0
                 ? prefill_ws(kv, max_rows_per_seq, top_k) : 0;
    case MSA_OP_DECODE:
      return use_decode_splitk(kv) ? decode_ws(kv, top_k, num_sms()) : 0;
    default:
      break;
  }
  return 0;
}

msa_status_t msa_build_block_cache(const msa_paged_kv_t* kv, const void* k_new, const void* v_new,
                                   const int32_t* cu_new, int32_t max_new_per_seq,
                                   msa_stream_t stream) {
  msa_status_t s = check_kv(kv);
  if (s != MSA_OK) return s;
  if (max_new_per_seq < 0) return MSA_ERR_INVALID_ARG;
  if (max_new_per_seq == 0) return MSA_OK;
  if (!k_new || !v_new || !cu_new || !aligned(k_new, 16) || !aligned(v_new, 16) ||
      !aligned(cu_new, 4))
    return MSA_ERR_INVALID_ARG;
  return from_cuda(append_pool(kv, k_new, v_new, cu_new, max_new_per_seq, (cudaStream_t)stream));
}

msa_status_t msa_select_topk(const msa_paged_kv_t* kv, const void* q, const int32_t* cu_q,
                             int32_t num_rows, int32_t max_rows_per_seq, int32_t top_k,
                             int32_t* block_idx, float* block_score, void* workspace,
                             size_t workspace_bytes, msa_stream_t stream) {
  msa_status_t s = check_kv(kv);
  if (s != MSA_OK) return s;
  if (top_k < 1 || top_k > 256) return MSA_ERR_UNSUPPORTED;
  if (num_rows < 0 || max_rows_per_seq < 0) return MSA_ERR_INVALID_ARG;
  if (num_rows == 0) return MSA_OK;
  if (!q || !block_idx || !aligned(q, 16) || !aligned(block_idx, 4) ||
      (block_score && !aligned(block_score, 4)))
    return MSA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (!cu_q) {
    if (num_rows != kv->batch) return MSA_ERR_INVALID_ARG;
    if (!select_decode_supported(kv)) return MSA_ERR_UNSUPPORTED;
    const size_t need = select_decode_ws(kv, top_k);
    if (workspace_bytes < need || (need && (!workspace || !aligned(workspace, 16))))
      return MSA_ERR_WORKSPACE;
    return from_cuda(select_decode(kv, q, top_k, block_idx, block_score, workspace, st));
  }
  if (!aligned(cu_q, 4) || max_rows_per_seq < 1) return MSA_ERR_INVALID_ARG;
  if (!select_rows_supported(top_k)) return MSA_ERR_UNSUPPORTED;
  return from_cuda(select_rows(kv, q, cu_q, max_rows_per_seq, top_k, block_idx, block_score, st));
}

static msa_status_t attn_prefill(const msa_paged_kv_t* kv, const void* q, const int32_t* cu_q,
                                 int32_t num_rows, int32_t max_rows_per_seq,
                                 const int32_t* block_idx, int32_t top_k, float softmax_scale,
                                 gate_t gate, void* out, float* lse, void* workspace,
                                 size_t workspace_bytes, msa_stream_t stream) {
  msa_status_t s = check_kv(kv);
  if (s != MSA_OK) return s;
  if (top_k < 1 || top_k > 256) return MSA_ERR_UNSUPPORTED;
  if (num_rows < 0 || max_rows_per_seq < 0) return MSA_ERR_INVALID_ARG;
  if (num_rows == 0) return MSA_OK;
  if (!q || !cu_q || !block_idx || !out || !aligned(q, 16) || !aligned(out, 16) ||
      !aligned(cu_q, 4) || !aligned(block_idx, 4) || (lse && !aligned(lse, 4)) ||
      max_rows_per_seq < 1 || !(softmax_scale > 0.f))
    return MSA_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (prefill_tc_supported(kv)) {
    const size_t need = prefill_ws(kv, max_rows_per_seq, top_k);
    if (workspace_bytes < need || !workspace || !aligned(workspace, 16)) return MSA_ERR_WORKSPACE;
    return from_cuda(prefill_tc(kv, q, cu_q, max_rows_per_seq, block_idx, top_k, softmax_scale, out,
                                lse, workspace, gate, st));
  }
  return from_cuda(attn_simt(kv, q, cu_q, max_rows_per_seq, block_idx, top_k, softmax_scale, out,
                             lse, gate, st));
}

static msa_status_t attn_decode(const msa_paged_kv_t* kv, const void* q, const int32_t* block_idx,
                                int32_t top_k, float softmax_scale, gate_t gate, void* out,
                                float* lse, void* workspace, size_t workspace_bytes,
                                msa_stream_t stream) {
  msa_status_t s = check_decode_args(kv, q, block_idx, top_k, softmax_scale, out, lse);
  if (s != MSA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (use_decode_splitk(kv)) {
    const int sms = num_sms();
    const size_t need = decode_ws(kv, top_k, sms);
    if (workspace_bytes < need || !workspace || !aligned(workspace, 16)) return MSA_ERR_WORKSPACE;
    return from_cuda(
        decode_splitk(kv, q, block_idx, top_k, softmax_scale, out, lse, workspace, sms, gate, st));
  }
  return from_cuda(
      attn_simt(kv, q, nullptr, 1, block_idx, top_k, softmax_scale, out, lse, gate, st));
}

static bool gate_ok(const float* gate, int32_t per_dim, const void* x) {
  return gate && x && aligned(gate, 4) && aligned(x, 16) && (per_dim == 0 || per_dim == 1);
}

msa_status_t msa_sparse_attn_prefill(const msa_paged_kv_t* kv, const void* q, const int32_t* cu_q,
                                     int32_t num_rows, int32_t max_rows_per_seq,
                                     const int32_t* block_idx, int32_t top_k, float softmax_scale,
                                     void* out, float* lse, void* workspace,
                                     size_t workspace_bytes, msa_stream_t stream) {
  return attn_prefill(kv, q, cu_q, num_rows, max_rows_per_seq, block_idx, top_k, softmax_scale,
                      gate_t{}, out, lse, workspace, workspace_bytes, stream);
}

msa_status_t msa_sparse_attn_prefill_gated(const msa_paged_kv_t* kv, const void* q,
                                           const int32_t* cu_q, int32_t num_rows,
                                           int32_t max_rows_per_seq, const int32_t* block_idx,
                                           int32_t top_k, float softmax_scale, const float* gate,
                                           int32_t gate_per_dim, const void* x, void* out,
                                           float* lse, void* workspace, size_t workspace_bytes,
                                           msa_stream_t stream) {
  if (!gate_ok(gate, gate_per_dim, x)) return MSA_ERR_INVALID_ARG;
  gate_t gt;
  gt.g = gate;
  gt.x = x;
  gt.per_dim = gate_per_dim;
  return attn_prefill(kv, q, cu_q, num_rows, max_rows_per_seq, block_idx, top_k, softmax_scale, gt,
                      out, lse, workspace, workspace_bytes, stream);
}

msa_status_t msa_sparse_attn_decode(const msa_paged_kv_t* kv, const void* q,
                                    const int32_t* block_idx, int32_t top_k, float softmax_scale,
                                    void* out, float* lse, void* workspace, size_t workspace_bytes,
                                    msa_stream_t stream) {
  return attn_decode(kv, q, block_idx, top_k, softmax_scale, gate_t{}, out, lse, workspace,
                     workspace_bytes, stream);
}

msa_status_t msa_sparse_attn_decode_gated(const msa_paged_kv_t* kv, const void* q,
                                          const int32_t* block_idx, int32_t top_k,
                                          float softmax_scale, const float* gate,
                                          int32_t gate_per_dim, const void* x, void* out,
                                          float* lse, void* workspace, size_t workspace_bytes,
                                          msa_stream_t stream) {
  if (!gate_ok(gate, gate_per_dim, x)) return MSA_ERR_INVALID_ARG;
  gate_t gt;
  gt.g = gate;
  gt.x = x;
  gt.per_dim = gate_per_dim;
  return attn_decode(kv, q, block_idx, top_k, softmax_scale, gt, out, lse, workspace,
                     workspace_bytes, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// token-granular variant (decode)
// ---------------------------------------------------------------------------
extern "C" {

static msa_status_t select_tokens_any(const msa_paged_kv_t* kv, const void* ki_pages,
                                      const void* qi, const int32_t* cu_q, int32_t num_rows,
                                      int32_t num_index_heads, int32_t top_k, int32_t* tok_idx,
                                      void* workspace, size_t workspace_bytes,
                                      msa_stream_t stream) {
  msa_status_t s = msa::check_kv(kv);
  if (s != MSA_OK) return s;
  if (top_k < 1 || num_index_heads < 1 || num_index_heads > 256 || num_rows < 0 ||
      num_rows > 65535)
    return MSA_ERR_INVALID_ARG;
  if (num_rows == 0) return MSA_OK;
  if (!ki_pages || !qi || !tok_idx || !msa::aligned(ki_pages, 16) || !msa::aligned(qi, 16) ||
      !msa::aligned(tok_idx, 4) || (cu_q && !msa::aligned(cu_q, 4)))
    return MSA_ERR_INVALID_ARG;
  const size_t need = msa::tokens_ws(kv, num_rows);
  if (workspace_bytes < need || !workspace || !msa::aligned(workspace, 16)) return MSA_ERR_WORKSPACE;
  return msa::from_cuda(msa::select_tokens(kv, ki_pages, qi, num_index_heads, top_k, tok_idx,
                                           workspace, cu_q, num_rows, (cudaStream_t)stream));
}

static msa_status_t attn_tokens_any(const msa_paged_kv_t* kv, const void* q, const int32_t* cu_q,
                                    int32_t num_rows, const int32_t* tok_idx, int32_t top_k,
                                    float softmax_scale, void* out, float* lse,
                                    msa_stream_t stream) {
  msa_status_t s = msa::check_kv(kv);
  if (s != MSA_OK) return s;
  if (top_k < 1 || num_rows < 0 || num_rows > 65535) return MSA_ERR_INVALID_ARG;
  if (num_rows == 0) return MSA_OK;
  if (!q || !tok_idx || !out || !msa::aligned(q, 16) || !msa::aligned(out, 16) ||
      !msa::aligned(tok_idx, 4) || (lse && !msa::aligned(lse, 4)) || (cu_q && !msa::aligned(cu_q, 4)) ||
      !(softmax_scale > 0.f))
    return MSA_ERR_INVALID_ARG;
  return msa::from_cuda(msa::attn_tokens(kv, q, tok_idx, top_k, softmax_scale, out, lse, cu_q,
                                         num_rows, (cudaStream_t)stream));
}

msa_status_t msa_select_tokens(const msa_paged_kv_t* kv, const void* ki_pages, const void* qi,
                               int32_t num_index_heads, int32_t top_k, int32_t* tok_idx,
                               void* workspace, size_t workspace_bytes, msa_stream_t stream) {
  if (!kv) return MSA_ERR_INVALID_ARG;
  return select_tokens_any(kv, ki_pages, qi, nullptr, kv->batch, num_index_heads, top_k, tok_idx,
                           workspace, workspace_bytes, stream);
}

msa_status_t msa_sparse_attn_decode_tokens(const msa_paged_kv_t* kv, const void* q,
                                           const int32_t* tok_idx, int32_t top_k,
                                           float softmax_scale, void* out, float* lse,
                                           msa_stream_t stream) {
  if (!kv) return MSA_ERR_INVALID_ARG;
  return attn_tokens_any(kv, q, nullptr, kv->batch, tok_idx, top_k, softmax_scale, out, lse,
                         stream);
}

msa_status_t msa_select_tokens_rows(const msa_paged_kv_t* kv, const void* ki_pages,
                                    const void* qi, const int32_t* cu_q, int32_t num_rows,
                                    int32_t num_index_heads, int32_t top_k, int32_t* tok_idx,
                                    void* workspace, size_t workspace_bytes,
                                    msa_stream_t stream) {
  if (!cu_q) return MSA_ERR_INVALID_ARG;
  return select_tokens_any(kv, ki_pages, qi, cu_q, num_rows, num_index_heads, top_k, tok_idx,
                           workspace, workspace_bytes, stream);
}

msa_status_t msa_sparse_attn_prefill_tokens(const msa_paged_kv_t* kv, const void* q,
                                            const int32_t* cu_q, int32_t num_rows,
                                            const int32_t* tok_idx, int32_t top_k,
                                            float softmax_scale, void* out, float* lse,
                                            msa_stream_t stream) {
  if (!cu_q) return MSA_ERR_INVALID_ARG;
  return attn_tokens_any(kv, q, cu_q, num_rows, tok_idx, top_k, softmax_scale, out, lse, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// context-sharded decode
// ---------------------------------------------------------------------------
extern "C" {

msa_status_t msa_select_topk_range(const msa_paged_kv_t* kv, const void* q, int32_t block_lo,
                                   int32_t block_hi, int32_t top_k, uint64_t* cand_keys,
                                   void* workspace, size_t workspace_bytes, msa_stream_t stream) {
  msa_status_t s = msa::check_kv(kv);
  if (s != MSA_OK) return s;
  if (top_k < 1 || top_k - 1 > 64) return MSA_ERR_UNSUPPORTED;
  if (!msa::select_decode_supported(kv)) return MSA_ERR_UNSUPPORTED;
  if (!q || !msa::aligned(q, 16) || block_lo < 0 || block_hi < block_lo ||
      (top_k > 1 && (!cand_keys || !msa::aligned(cand_keys, 8))))
    return MSA_ERR_INVALID_ARG;
  const size_t need = msa::select_decode_ws(kv, top_k);
  if (workspace_bytes < need || !workspace || !msa::aligned(workspace, 16))
    return MSA_ERR_WORKSPACE;
  return msa::from_cuda(msa::select_decode_range(kv, q, top_k, block_lo, block_hi, cand_keys,
                                                 workspace, (cudaStream_t)stream));
}

msa_status_t msa_select_merge(const msa_paged_kv_t* kv, const uint64_t* cand_keys,
                              int32_t num_lists, int32_t top_k, int32_t* block_idx,
                              float* block_score, msa_stream_t stream) {
  msa_status_t s = msa::check_kv(kv);
  if (s != MSA_OK) return s;
  if (top_k < 1 || top_k - 1 > 64) return MSA_ERR_UNSUPPORTED;
  if (num_lists < 1 || !block_idx || !msa::aligned(block_idx, 4) ||
      (block_score && !msa::aligned(block_score, 4)) ||
      (top_k > 1 && (!cand_keys || !msa::aligned(cand_keys, 8))))
    return MSA_ERR_INVALID_ARG;
  return msa::from_cuda(msa::select_merge_lists(kv, cand_keys, num_lists, top_k, block_idx,
                                                block_score, (cudaStream_t)stream));
}

msa_status_t msa_sparse_attn_decode_range(const msa_paged_kv_t* kv, const void* q,
                                          const int32_t* block_idx, int32_t top_k,
                                          int32_t block_lo, int32_t block_hi, float softmax_scale,
                                          float* o_part, float* lse_part, void* workspace,
                                          size_t workspace_bytes, msa_stream_t stream) {
  msa_status_t s = msa::check_decode_args(kv, q, block_idx, top_k, softmax_scale, o_part, lse_part);
  if (s != MSA_OK) return s;
  if (!msa::use_decode_splitk(kv)) return MSA_ERR_UNSUPPORTED;
  if (!lse_part || block_lo < 0 || block_hi < block_lo) return MSA_ERR_INVALID_ARG;
  const int sms = msa::num_sms();
  const size_t need = msa::decode_ws(kv, top_k, sms);
  if (workspace_bytes < need || !workspace || !msa::aligned(workspace, 16))
    return MSA_ERR_WORKSPACE;
  return msa::from_cuda(msa::decode_splitk_range(kv, q, block_idx, top_k, softmax_scale, o_part,
                                                 lse_part, workspace, sms, block_lo, block_hi,
                                                 (cudaStream_t)stream));
}

msa_status_t msa_lse_merge(const float* o_parts, const float* lse_parts, int32_t num_parts,
                           int32_t rows, int32_t head_dim, int32_t out_dtype, void* out,
                           float* lse, msa_stream_t stream) {
  if (num_parts < 1 || rows < 0 || head_dim < 1) return MSA_ERR_INVALID_ARG;
  if (out_dtype != MSA_DTYPE_BF16 && out_dtype != MSA_DTYPE_F32) return MSA_ERR_UNSUPPORTED;
  if (rows == 0) return MSA_OK;
  if (!o_parts || !lse_parts || !out || !msa::aligned(o_parts, 4) || !msa::aligned(lse_parts, 4) ||
      !msa::aligned(out, 4) || (lse && !msa::aligned(lse, 4)))
    return MSA_ERR_INVALID_ARG;
  return msa::from_cuda(msa::lse_merge(o_parts, lse_parts, num_parts, rows, head_dim,
                                       out_dtype == MSA_DTYPE_BF16, out, lse,
                                       (cudaStream_t)stream));
}

}  // extern "C"
