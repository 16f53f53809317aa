/*
 * msa.h - C ABI of the block-sparse GQA attention library (libmsa.so).
 *
 * The library implements MoBA-style block-sparse attention over a paged KV
 * cache on NVIDIA B200 (sm_100a):
 *
 *   1. the keys of each block are mean-pooled into an fp32 centroid kept in a
 *      block cache that is indexed by the same page ids as the K/V cache
 *      ("Art of Focus: Ling 2.0 ...", section "Summarizing the Breakthrough":
 *      blocks are aggregated into representations stored in a page-aware
 *      block cache that shares the KV cache's indexing);
 *   2. every query row scores the complete past blocks with its GQA group's
 *      summed query and keeps its own block plus the best k-1 others, without
 *      exponentials, ties to the lower block index ("MiniMax Sparse Attention",
 *      method and results paragraphs: per-GQA-group top-k over KV blocks,
 *      exp-free selection);
 *   3. exact causal attention softmax(q k^T * scale) v runs over the tokens of
 *      the selected blocks only ("MiniMax Sparse Attention", method paragraph;
 *      "Sparse Attention + Linear Backbones", section 5.5).
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - All tensor arguments are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or synchronises. Except for
 *    msa_sparse_attn_decode_noalloc, it keeps no mutable global state, so
 *    those entry points may be called from several host threads on different
 *    streams. msa_sparse_attn_decode_noalloc is the one exception: it keeps
 *    its scratch in one library-owned device array per GPU, and its calls
 *    must not overlap on the GPU (see its own comment). Every call is
 *    asynchronous on `stream`.
 *  - Host-side validation runs before any launch. It returns
 *    MSA_ERR_INVALID_ARG for null or misaligned pointers (16-byte alignment is
 *    required for every tensor) and inconsistent sizes, MSA_ERR_UNSUPPORTED
 *    for shapes outside the supported set, MSA_ERR_WORKSPACE when the
 *    workspace is smaller than msa_workspace_size() asks for, and MSA_ERR_CUDA
 *    when a launch fails. Nothing is launched on an error return.
 *  - Kernels that find bad device-side data (a page id outside
 *    [0, num_pages), a length beyond the cache's capacity, a block index out of
 *    range) set bits of *kv->status_word (MSA_DEV_* below) and skip that unit
 *    of work; its outputs are then unspecified. They never trap. The caller
 *    reads the status word after synchronising and clears it when it wishes.
 *  - Supported shapes: head_dim 64 or 128; block_size 64 or 128;
 *    G = num_q_heads / num_kv_heads an integer in 1..16; 1 <= top_k <= 256.
 *    bf16 attention needs head_dim 128; bf16 prefill attention needs G 8 or 16;
 *    decode selection (cu_q == NULL) needs max_blocks_per_seq <= 16384.
 *
 * Memory layout (all row-major)
 *  - K/V pages       : [num_pages][num_kv_heads][block_size][head_dim], dtype
 *  - centroids       : [num_pages][num_kv_heads][head_dim] fp32, page id as index
 *  - page_table      : [batch][max_blocks_per_seq] int32, logical block -> page
 *  - seq_lens        : [batch] int32, tokens in each sequence (after appends)
 *  - queries / out   : [rows][num_q_heads][head_dim], dtype
 *  - block_idx       : [rows][num_kv_heads][top_k] int32
 *  Query head h belongs to KV head floor(h / G).
 */
#ifndef MSA_H_
#define MSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* msa_stream_t;

typedef enum msa_status {
  MSA_OK = 0,
  MSA_ERR_INVALID_ARG = 1,
  MSA_ERR_UNSUPPORTED = 2,
  MSA_ERR_WORKSPACE = 3,
  MSA_ERR_CUDA = 4
} msa_status_t;

typedef enum msa_dtype { MSA_DTYPE_BF16 = 0, MSA_DTYPE_F32 = 1 } msa_dtype_t;

/* Bits set in *status_word by kernels that meet bad device-side data. */
#define MSA_DEV_BAD_PAGE 0x1u   /* page id outside [0, num_pages)                   */
#define MSA_DEV_BAD_LENGTH 0x2u /* length beyond capacity, or rows beyond seq_len   */
#define MSA_DEV_BAD_INDEX 0x4u  /* block index outside [0, own block] or unsorted   */
#define MSA_DEV_TIMEOUT 0x8u    /* a bounded device-side wait gave up               */
#define MSA_DEV_BOUNDS 0x10u    /* bounds-checked build only: an index derived from
                                   device data or a launch-size assumption fell
                                   outside its buffer; the access was skipped      */

/* The paged cache, passed by pointer. Host integers size the grids, so no
 * entry point reads device memory on the host. */
typedef struct msa_paged_kv {
  int32_t dtype;              /* msa_dtype_t of K/V pages, queries and outputs     */
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t block_size;         /* tokens per block == tokens per page              */
  int32_t batch;
  int32_t num_pages;
  int32_t max_blocks_per_seq; /* columns of page_table                            */
  void* k_pages;              /* device, see layout above                         */
  void* v_pages;              /* device                                           */
  float* centroids;           /* device, fp32                                     */
  const int32_t* page_table;  /* device                                           */
  const int32_t* seq_lens;    /* device                                           */
  uint32_t* status_word;      /* device, one word                                 */
} msa_paged_kv_t;

typedef enum msa_op {
  MSA_OP_SELECT = 0,
  MSA_OP_PREFILL = 1,
  MSA_OP_DECODE = 2,
  MSA_OP_SELECT_TOKENS = 3
} msa_op_t;

/*
 * msa_build_block_cache - append tokens to the paged cache and re-pool the
 * centroids of every block they touch.
 *
 * Follows "Art of Focus: Ling 2.0 ...", "Summarizing the Breakthrough": during
 * prefill the tokens are aggregated into block representations stored in the
 * cache, which shares the KV cache's page indexing; "Sparse Attention for
 * Long-Context LLMs: Evolution and Practical Deployment", section 7.3: cache
 * writes must stay consistent with the index, so every KV write here also
 * refreshes the block representation. The representation is the mean of the
 * block's keys over the tokens present, in fp32.
 *
 *   k_new, v_new      : device [N_new][num_kv_heads][head_dim], kv->dtype. The
 *                       rows of sequence b are cu_new[b] .. cu_new[b+1]-1.
 *   cu_new            : device [batch+1] int32, non-decreasing, cu_new[0] = 0.
 *   max_new_per_seq   : host bound on cu_new[b+1]-cu_new[b] (sizes the grid; a
 *                       sequence with more new rows is only partly appended,
 *                       which the bounds-checked build reports as
 *                       MSA_DEV_BOUNDS).
 *
 * kv->seq_lens must already count the new tokens: sequence b's new rows go to
 * positions seq_lens[b]-n_b .. seq_lens[b]-1. Writes those rows into the pages
 * named by page_table and recomputes, for each touched block j,
 *   centroids[page(b, j)][g][:] = (sum of the keys present in block j) / count
 * with a fixed summation order, so appending token by token gives the same
 * bits as pooling the full block at once. Untouched blocks are not read.
 */
msa_status_t msa_build_block_cache(const msa_paged_kv_t* kv, const void* k_new, const void* v_new,
                                   const int32_t* cu_new, int32_t max_new_per_seq,
                                   msa_stream_t stream);

/*
 * msa_select_topk - exp-free per-group top-k block selection.
 *
 * Follows "MiniMax Sparse Attention", method paragraph (a light index branch
 * scores KV blocks and independently keeps a top-k subset for each GQA group)
 * and results paragraph (exp-free top-k). For query row r at position t and KV
 * group g, with qbar = sum of the group's G query heads (fp32):
 *   score_j = qbar . centroid_j          for complete past blocks j < t / B;
 *   S(r, g) = {t / B} plus the min(k-1, t/B) best j under
 *             (score descending, block index ascending).
 *
 *   q                 : device [num_rows][num_q_heads][head_dim], kv->dtype.
 *   cu_q              : device [batch+1] int32 or NULL. With cu_q, the rows of
 *                       sequence b are cu_q[b] .. cu_q[b+1]-1 and sit at the
 *                       LAST n_b positions: seq_lens[b]-n_b .. seq_lens[b]-1.
 *                       NULL means decode: num_rows == batch, row b at
 *                       position seq_lens[b]-1.
 *   max_rows_per_seq  : host bound on n_b (sizes the grid; 1 for decode). Rows
 *                       of a sequence past this bound get no output (the
 *                       bounds-checked build reports MSA_DEV_BOUNDS).
 *   block_idx         : device out [num_rows][num_kv_heads][top_k] int32, the
 *                       selected logical blocks in ascending order, -1 padded.
 *   block_score       : device out, same shape, fp32, or NULL: the score of
 *                       each selected past block, +INF for the own block,
 *                       -INF for padding.
 *   workspace         : device scratch of msa_workspace_size(MSA_OP_SELECT,..)
 *                       bytes (may be NULL when that size is 0).
 */
msa_status_t msa_select_topk(const msa_paged_kv_t* kv, const void* q, const int32_t* cu_q,
                             int32_t num_rows, int32_t max_rows_per_seq, int32_t top_k,
                             int32_t* block_idx, float* block_score, void* workspace,
                             size_t workspace_bytes, msa_stream_t stream);

/*
 * msa_sparse_attn_prefill - exact attention of many query rows over their
 * selected blocks.
 *
 * Follows "MiniMax Sparse Attention", method paragraph (exact blockwise sparse
 * attention over the selected blocks only) and "Sparse Attention + Linear
 * Backbones", section 5.5 (softmax(q k_sel^T / sqrt(d)) v_sel). For row r at
 * position t and query head h in group g:
 *   U    = tokens u of the blocks in block_idx[r][g] with u <= t,
 *   out  = sum_{u in U} softmax_u(scale * q.k_u) v_u     (kv->dtype, RNE),
 *   lse  = log sum_{u in U} exp(scale * q.k_u)           (fp32, may be NULL).
 *
 *   q, cu_q, num_rows, max_rows_per_seq : as for msa_select_topk (cu_q must
 *                       not be NULL here).
 *   block_idx         : device [num_rows][num_kv_heads][top_k] int32, as
 *                       produced by msa_select_topk (ascending, -1 padded,
 *                       every entry <= t / B). U is a set: a block repeated
 *                       in the adjacent slot counts once; a row without any
 *                       block gives out = 0 (A = 0 before a gate) and
 *                       lse = -inf.
 *   out               : device [num_rows][num_q_heads][head_dim], kv->dtype.
 *   lse               : device [num_rows][num_q_heads] fp32, or NULL.
 *   workspace         : device scratch, msa_workspace_size(MSA_OP_PREFILL, ..).
 */
msa_status_t msa_sparse_attn_prefill(const msa_paged_kv_t* kv, const void* q, const int32_t* cu_q,
                                     int32_t num_rows, int32_t max_rows_per_seq,
                                     const int32_t* block_idx, int32_t top_k, float softmax_scale,
                                     void* out, float* lse, void* workspace,
                                     size_t workspace_bytes, msa_stream_t stream);

/*
 * msa_sparse_attn_decode - the same attention for one new query per sequence
 * (position seq_lens[b]-1, its own token already appended). One kernel: the
 * selection slots of all sequences and groups are split evenly over one wave
 * of resident CTAs; a (sequence, group) split over several CTAs is finished,
 * by log-sum-exp, by the CTA that holds its first blocks.
 *
 * Follows "Art of Focus: Ling 2.0 ...", "Summarizing the Breakthrough" (during
 * decode only the top-k relevant blocks are fetched) and the attention rule
 * above.
 *
 *   q                 : device [batch][num_q_heads][head_dim], kv->dtype.
 *   block_idx         : device [batch][num_kv_heads][top_k] int32, the same
 *                       rules as for prefill (ascending, -1 padded, an
 *                       adjacent repeat counts once, an empty row gives 0).
 *   out, lse          : device [batch][num_q_heads][head_dim] / [batch][num_q_heads].
 *   workspace         : device scratch, msa_workspace_size(MSA_OP_DECODE, ..):
 *                       one part per resident CTA (about 4 * SMs * G * 516
 *                       bytes, whatever the batch) and its flag. Its content
 *                       on entry does not matter; concurrent calls need
 *                       separate workspaces.
 */
msa_status_t msa_sparse_attn_decode(const msa_paged_kv_t* kv, const void* q,
                                    const int32_t* block_idx, int32_t top_k, float softmax_scale,
                                    void* out, float* lse, void* workspace, size_t workspace_bytes,
                                    msa_stream_t stream);

/*
 * msa_sparse_attn_prefill_gated / msa_sparse_attn_decode_gated - the two
 * attention calls above with the output gate fused into their epilogues:
 *
 *   O = g * A + (1 - g) * X
 *
 * where A is the sparse attention output. Follows "Sparse Attention for
 * Long-Context LLMs: Evolution and Practical Deployment", section 4.3 (step 6
 * of the computation flow: the gate weights the sparse attention output
 * against the original representation; it may be a scalar or vary with the
 * dimension). The gate values are the caller's (a learned gate is applied
 * before the call); the library does not compute them. A is not rounded
 * before the gate: the result is rounded to kv->dtype once.
 *
 *   gate          : device fp32, [rows][num_q_heads] (gate_per_dim = 0: one
 *                   value per row and head) or [rows][num_q_heads][head_dim]
 *                   (gate_per_dim = 1); rows = num_rows (prefill) or batch
 *                   (decode). 4-byte aligned.
 *   x             : device [rows][num_q_heads][head_dim] in kv->dtype, the
 *                   other branch (the query itself, or a residual). 16-byte
 *                   aligned. May alias q, not out.
 *   lse           : the attention's log-sum-exp, not gated.
 *   other arguments, workspace and errors: as for the ungated calls;
 *   MSA_ERR_INVALID_ARG also for a NULL or misaligned gate or x, or
 *   gate_per_dim not 0 or 1.
 */
msa_status_t msa_sparse_attn_prefill_gated(const msa_paged_kv_t* kv, const void* q,
                                           const int32_t* cu_q, int32_t num_rows,
                                           int32_t max_rows_per_seq, const int32_t* block_idx,
                                           int32_t top_k, float softmax_scale, const float* gate,
                                           int32_t gate_per_dim, const void* x, void* out,
                                           float* lse, void* workspace, size_t workspace_bytes,
                                           msa_stream_t stream);

msa_status_t msa_sparse_attn_decode_gated(const msa_paged_kv_t* kv, const void* q,
                                          const int32_t* block_idx, int32_t top_k,
                                          float softmax_scale, const float* gate,
                                          int32_t gate_per_dim, const void* x, void* out,
                                          float* lse, void* workspace, size_t workspace_bytes,
                                          msa_stream_t stream);

/*
 * msa_sparse_attn_decode_noalloc - msa_sparse_attn_decode for callers that
 * cannot allocate device memory at the call: a plugin run by a host framework
 * that owns the device memory pool and offers no scratch allocator, or a
 * latency-bound loop that must not call the allocator. The pages describe no
 * such call; it exists for those callers only.
 *
 * Same arguments and results as msa_sparse_attn_decode minus the workspace:
 * the per-CTA parts and flags go to one 8 MiB device array inside libmsa.so,
 * which every GPU that loads the library keeps until the process exits.
 *  - Bad arguments give the same status as msa_sparse_attn_decode, checked
 *    before anything else (the array is not looked up).
 *  - The decode workspace does not grow with the batch (at most about
 *    4 * SMs * 16 * 516 bytes, under 5 MiB on 148 SMs), so every supported
 *    shape fits; MSA_ERR_WORKSPACE (nothing launched) is returned only if
 *    msa_workspace_size(MSA_OP_DECODE, ...) ever exceeded 8 MiB.
 *  - All calls on a device share the array: calls whose kernels may overlap
 *    on the GPU (unordered streams) race; calls on one stream do not. Nothing
 *    in the array needs to start at zero.
 *  - The first call on each device resolves the array's device address
 *    (cudaGetSymbolAddress, with that device current); make it before any
 *    stream capture.
 *  - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 */
msa_status_t msa_sparse_attn_decode_noalloc(const msa_paged_kv_t* kv, const void* q,
                                            const int32_t* block_idx, int32_t top_k,
                                            float softmax_scale, void* out, float* lse,
                                            msa_stream_t stream);

/*
 * msa_select_tokens / msa_sparse_attn_decode_tokens - the token-granular
 * variant for one new query per sequence (decode): a lightweight indexer
 * scores every earlier position and the attention runs over the kept
 * positions only.
 *
 * Follows "Sparse Attention + Linear Backbones: How LLM Long-Context
 * Architectures Are Evolving", sections 5.1-5.3 and 5.5 (an indexer without
 * positional encoding rates all earlier positions; top-K positions are
 * kept; attention over those positions). The page leaves the indexer's form
 * open; it is read here like the block score: for the query at t = seq_lens[b]-1
 *   s(u) = sum_h qi[b][h] . ki[u]        (u < t; fp32: the heads summed left to
 *                                         right, an fma chain over each
 *                                         16-byte chunk of the key, then the
 *                                         chunks' sums added pairwise),
 *   kept = {t} plus the top_k-1 best u < t (all of them when t < top_k),
 *          ties to the lower position.
 *
 *   ki_pages          : device [num_pages][block_size][head_dim], kv->dtype:
 *                       one indexer key per position, paged with kv's page
 *                       table (written by the caller).
 *   qi                : device [batch][num_index_heads][head_dim], kv->dtype.
 *   tok_idx           : device out [batch][top_k] int32, the kept positions
 *                       ascending (t last), -1 padded.
 *   workspace         : device scratch, msa_workspace_size(MSA_OP_SELECT_TOKENS,
 *                       kv, batch, 1, top_k) bytes (one fp32 score per position).
 *
 * msa_sparse_attn_decode_tokens: out / lse as for msa_sparse_attn_decode, over
 * the positions listed in tok_idx[b] (shared by all KV groups; -1 padding, a
 * position repeated in the adjacent slot counts once, a row without any
 * position gives 0 and lse = -inf).
 */
msa_status_t msa_select_tokens(const msa_paged_kv_t* kv, const void* ki_pages, const void* qi,
                               int32_t num_index_heads, int32_t top_k, int32_t* tok_idx,
                               void* workspace, size_t workspace_bytes, msa_stream_t stream);

msa_status_t msa_sparse_attn_decode_tokens(const msa_paged_kv_t* kv, const void* q,
                                           const int32_t* tok_idx, int32_t top_k,
                                           float softmax_scale, void* out, float* lse,
                                           msa_stream_t stream);

/*
 * msa_select_tokens_rows / msa_sparse_attn_prefill_tokens - the same two
 * steps for many query rows per sequence (prefill, chunked prefill): the rows
 * cu_q[b] .. cu_q[b+1]-1 of sequence b sit at its last n_b positions, as for
 * msa_select_topk with cu_q. Row r at position t scores the positions u < t
 * and keeps t plus the best top_k-1 of them; the attention of row r runs over
 * its own kept positions (rows share no keys, so each row gathers its own).
 *
 *   qi        : device [num_rows][num_index_heads][head_dim], kv->dtype.
 *   q, out    : device [num_rows][num_q_heads][head_dim]; lse [num_rows][num_q_heads].
 *   tok_idx   : device [num_rows][top_k] int32, ascending (t last), -1 padded.
 *   workspace : msa_workspace_size(MSA_OP_SELECT_TOKENS, kv, num_rows,
 *               max_rows_per_seq > 1, top_k) bytes: one fp32 score per row
 *               and position (num_rows * max_blocks_per_seq * block_size * 4).
 *   num_rows <= 65535; cu_q must not be NULL. Errors as for the decode form.
 */
msa_status_t msa_select_tokens_rows(const msa_paged_kv_t* kv, const void* ki_pages,
                                    const void* qi, const int32_t* cu_q, int32_t num_rows,
                                    int32_t num_index_heads, int32_t top_k, int32_t* tok_idx,
                                    void* workspace, size_t workspace_bytes, msa_stream_t stream);

msa_status_t msa_sparse_attn_prefill_tokens(const msa_paged_kv_t* kv, const void* q,
                                            const int32_t* cu_q, int32_t num_rows,
                                            const int32_t* tok_idx, int32_t top_k,
                                            float softmax_scale, void* out, float* lse,
                                            msa_stream_t stream);

/*
 * Context-sharded decode: the blocks of every sequence are split over several
 * ranks (GPUs) by block range, each rank holding the K/V pages and centroids
 * of its range [block_lo, block_hi). "Sparse Attention for Long-Context LLMs:
 * Evolution and Practical Deployment", section 8 (future directions) lists
 * sharing index results across devices and layers; the split follows the
 * method's own structure: a rank scores only its blocks, the ranks' best
 * candidates are gathered and the global top-k picked from them, each rank
 * attends over the chosen blocks it holds, and the partial results are merged
 * by log-sum-exp. The gathers between ranks are the caller's (NCCL all-gather
 * in the Python binding); these calls are the per-rank steps.
 *
 * A rank's cache: page_table[b][j] holds the page of GLOBAL block j when j is
 * in the rank's range (other entries are not read), seq_lens the global
 * lengths, the new token appended by the rank whose range holds it.
 *
 * msa_select_topk_range: decode rows (one per sequence, at seq_lens-1); the
 *   candidates are the complete past blocks j in [block_lo, block_hi). Writes
 *   cand_keys [batch][num_kv_heads][top_k-1] u64: the rank's best min(k-1,
 *   candidates) selection keys, descending (0 pads). A key is the block's fp32
 *   score in order-preserving bits << 32 | (0x7fffffff - j): one unsigned
 *   compare orders (score desc, index asc). 1 <= top_k <= 65. Workspace as
 *   for msa_select_topk with cu_q == NULL.
 * msa_select_merge: cand_keys [num_lists][batch][num_kv_heads][top_k-1] (the
 *   ranks' lists, gathered in rank order) -> block_idx / block_score exactly as
 *   msa_select_topk would produce them for the unsharded sequence.
 * msa_sparse_attn_decode_range: the decode attention restricted to the
 *   selected blocks in [block_lo, block_hi): o_part [batch][num_q_heads]
 *   [head_dim] fp32 (normalised over this rank's keys, 0 if none) and lse_part
 *   [batch][num_q_heads] (natural log, -inf if none). Workspace as for
 *   msa_sparse_attn_decode; bf16 and head_dim 128 only.
 * msa_lse_merge: o_parts [num_parts][rows][head_dim] fp32 and lse_parts
 *   [num_parts][rows] -> out [rows][head_dim] (out_dtype, RNE) and lse [rows]
 *   (may be NULL): sum_p exp(lse_p - M) o_p / sum_p exp(lse_p - M).
 */
msa_status_t msa_select_topk_range(const msa_paged_kv_t* kv, const void* q, int32_t block_lo,
                                   int32_t block_hi, int32_t top_k, uint64_t* cand_keys,
                                   void* workspace, size_t workspace_bytes, msa_stream_t stream);

msa_status_t msa_select_merge(const msa_paged_kv_t* kv, const uint64_t* cand_keys,
                              int32_t num_lists, int32_t top_k, int32_t* block_idx,
                              float* block_score, msa_stream_t stream);

msa_status_t msa_sparse_attn_decode_range(const msa_paged_kv_t* kv, const void* q,
                                          const int32_t* block_idx, int32_t top_k,
                                          int32_t block_lo, int32_t block_hi, float softmax_scale,
                                          float* o_part, float* lse_part, void* workspace,
                                          size_t workspace_bytes, msa_stream_t stream);

msa_status_t msa_lse_merge(const float* o_parts, const float* lse_parts, int32_t num_parts,
                           int32_t rows, int32_t head_dim, int32_t out_dtype, void* out,
                           float* lse, msa_stream_t stream);

/* Scratch bytes that `op` needs for these sizes (num_rows / max_rows_per_seq
 * as passed to the op; batch and 1 for decode). 0 means no scratch. */
size_t msa_workspace_size(msa_op_t op, const msa_paged_kv_t* kv, int32_t num_rows,
                          int32_t max_rows_per_seq, int32_t top_k);

/* Static, NUL-terminated description of a status code. */
const char* msa_status_string(msa_status_t status);

/* Library ABI version (major * 1000 + minor). */
int32_t msa_version(void);

/* How this copy of the library was compiled: a mask of MSA_BUILD_* bits.
 *  MSA_BUILD_DEBUG_BOUNDS: the bounds-checked build (compiled with
 *    -DMSA_DEBUG_BOUNDS, shipped as libmsa_debug.so beside libmsa.so). Every
 *    shared- or global-memory index that a kernel derives from device data
 *    (cu_q / cu_seqlens entries, block and token indices, plan and order
 *    tables the library writes itself) or from a launch-size assumption is
 *    compared with the extent of its buffer before the access; a failed check
 *    sets MSA_DEV_BOUNDS in *kv->status_word and skips the access (a TMA
 *    coordinate is replaced by a valid one so that the pipeline stays in
 *    step) instead of faulting. Outputs are identical to the regular build's
 *    when no check fails. It is a debugging aid that stands in for a memory
 *    checker and costs a few percent of speed; the regular build compiles the
 *    checks to nothing. */
#define MSA_BUILD_DEBUG_BOUNDS 0x1
int32_t msa_build_flags(void);

/* Self-test of the bounded device waits. Every wait of the library's kernels
 * on another agent (an mbarrier phase completed by TMA copies or other warps,
 * a flag another CTA publishes) gives up after about one second, sets
 * MSA_DEV_TIMEOUT in the status word and lets the kernel return. This call
 * launches one small kernel that runs such a wait on something never
 * completed - which = 0: an mbarrier phase nothing arrives at; which = 1: a
 * flag word nothing writes - so that after about one second *status_word has
 * MSA_DEV_TIMEOUT set and the context is still usable.
 *   status_word : device pointer to a uint32 (4-byte aligned).
 * Returns MSA_ERR_INVALID_ARG for a NULL or misaligned status_word or which
 * not 0 or 1, MSA_ERR_CUDA if the launch fails. */
msa_status_t msa_selftest_bounded_wait(int32_t which, uint32_t* status_word, msa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H_ */
