// Shared device helpers of libmsa (internal header).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "msa.h"

namespace msa {

typedef __nv_bfloat16 bf16;

// Bounded spin limit for every device-side wait (mbarrier polls). At a few
// hundred ns per poll this is well above any legitimate wait and well below a
// second, after which the kernel records MSA_DEV_TIMEOUT and unwinds.
constexpr uint32_t kSpinLimit = 1u << 22;

// Programmatic dependent launch. A kernel launched with launch_pdl may begin
// while its predecessor on the stream is still running: it calls pdl_wait()
// before it touches global memory (which returns once the predecessor has
// completed and its writes are visible) and pdl_release() once its last
// global write is done, which lets its successor launch as the CTAs drain
// (released earlier, waiting successor CTAs were measured to slow the running
// kernel). Both are no-ops for an ordinary launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... P, typename... A>
inline cudaError_t launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, A&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

// Host-side checks shared by the decode attention entry points (msa_api.cu).
msa_status_t check_decode_args(const msa_paged_kv_t* kv, const void* q, const int32_t* block_idx,
                               int32_t top_k, float softmax_scale, const void* out,
                               const float* lse);

__device__ __forceinline__ void report(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

// Bounds-checked build. Compiled with -DMSA_DEBUG_BOUNDS (libmsa_debug.so),
// every index a kernel derives from device data or from a launch-size
// assumption goes through MSA_IN_BOUNDS / MSA_RANGE_OK before the access it
// guards: a failed check records MSA_DEV_BOUNDS and the caller skips the
// access (or substitutes a valid index where a pipeline must stay in step).
// In the regular build both macros are the constant true and their
// arguments are not evaluated, so the checks cost nothing there.
#ifdef MSA_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
__device__ __forceinline__ bool debug_range_ok(long long lo, long long hi, long long n,
                                               uint32_t* status) {
  const bool ok = 0 <= lo && lo <= hi && hi <= n;
  if (!ok) report(status, MSA_DEV_BOUNDS);
  return ok;
}
// 0 <= i < n
#define MSA_IN_BOUNDS(i, n, status) \
  ::msa::debug_range_ok((long long)(i), (long long)(i) + 1, (long long)(n), (status))
// 0 <= lo <= hi <= n: the half-open range [lo, hi) lies inside [0, n)
#define MSA_RANGE_OK(lo, hi, n, status) \
  ::msa::debug_range_ok((long long)(lo), (long long)(hi), (long long)(n), (status))
#else
constexpr bool kDebugBounds = false;
#define MSA_IN_BOUNDS(i, n, status) true
#define MSA_RANGE_OK(lo, hi, n, status) true
#endif

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<bf16>(bf16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

// Position of query row i of sequence b: the rows are the last n_b tokens.
__device__ __forceinline__ int row_position(int seq_len, int n_rows, int i) {
  return seq_len - n_rows + i;
}

// ---------------------------------------------------------------------------
// Canonical block score. Every selection kernel computes
//   qbar[i]  = q_{h0}[i] + q_{h0+1}[i] + ... (left to right over the group's heads)
//   score    = fma(qbar[D-1], c[D-1], ... fma(qbar[1], c[1], fma(qbar[0], c[0], 0)))
// i.e. one fp32 fma chain in coordinate order, so a row scored by the prefill
// kernel and the same row scored by the decode kernel give identical bits,
// and identical centroids give identical scores (exact ties).
// ---------------------------------------------------------------------------
// Orderable 64-bit selection key: larger key = better (higher score, then
// lower block index). 0 is below every real key.
__device__ __forceinline__ uint64_t sel_key(float s, int j) {
  if (s == 0.f) s = 0.f;  // one key for +0 and -0
  uint32_t b = __float_as_uint(s);
  b = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return ((uint64_t)b << 32) | (uint32_t)(0x7fffffff - j);
}
__device__ __forceinline__ int key_block(uint64_t k) { return 0x7fffffff - (int)(uint32_t)k; }
__device__ __forceinline__ float key_score(uint64_t k) {
  uint32_t b = (uint32_t)(k >> 32);
  b = (b & 0x80000000u) ? (b & 0x7fffffffu) : ~b;
  return __uint_as_float(b);
}

// Output gate fused into the attention epilogues ("Sparse Attention for
// Long-Context LLMs: Evolution and Practical Deployment", section 4.3, step 6
// of the computation flow): O = g * A + (1 - g) * X with g and X from the
// caller (the gate may be a scalar or vary with the dimension); g is one value per (row, head), or one per (row, head, coordinate)
// when per_dim is set. g == nullptr: no gate, O = A.
struct gate_t {
  const float* g = nullptr;
  const void* x = nullptr;
  int per_dim = 0;
};

// head = row * num_q_heads + query head; c = coordinate; a = attention output
template <typename T>
__device__ __forceinline__ float gate_apply(const gate_t& gt, size_t head, int c, int D, float a) {
  if (!gt.g) return a;
  const float gv = gt.per_dim ? gt.g[head * D + c] : gt.g[head];
  const float xv = to_f32(reinterpret_cast<const T*>(gt.x)[head * D + c]);
  return fmaf(gv, a - xv, xv);
}

}  // namespace msa
