// Allocation-free decode attention: msa_sparse_attn_decode with its scratch
// (one attention part and one flag per resident CTA) in a fixed device array
// owned by the library.
//
// Who needs this: callers that cannot allocate device memory at the point of
// the call - for instance a plugin invoked from a host framework that owns the
// whole device memory pool and gives its plugins no scratch allocator, or a
// latency-critical loop that must not touch the allocator (cudaMalloc can
// synchronise the device). They pass only inputs and outputs; the partial
// results of the attention kernel live in g_decode_scratch below.
//
// Costs and rules of use:
//  * the array is kNoAllocScratchBytes (8 MiB) of device memory that every
//    GPU which loads libmsa.so holds until the process exits;
//  * the decode workspace is bounded by the resident grid, not the batch
//    (under 5 MiB on 148 SMs at 16 query heads per group), so every supported
//    shape fits; a problem that needed more than 8 MiB would be rejected with
//    MSA_ERR_WORKSPACE before anything is launched;
//  * all calls on a device share the one array, so two calls whose kernels
//    overlap on the GPU (different streams without ordering between them)
//    race on it; calls on one stream are safe. A part is read only after its
//    flag carries the reading call's own tag, so nothing has to start at zero
//    and the contents left by the previous call do not matter;
//  * the first call on each device looks up the array's device address with
//    cudaGetSymbolAddress (the host-side name of a __device__ array is not a
//    device address); make that first call before any stream capture.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 8u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_decode_scratch on the current device (set up once per
// device, with that device current). nullptr on failure.
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" msa_status_t msa_sparse_attn_decode_noalloc(const msa_paged_kv_t* kv, const void* q,
                                                       const int32_t* block_idx, int32_t top_k,
                                                       float softmax_scale, void* out, float* lse,
                                                       msa_stream_t stream) {
  // bad arguments are reported as such, before the scratch array is looked up
  const msa_status_t s =
      msa::check_decode_args(kv, q, block_idx, top_k, softmax_scale, out, lse);
  if (s != MSA_OK) return s;
  const size_t need = msa_workspace_size(MSA_OP_DECODE, kv, kv->batch, 1, top_k);
  if (need > kNoAllocScratchBytes) return MSA_ERR_WORKSPACE;
  void* scratch = scratch_on_current_device();
  if (!scratch) return MSA_ERR_CUDA;
  return msa_sparse_attn_decode(kv, q, block_idx, top_k, softmax_scale, out, lse, scratch,
                                kNoAllocScratchBytes, stream);
}
