// Self-test of the bounded device waits (msa_selftest_bounded_wait).
//
// Every wait of the library's kernels on another agent - an mbarrier phase
// that TMA copies or other warps complete, or a flag another CTA publishes -
// gives up after about one second of %globaltimer time, records
// MSA_DEV_TIMEOUT in the status word and lets the kernel return, so a lost
// completion costs a second and an error status, never a hung GPU. This file
// runs those same waits (mbar_wait and wait_flag from tma.cuh) on something
// that is never completed: an mbarrier nothing arrives at, and a flag word
// nothing writes. Nothing is in flight when they give up (no copy was issued),
// so the kernel returns normally and the context stays usable.
#include "tma.cuh"

namespace msa {

namespace {

// never written: a flag that no CTA publishes
__device__ __align__(8) uint64_t g_never_published = 0;

__global__ void __launch_bounds__(32) selftest_wait_kernel(int which, uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  if (which == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
    if (!mbar_wait(&bar, 0)) report(status, MSA_DEV_TIMEOUT);  // nothing arrives
  } else {
    if (!wait_flag(&g_never_published, 1ull, global_timer_ns())) report(status, MSA_DEV_TIMEOUT);
  }
}

}  // namespace

cudaError_t selftest_wait(int which, uint32_t* status, cudaStream_t st) {
  selftest_wait_kernel<<<1, 32, 0, st>>>(which, status);
  return cudaGetLastError();
}

}  // namespace msa
