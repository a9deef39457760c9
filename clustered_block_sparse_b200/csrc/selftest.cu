// Failure-path self-test: a bounded wait that nothing completes.
//
// Every wait in the library's kernels gives up after a bounded time, latches
// EAR_ERR_TIMEOUT in the device status word and lets the kernel return, so a
// lost producer or a stuck peer costs one error status instead of a hung GPU.
// This entry point exercises exactly that path on purpose: one warp waits on
// an mbarrier with no arrivals, the wait runs out, the status is latched and
// the kernel ends normally.  No fault, trap or unbounded loop is involved.
#include "ear_internal.cuh"
#include "sm100.cuh"

namespace ear {
namespace {

__global__ void st_wait_timeout(int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);  // one arrival expected; none ever comes
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  const bool ok = sm100::mbar_wait_warp(&bar, 0, &abort_flag);
  if (!ok && threadIdx.x == 0) latch(status, EAR_ERR_TIMEOUT);
}

}  // namespace
}  // namespace ear

extern "C" ear_status ear_selftest_wait_timeout(void* stream) {
  int* word = ear::device_status_word();
  if (word == nullptr) return EAR_ERR_CUDA;
  ear::st_wait_timeout<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(word);
  return ear::after_launch();
}
