// debug.cu -- a test hook for failure detection. One thread waits on a flag
// with the bounded acquire loop that the library's cross-CTA waits use
// (%globaltimer limit, acquire loads), and reports a time-out through the
// context's device status word instead of trapping or spinning on. A test sets
// no flag, reads MOE_DEV_TIMEOUT back on the host, and keeps using the context.
#include "common.cuh"

namespace moe {

namespace {

// Bounded twice: by the clock, and by an iteration count (2^24 acquire loads,
// seconds at most) that ends the loop even if the clock did not advance.
__global__ void debug_wait_flag_kernel(const int* flag, uint64_t limit_ns, int* status) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0; ld_acquire_gpu(flag) == 0; ++it) {
    if (global_timer_ns() - t0 > limit_ns || it >= (1u << 24)) {
      flag_status(status, MOE_DEV_TIMEOUT);
      return;
    }
  }
}

}  // namespace

cudaError_t launch_debug_wait_flag(const int* flag, uint64_t limit_ns, int* status, cudaStream_t s) {
  debug_wait_flag_kernel<<<1, 1, 0, s>>>(flag, limit_ns, status);
  return cudaGetLastError();
}

}  // namespace moe
