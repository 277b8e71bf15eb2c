// selftest.cu -- a kernel whose bounded wait is meant to run out: one thread waits on an
// mbarrier that nothing arrives on, with a short limit, then records its fault code and
// returns. It exercises the path every real wait takes when it gives up (fault word,
// early return, a context that stays usable) without faulting or hanging the GPU.
#include "sm100_async.cuh"

namespace {

using namespace lbq;

constexpr unsigned kFaultSelfTest = 11;

__global__ void wait_selftest_kernel(unsigned* fault, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
    // phase 0 never completes: the wait gives up after limit_ns
    mbar_wait(b, 0, fault, kFaultSelfTest, /*give_up_after_fault=*/false, limit_ns);
  }
}

}  // namespace

cudaError_t lbq_launch_wait_selftest(cudaStream_t s) {
  unsigned* fault = lbq_fault_word();
  if (!fault) return cudaErrorInvalidDevicePointer;
  wait_selftest_kernel<<<1, 32, 0, s>>>(fault, 20ull * 1000 * 1000);  // 20 ms
  return cudaGetLastError();
}
