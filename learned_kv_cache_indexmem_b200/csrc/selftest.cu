// selftest.cu -- exercises the failure path of the bounded device waits
// without a fault: one CTA waits on a transaction barrier that nothing
// completes, through the same bounded-wait helper every kernel uses; the wait
// ends after the given limit and records a timeout in the context's error
// word, which imem_sync reports. Nothing hangs and nothing faults.
#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace imem {
namespace {

__global__ void wait_selftest_kernel(long long limit, int* err) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = tc::smem_addr(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(b, 1);
    tc::fence_mbar_init();
  }
  __syncthreads();
  // nothing arrives on the barrier: phase 0 never completes
  if (!tc::mbar_wait(b, 0, limit) && threadIdx.x == 0) record_error(err, DEV_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_selftest(const Ctx& c, long long limit, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(limit, c.err);
  return cudaGetLastError();
}

}  // namespace imem
