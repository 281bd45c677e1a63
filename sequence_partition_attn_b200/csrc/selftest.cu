// selftest.cu -- exercises the bounded device-side wait that every pipeline barrier of the
// library uses: a block waits on an mbarrier that nothing completes, with a short limit.
// Warp 0 waits with the whole-warp form (the MMA issuer's), warp 1 with the per-thread form
// (the softmax's); the first to give up records PA_ETIMEOUT in the context status word and
// raises the block's abort flag, which ends the other wait at once.  No fault, no hang:
// both waits return within the limit.
#include "pa_device.cuh"
#include "pa_launch.h"

namespace pa {
namespace {

__global__ void __launch_bounds__(64) wait_selftest_kernel(int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar_storage;
  __shared__ int abort_flag;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);          // one arrival expected; none ever comes
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* af = &abort_flag;
  if (threadIdx.x < 32) mbar_wait_warp(bar, 0, af, status, limit_ns);
  else mbar_wait(bar, 0, af, status, limit_ns);
}

}  // namespace

int launch_wait_selftest(int* status, uint64_t limit_ns, cudaStream_t st) {
  wait_selftest_kernel<<<1, 64, 0, st>>>(status, limit_ns);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace pa
