// Failure-detection self-test: a bounded mbarrier wait that nothing completes.
//
// One CTA initialises an mbarrier that no thread or copy ever arrives at and
// waits on its first phase, polling it with try_wait the way the layer's
// kernels do.  The wait gives up after `limit_ns` of global time (and, as a
// second bound, after a fixed number of polls), records the timeout code in
// the error word and returns, so the context stays usable and the host reads
// the code with gsa_get_status.  Nothing here faults, traps or spins without
// a bound.
#include "gsa_kernels.h"
#include "tc_ptx.cuh"

namespace gsa {

namespace {

__global__ void __launch_bounds__(32) expire_wait_kernel(int* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(b, 1);
    tc::fence_mbar_init();
  }
  __syncwarp();
  const unsigned long long t0 = tc::gtimer();
  bool done = false;
#pragma unroll 1
  for (int i = 0; i < (1 << 22) && !done; ++i) {
    if (tc::mbar_try_wait(b, 0)) done = true;                 // never: nothing arrives
    else if (tc::gtimer() - t0 > limit_ns) break;
  }
  if (!done && threadIdx.x == 0) set_error(err, ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_expire_wait(int* err, unsigned long long limit_ns, cudaStream_t st) {
  expire_wait_kernel<<<1, 32, 0, st>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace gsa
