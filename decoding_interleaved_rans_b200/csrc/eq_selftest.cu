// eq_selftest_bounded_wait: shows that a copy that never lands ends in a status, not a hang.
//
// The decoders wait on mbarriers for their own bulk copies only, always through
// mbar_wait_bounded, which gives up after about a second; the warp then records EQ_DEV_TIMEOUT
// and stops.  No input through the decode calls can make a copy fail to land, so this kernel
// arms a barrier for 16 bytes that no copy will deliver (nothing is in flight) and waits on it
// with the same bounded wait.
#include "eq_internal.cuh"

namespace eq {

__global__ void __launch_bounds__(32) selftest_wait_kernel(uint32_t *status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_expect_tx(&bar, 16);  // the one arrival, and 16 bytes that never come
  }
  __syncwarp();
  const bool landed = mbar_wait_bounded(&bar, 0);
  if (threadIdx.x == 0 && !landed) report(status, EQ_DEV_TIMEOUT);
}

}  // namespace eq

using namespace eq;

extern "C" eq_status eq_selftest_bounded_wait(uint32_t *d_status, void *stream) {
  if (!d_status) return EQ_ERR_ARG;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(d_status);
  return cuda_status(cudaGetLastError());
}
