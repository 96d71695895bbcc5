// selftest.cu -- a check of the bounded device wait that every kernel of the
// library uses for its mbarrier hand-offs (a wait that gives up after a fixed
// number of polls, writes CSKV_ERR_TIMEOUT into the caller's status word and
// lets the kernel return, so a lost arrival never hangs the GPU).
//
// One warp initialises an mbarrier in shared memory with one expected arrival.
// With `arrive` set, lane 0 arrives before the wait, which must then succeed;
// without it nothing ever arrives and no asynchronous copy is in flight, so
// the wait runs out after `spin_limit` polls and reports the timeout.
#include "cskv_device.cuh"
#include "cskv_internal.h"

namespace cskv {
namespace {

__global__ void __launch_bounds__(32) wait_selftest_kernel(int arrive, uint32_t spin_limit, int32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (arrive && threadIdx.x == 0) mbar_arrive(&bar);
  __syncwarp();
  // every lane waits (as the consumer warps of the kernels do); the first failure wins the status word
  mbar_wait_limit(&bar, 0u, status, spin_limit);
}

}  // namespace

cudaError_t launch_wait_selftest(int arrive, uint32_t spin_limit, int32_t* status, cudaStream_t st) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(arrive, spin_limit, status);
  return cudaGetLastError();
}

}  // namespace cskv
