// Diagnostics entry point: exercises the bounded-wait path that every kernel
// with an mbarrier wait relies on, without a fault. One warp waits (through
// the same tc::mbar_wait) on an mbarrier that nothing ever arrives on; after
// `limit_cycles` SM clock cycles the wait gives up, records LH_ERR_TIMEOUT in
// the device error word and the kernel returns normally.
#include "tc_ptx.cuh"

namespace lh {
namespace {

constexpr int kSelftestSite = 900;

__global__ void k_wait_unarrived(long long limit_cycles, int* err, int* gave_up) {
  __shared__ uint64_t bar;
  __shared__ tc::Abort ab;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);          // expects one arrival; none is ever made
    tc::fence_mbar_init();
    ab.flag = 0;
  }
  __syncthreads();
  const bool ok = tc::mbar_wait(&bar, 0, &ab, err, kSelftestSite, limit_cycles);
  if (threadIdx.x == 0) *gave_up = ok ? 0 : 1;
}

}  // namespace

cudaError_t launch_selftest_wait(long long limit_cycles, int* err, int* gave_up, cudaStream_t s) {
  k_wait_unarrived<<<1, 32, 0, s>>>(limit_cycles, err, gave_up);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lh
