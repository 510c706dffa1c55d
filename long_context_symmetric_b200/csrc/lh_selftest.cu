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

// 2^x of n inputs two ways: the FMA-pipe polynomial the attention softmax uses
// for part of its exponentials, and the special-function unit's ex2.approx.
__global__ void k_exp2_pair(const float* __restrict__ x, float* __restrict__ y_fma, float* __restrict__ y_sfu,
                            int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = i + 1 < n ? x[i + 1] : 0.f;
  const float2 r = tc::exp2_fma2(make_float2(a, b));
  y_fma[i] = r.x;
  y_sfu[i] = tc::ex2(a);
  if (i + 1 < n) {
    y_fma[i + 1] = r.y;
    y_sfu[i + 1] = tc::ex2(b);
  }
}

}  // namespace

cudaError_t launch_selftest_exp2(const float* x, float* y_fma, float* y_sfu, int n, cudaStream_t s) {
  const int pairs = (n + 1) / 2;
  k_exp2_pair<<<(pairs + 255) / 256, 256, 0, s>>>(x, y_fma, y_sfu, n);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_selftest_wait(long long limit_cycles, int* err, int* gave_up, cudaStream_t s) {
  k_wait_unarrived<<<1, 32, 0, s>>>(limit_cycles, err, gave_up);
  count_launch();
  return cudaGetLastError();
}

}  // namespace lh
