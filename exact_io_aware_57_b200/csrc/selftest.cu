// Self-tests.  (1) The failure path every kernel shares: a bounded mbarrier wait
// that gives up, raises the CTA's abort flag and records ATTN_ERR_TIMEOUT in
// the device status word, after which the kernel returns normally and the
// context stays usable.  The kernel waits on a barrier that nothing arrives
// on, with a caller-chosen (short) limit -- no fault, no hang.  (2) The
// FMA-pipe exponential ex2_poly that the kernels use for a share of their
// exponentials, evaluated elementwise so that its error can be measured
// against exact 2^x.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace attn {
namespace {

__global__ void __launch_bounds__(32) wait_selftest_kernel(int* status, long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncwarp();
  const Abort ab{&abort_flag, status, limit};
  if (threadIdx.x == 0) {
    const bool done = mbar_wait(&bar, 0, ab);  // phase 0 never completes
    if (done) atomicExch(status, ATTN_ERR_CUDA);  // cannot happen: flag it if it does
  }
}

__global__ void __launch_bounds__(256) ex2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y,
                                                           long long n) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n; i += stride)
    y[i] = ex2_poly(x[i]);
}

}  // namespace

int launch_ex2_selftest(const float* x, float* y, long long n, cudaStream_t st) {
  const long long blocks = std::min<long long>((n + 255) / 256, 148LL * 8);
  ex2_selftest_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(x, y, n);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

int launch_wait_selftest(long long limit_cycles, cudaStream_t st) {
  int* status = device_status_ptr();
  if (!status) return ATTN_ERR_CUDA;
  wait_selftest_kernel<<<1, 32, 0, st>>>(status, limit_cycles);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? ATTN_OK : ATTN_ERR_CUDA;
}

}  // namespace attn
