// Self-test of the bounded-wait path: a kernel whose wait can never be
// satisfied must give up on its own, record the failure in the error word and
// return, leaving the CUDA context usable. This is how every wait in the
// library behaves when a logic error would otherwise leave it spinning.
#include "exp2_poly.cuh"
#include "isa_internal.h"
#include "ptx.cuh"

namespace isa {
namespace {

__global__ void wait_selftest_kernel(uint32_t* err, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  mbar_fence_init();
  // nothing ever arrives on `bar`: phase 0 never completes
  if (!mbar_wait(&bar, 0, timeout_ns)) atomicOr(err, kErrSelftest);
}

// The polynomial 2^x used by the attention softmax, next to CUDA's exp2f, for testing.
__global__ void exp2_selftest_kernel(const float* x, float* y_poly, float* y_ref, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  y_poly[i] = exp2_poly(x[i]);
  y_ref[i] = exp2f(x[i]);
}

}  // namespace

cudaError_t launch_exp2_selftest(const float* x, float* y_poly, float* y_ref, int n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  exp2_selftest_kernel<<<(n + 255) / 256, 256, 0, s>>>(x, y_poly, y_ref, n);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(uint32_t* err, int timeout_ms, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(err, (uint64_t)timeout_ms * 1000000ull);
  return cudaGetLastError();
}

}  // namespace isa
