// selftest.cu -- device-side checks exposed for the test suite (not part of an attention call).
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"
#include "vsa.h"

namespace vsa {

__global__ void exp2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y_poly,
                                     float* __restrict__ y_mufu, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    // the packed form the attention kernel runs, on the pair (x[i], x[i ^ 1]); it must agree
    // with the scalar form bit for bit, else the result is NaN
    const float other = (i ^ 1) < n ? x[i ^ 1] : 0.0f;
    float lo, hi;
    f2_split(exp2_poly2((i & 1) ? f2_make(other, x[i]) : f2_make(x[i], other)), lo, hi);
    const float packed = (i & 1) ? hi : lo;
    const float scalar = exp2_poly(x[i]);
    y_poly[i] = __float_as_uint(packed) == __float_as_uint(scalar) ? scalar : __int_as_float(0x7fc00000);
    y_mufu[i] = fast_exp2(x[i]);
  }
}

// One thread waits, with the bounded wait every kernel uses, on an mbarrier that expects one
// arrival which never comes: after the wait limit it must give up, raise the timeout bit of
// the error word and return.
__global__ void wait_timeout_selftest_kernel(int* __restrict__ err, int* __restrict__ waited) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    mbar_init_fence();
    abort_flag = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) *waited = mbar_wait(smem_u32(&bar), 0, &abort_flag, err) ? 1 : 0;
}

}  // namespace vsa

extern "C" vsa_status vsa_selftest_wait_timeout(int* d_err, int* d_waited, cudaStream_t stream) {
  if (d_err == nullptr || d_waited == nullptr) return VSA_ERR_INVALID_ARG;
  vsa::wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(d_err, d_waited);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

extern "C" vsa_status vsa_selftest_exp2(const float* x, float* y_poly, float* y_mufu, int n, cudaStream_t stream) {
  if (x == nullptr || y_poly == nullptr || y_mufu == nullptr || n < 0) return VSA_ERR_INVALID_ARG;
  if (n == 0) return VSA_OK;
  vsa::exp2_selftest_kernel<<<(n + 255) / 256, 256, 0, stream>>>(x, y_poly, y_mufu, n);
  return cudaGetLastError() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}

// Test hook: reset the current device's primary context through this library's own CUDA
// runtime, so that a test can check that later calls still find their device state.
extern "C" vsa_status vsa_selftest_device_reset(void) {
  return cudaDeviceReset() == cudaSuccess ? VSA_OK : VSA_ERR_CUDA;
}
