// Device self-test of the FMA-pipe exp2 approximations (dev::exp2_poly3/5)
// against CUDA's exp2f, so their error bounds are checked on the hardware
// that runs them.
#include "crisp.h"
#include "internal.h"
#include "ptx.cuh"

namespace crisp {
namespace {
__global__ void exp2_selftest_kernel(const float* __restrict__ x, float* p3, float* p5, float* ref, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float v = x[i];
  p3[i] = dev::exp2_poly3(v);
  p5[i] = dev::exp2_poly5(v);
  ref[i] = exp2f(v);
}
}  // namespace
}  // namespace crisp

extern "C" crisp_status crisp_exp2_selftest(const float* x, float* poly3, float* poly5, float* ref, int32_t n,
                                            void* stream) {
  if (x == nullptr || poly3 == nullptr || poly5 == nullptr || ref == nullptr || n < 0) return CRISP_ERR_INVALID_ARG;
  if (n == 0) return CRISP_OK;
  crisp::exp2_selftest_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, poly3, poly5, ref,
                                                                                              n);
  return cudaGetLastError() == cudaSuccess ? CRISP_OK : CRISP_ERR_CUDA;
}
