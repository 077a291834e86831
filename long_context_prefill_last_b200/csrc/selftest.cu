// Device self-tests: the FMA-pipe exp2 approximations (dev::exp2_poly3/5)
// against CUDA's exp2f, so their error bounds are checked on the hardware
// that runs them; and the bounded mbarrier wait every kernel uses, made to
// run out on a barrier nothing arrives on.
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
// One thread waits on phase 0 of an mbarrier that expects one arrival and
// never gets it. dev::mbar_wait gives up after `limit` cycles, raises the
// abort flag and writes CRISP_ERR_TIMEOUT (info = 99) to the status word.
__global__ void wait_selftest_kernel(long long limit, int32_t* status) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  const uint32_t b = dev::smem_u32(&bar);
  dev::mbar_init(b, 1);
  dev::fence_mbar_init();
  volatile int* af = &abort_flag;
  const bool ok = dev::mbar_wait(b, 0, af, status, 99, limit);
  if (ok) dev::report(status, CRISP_ERR_INVALID_ARG, 98);   // cannot happen: nothing arrived
}
}  // namespace
}  // namespace crisp

extern "C" crisp_status crisp_wait_selftest(int64_t limit_cycles, int32_t* status, void* stream) {
  if (status == nullptr || limit_cycles < 1000 || limit_cycles > 4000000000LL) return CRISP_ERR_INVALID_ARG;
  crisp::wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles, status);
  return cudaGetLastError() == cudaSuccess ? CRISP_OK : CRISP_ERR_CUDA;
}

extern "C" crisp_status crisp_exp2_selftest(const float* x, float* poly3, float* poly5, float* ref, int32_t n,
                                            void* stream) {
  if (x == nullptr || poly3 == nullptr || poly5 == nullptr || ref == nullptr || n < 0) return CRISP_ERR_INVALID_ARG;
  if (n == 0) return CRISP_OK;
  crisp::exp2_selftest_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, poly3, poly5, ref,
                                                                                              n);
  return cudaGetLastError() == cudaSuccess ? CRISP_OK : CRISP_ERR_CUDA;
}
