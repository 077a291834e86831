// crisp_route_noalloc: the route stage (proxy map, finalisation, route and VS
// masses) with its scratch in a static device array instead of a caller
// workspace, for callers that cannot give the library device memory.
//
// The array is a file-scope __device__ variable; host code must not pass its
// name to a kernel (on the host the name is only a stand-in for the device
// symbol). Its device address is looked up here with cudaGetSymbolAddress,
// with the device current, and that pointer is what the kernels receive.
#include <cuda_runtime.h>

#include <math.h>

#include <mutex>

#include "crisp.h"
#include "internal.h"

namespace crisp {
namespace {

constexpr size_t kScratchBytes = CRISP_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_lock[kMaxDevices];
void* g_scratch[kMaxDevices];   // set once a lookup on that device succeeded

// Device address of the array on the current device. Only a successful
// lookup is kept: a failed one (for example inside a stream capture) clears
// the runtime's error and is tried again on the next call.
cudaError_t scratch_for_device(char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> guard(g_lock[dev]);
  if (g_scratch[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) {
      (void)cudaGetLastError();
      return e;
    }
    g_scratch[dev] = p;
  }
  *out = static_cast<char*>(g_scratch[dev]);
  return cudaSuccess;
}

// Copy the routes and C_struct out of the array; if any kernel of this call
// recorded a device-side failure in the array's status word, publish
// route = -1 and C_struct = NaN for every head instead.
__global__ void publish_route_kernel(const int32_t* __restrict__ status, const int32_t* __restrict__ route_in,
                                     const float* __restrict__ c_in, int32_t* __restrict__ route_out,
                                     float* __restrict__ c_out, int h_q) {
  const bool failed = status[0] != 0;
  for (int h = blockIdx.x * blockDim.x + threadIdx.x; h < h_q; h += gridDim.x * blockDim.x) {
    route_out[h] = failed ? -1 : route_in[h];
    c_out[h] = failed ? nanf("") : c_in[h];
  }
}

// Only the regions the route stage touches, packed from offset 0.
WsLayout route_layout(const Shape& s) {
  WsLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = (off + bytes + 255) & ~(size_t)255;
    return o;
  };
  const size_t hq = s.h_q, nb = s.nb, rows = (size_t)s.h_q * s.last_q;
  L.status = take(256);
  L.part_lo = take(rows * nb * 4);
  L.part_hi = take(rows * nb * 4);
  L.chunk_ml = take(rows * s.n_chunks * 8);
  L.chunk_w = take(rows * s.n_chunks * 4);
  L.tile_a = take(hq * nb * 4);
  L.tile_b = take(hq * nb * 4);
  L.kv_pe = take((size_t)s.h_kv * 4);
  L.route = take(hq * 4);
  L.c_struct = take(hq * 4);
  L.p_v = take(hq * nb * 4);
  L.p_s = take(hq * nb * 4);
  L.mu = take(hq * 2 * 4);
  L.vs_mask = take(hq * 2 * (size_t)s.words * 4);
  L.v_idx = take(hq * nb * 4);
  L.s_idx = take(hq * nb * 4);
  L.nv = take(hq * 4);
  L.ns = take(hq * 4);
  L.pe_count = take(hq * 8);
  L.pe_cut = take(hq * 4);
  L.total = off;
  return L;
}

}  // namespace
}  // namespace crisp

using namespace crisp;

extern "C" crisp_status crisp_route_noalloc(const void* q, const void* k, const crisp_cfg* cfg, int32_t* route,
                                            float* c_struct, void* stream) {
  Shape s;
  crisp_status r = shape_from_cfg(cfg, &s);
  if (r != CRISP_OK) return r;
  if (q == nullptr || k == nullptr || route == nullptr || c_struct == nullptr) return CRISP_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(q) % 16 != 0 || reinterpret_cast<uintptr_t>(k) % 16 != 0) return CRISP_ERR_ALIGN;
  const WsLayout L = route_layout(s);
  if (L.total > kScratchBytes) return CRISP_ERR_TOO_LARGE;
  char* ws = nullptr;
  if (scratch_for_device(&ws) != cudaSuccess) return CRISP_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  IndexPtrs ix{};
  ix.route = reinterpret_cast<int32_t*>(ws + L.route);
  ix.c_struct = reinterpret_cast<float*>(ws + L.c_struct);
  ix.p_v = reinterpret_cast<float*>(ws + L.p_v);
  ix.p_s = reinterpret_cast<float*>(ws + L.p_s);
  ix.mu = reinterpret_cast<float*>(ws + L.mu);
  ix.vs_mask = reinterpret_cast<uint32_t*>(ws + L.vs_mask);
  ix.v_idx = reinterpret_cast<int32_t*>(ws + L.v_idx);
  ix.s_idx = reinterpret_cast<int32_t*>(ws + L.s_idx);
  ix.nv = reinterpret_cast<int32_t*>(ws + L.nv);
  ix.ns = reinterpret_cast<int32_t*>(ws + L.ns);
  ix.pe_mask = nullptr;
  ix.pe_count = reinterpret_cast<int64_t*>(ws + L.pe_count);
  ix.pe_cut = reinterpret_cast<float*>(ws + L.pe_cut);
  // what must start at zero: the status word and the per-group PE flags
  if (cudaMemsetAsync(ws + L.status, 0, 32, st) != cudaSuccess) return CRISP_ERR_CUDA;
  if (cudaMemsetAsync(ws + L.kv_pe, 0, (size_t)s.h_kv * 4, st) != cudaSuccess) return CRISP_ERR_CUDA;
  cudaError_t e = !s.fp32 ? launch_proxy_tc(q, k, s, ws, L, st) : launch_proxy_simt(q, k, s, ws, L, st);
  if (e == cudaSuccess) e = launch_finalize(s, ws, L, ix, st);
  if (e == cudaSuccess) e = launch_vs_select(s, ws, L, ix, st);
  if (e == cudaSuccess) {
    publish_route_kernel<<<(s.h_q + 255) / 256, 256, 0, st>>>(reinterpret_cast<const int32_t*>(ws + L.status),
                                                              ix.route, ix.c_struct, route, c_struct, s.h_q);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return CRISP_ERR_CUDA;
  }
  return CRISP_OK;
}
