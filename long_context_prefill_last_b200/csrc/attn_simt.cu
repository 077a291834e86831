// Block-sparse causal attention on CUDA cores (FFMA, fp32 accumulation).
// Used for fp32 layers, where tensor-core formats cannot meet a 1e-4
// tolerance, and as an independent cross-check of the tensor-core kernel.
// CRISP summary page, Algorithm 1: exact softmax attention over the selected
// keys; the per-tile selection rule is dev::tile_kind.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace crisp {
namespace {

struct AttnArgs {
  int n, nb, words, group, h_q;
  float scale_log2;
  bool dense;
  const int32_t* route;
  const uint32_t* vs_mask;
  const uint32_t* pe_mask;
  int32_t* status;
};

constexpr int kSub = 32;                     // keys staged per step
constexpr int kStride = kSub * 36 + 4;       // floats per 32-dim slice of a staged sub-tile

// One CTA per (64-query half tile, head), heaviest query tiles first.
// Thread (r, part): query row r of the half tile, output dims [32 part, 32 part + 32).
template <typename T>
__global__ void __launch_bounds__(256) attn_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                        const T* __restrict__ v, T* __restrict__ out, AttnArgs a) {
  __shared__ __align__(16) float ks[4 * kStride];
  __shared__ __align__(16) float vs[4 * kStride];
  const int lin = blockIdx.x;
  const int h = lin % a.h_q;
  const int half_tile = (2 * a.nb - 1) - lin / a.h_q;
  const int I = half_tile >> 1, half = half_tile & 1;
  const int g = h / a.group;
  const int tid = threadIdx.x, r = tid >> 2, part = tid & 3;
  const int rr = half * 64 + r;                 // row inside the 128-query tile
  const int i = I * kBlock + rr;
  const int route = a.dense ? 0 : a.route[h];
  const uint32_t* vmask = a.vs_mask + (size_t)h * 2 * a.words;
  const uint32_t* smask = vmask + a.words;
  const uint32_t* pe_row = a.pe_mask + ((size_t)h * a.nb + I) * a.words;

  float qr[32], o[32];
  const T* qp = q + ((size_t)h * a.n + i) * kHeadDim + part * 32;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    qr[j] = dev::to_f32(qp[j]) * a.scale_log2;
    o[j] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const T* kg = k + (size_t)g * a.n * kHeadDim;
  const T* vg = v + (size_t)g * a.n * kHeadDim;

  for (int t = 0; t <= I; ++t) {
    const int kind = dev::tile_kind(route, vmask, smask, pe_row, a.dense, I, t);
    if (kind == dev::kSkip) continue;
    for (int sub = 0; sub < kBlock / kSub; ++sub) {
      __syncthreads();
      // every load of the sub-tile is issued before the first store (16 per thread)
#pragma unroll
      for (int e = tid; e < kSub * kHeadDim; e += 256) {
        const int key = e >> 7, dcol = e & 127;
        const size_t src = (size_t)(t * kBlock + sub * kSub + key) * kHeadDim + dcol;
        const int dst = (dcol >> 5) * kStride + key * 36 + (dcol & 31);
        ks[dst] = dev::to_f32(kg[src]);
        vs[dst] = dev::to_f32(vg[src]);
      }
      __syncthreads();
      float s[kSub];
      const float* kp = ks + part * kStride;
#pragma unroll
      for (int key = 0; key < kSub; ++key) {
        float acc = 0.f;
#pragma unroll
        for (int dd = 0; dd < 32; dd += 4) {
          const float4 k4 = *reinterpret_cast<const float4*>(kp + key * 36 + dd);
          acc = fmaf(qr[dd], k4.x, acc);
          acc = fmaf(qr[dd + 1], k4.y, acc);
          acc = fmaf(qr[dd + 2], k4.z, acc);
          acc = fmaf(qr[dd + 3], k4.w, acc);
        }
        acc += __shfl_xor_sync(0xffffffffu, acc, 1);
        acc += __shfl_xor_sync(0xffffffffu, acc, 2);
        const int c = sub * kSub + key;
        const bool keep = kind == dev::kFull || (kind == dev::kLower && c <= rr) || (kind == dev::kUpper && c > rr);
        s[key] = keep ? acc : -INFINITY;
      }
      float smax = -INFINITY;
#pragma unroll
      for (int key = 0; key < kSub; ++key) smax = fmaxf(smax, s[key]);
      const float m_new = fmaxf(m, smax);
      if (m_new == -INFINITY) continue;      // nothing visible yet for this row
      const float corr = dev::ex2(m - m_new);
      l *= corr;
#pragma unroll
      for (int j = 0; j < 32; ++j) o[j] *= corr;
      m = m_new;
      const float* vp = vs + part * kStride;
#pragma unroll
      for (int key = 0; key < kSub; ++key) {
        const float p = dev::ex2(s[key] - m);
        l += p;
#pragma unroll
        for (int dd = 0; dd < 32; dd += 4) {
          const float4 v4 = *reinterpret_cast<const float4*>(vp + key * 36 + dd);
          o[dd] = fmaf(p, v4.x, o[dd]);
          o[dd + 1] = fmaf(p, v4.y, o[dd + 1]);
          o[dd + 2] = fmaf(p, v4.z, o[dd + 2]);
          o[dd + 3] = fmaf(p, v4.w, o[dd + 3]);
        }
      }
    }
  }
  const float inv = 1.f / l;
  T* op = out + ((size_t)h * a.n + i) * kHeadDim + part * 32;
#pragma unroll
  for (int j = 0; j < 32; ++j) op[j] = dev::from_f32<T>(o[j] * inv);
}

}  // namespace

cudaError_t launch_attn_simt(const void* q, const void* k, const void* v, void* out, const Shape& s,
                             const int32_t* route, const uint32_t* vs_mask, const uint32_t* pe_mask, bool dense,
                             int32_t* status, cudaStream_t st) {
  AttnArgs a;
  a.n = s.n;
  a.nb = s.nb;
  a.words = s.words;
  a.group = s.group;
  a.h_q = s.h_q;
  a.scale_log2 = s.scale_log2;
  a.dense = dense;
  a.route = route;
  a.vs_mask = vs_mask;
  a.pe_mask = pe_mask;
  a.status = status;
  const int grid = 2 * s.nb * s.h_q;
  if (s.fp32)
    attn_simt_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                                  static_cast<const float*>(v), static_cast<float*>(out), a);
  else
    attn_simt_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(out), a);
  return cudaGetLastError();
}

}  // namespace crisp
