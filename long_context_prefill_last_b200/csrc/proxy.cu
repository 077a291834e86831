// Proxy map reduction (CRISP summary page, Algorithm 2 and Algorithm 3's
// directional scores) and its finalisation into block masses.
//
// The proxy map A-hat[i, j] = softmax_j(sm_scale * q_i . k_j), j <= i, for the
// last 64 queries i is never materialised. For every (proxy row, key tile)
// the kernels keep two partial sums of exp(score - m): keys whose offset
// i - j falls in offset block I - t (columns c <= r of the tile, r = i mod B)
// and keys whose offset falls in block I - t - 1 (c > r). Together they are
// the tile's column mass; separately they are its two diagonal-block masses.
// m is a per-(row, chunk of 8 tiles) running maximum, so finalisation only
// needs one (m, l) pair per chunk.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace crisp {
namespace {

struct ProxyArgs {
  int n, nb, group, n_chunks;
  float scale_log2;
  float* part_lo;
  float* part_hi;
  float2* chunk_ml;
  int32_t* status;
};

constexpr int kPartStride = 32 * 36 + 4;   // floats per 32-dim slice of a staged key sub-tile

// One CTA per (chunk of 8 key tiles, query head); thread (r = proxy row,
// part = 32-dim slice of d). CUDA-core FFMA, any input type.
template <typename T>
__global__ void __launch_bounds__(256) proxy_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                         ProxyArgs a) {
  __shared__ __align__(16) float ks[4 * kPartStride];
  const int h = blockIdx.y, chunk = blockIdx.x;
  const int g = h / a.group;
  const int tid = threadIdx.x, r = tid >> 2, part = tid & 3;
  const int I = a.nb - 1;                 // every proxy row lies in the last query block
  const int rr = (a.n - kProxyRows + r) - I * kBlock;   // row position inside its block

  float qr[32];
  {
    const T* qp = q + ((size_t)h * a.n + (a.n - kProxyRows + r)) * kHeadDim + part * 32;
#pragma unroll
    for (int j = 0; j < 32; ++j) qr[j] = dev::to_f32(qp[j]) * a.scale_log2;
  }
  float m_run = -INFINITY, l_run = 0.f;
  float lo[kChunkTiles], hi[kChunkTiles];
#pragma unroll
  for (int u = 0; u < kChunkTiles; ++u) lo[u] = hi[u] = 0.f;

  const T* kg = k + (size_t)g * a.n * kHeadDim;
#pragma unroll
  for (int u = 0; u < kChunkTiles; ++u) {
    const int t = chunk * kChunkTiles + u;
    if (t >= a.nb) break;
    float sc[32];   // this lane's 8 scores of each 32-key sub-tile
#pragma unroll
    for (int sub = 0; sub < 4; ++sub) {
      __syncthreads();
      // stage keys [128t + 32sub, +32) as fp32: ks[part][key][dd]; every
      // load issued before the first store (16 per thread)
#pragma unroll
      for (int e = tid; e < 32 * kHeadDim; e += 256) {
        const int key = e >> 7, dcol = e & 127;
        ks[(dcol >> 5) * kPartStride + key * 36 + (dcol & 31)] =
            dev::to_f32(kg[(size_t)(t * kBlock + sub * 32 + key) * kHeadDim + dcol]);
      }
      __syncthreads();
      float acc[32];
      const float* kp = ks + part * kPartStride;
#pragma unroll
      for (int key = 0; key < 32; ++key) {
        float s = 0.f;
#pragma unroll
        for (int dd = 0; dd < 32; dd += 4) {
          const float4 kv4 = *reinterpret_cast<const float4*>(kp + key * 36 + dd);
          s = fmaf(qr[dd], kv4.x, s);
          s = fmaf(qr[dd + 1], kv4.y, s);
          s = fmaf(qr[dd + 2], kv4.z, s);
          s = fmaf(qr[dd + 3], kv4.w, s);
        }
        acc[key] = s;
      }
      // reduce-scatter over the 4 lanes of the row: lane keeps 8 keys
      const bool b0 = part & 1, b1 = (part >> 1) & 1;
      float h16[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float send = b0 ? acc[j] : acc[j + 16];
        const float keep = b0 ? acc[j + 16] : acc[j];
        h16[j] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float send = b1 ? h16[j] : h16[j + 8];
        const float keep = b1 ? h16[j + 8] : h16[j];
        sc[sub * 8 + j] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
      }
    }
    // this lane's key columns: sub*32 + base + j
    const int base = (part & 1) * 16 + ((part >> 1) & 1) * 8;
    float tmax = -INFINITY;
#pragma unroll
    for (int sub = 0; sub < 4; ++sub)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = sub * 32 + base + j;
        if (t == I && c > rr) sc[sub * 8 + j] = -INFINITY;   // causal: keys after the query
        tmax = fmaxf(tmax, sc[sub * 8 + j]);
      }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    if (tmax > m_run + 8.f) {   // lazy rescale (same decision on the 4 lanes)
      const float f = dev::ex2(m_run - tmax);
      l_run *= f;
#pragma unroll
      for (int w = 0; w < kChunkTiles; ++w) {
        lo[w] *= f;
        hi[w] *= f;
      }
      m_run = tmax;
    }
    float slo = 0.f, shi = 0.f;
#pragma unroll
    for (int sub = 0; sub < 4; ++sub)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = sub * 32 + base + j;
        const float p = dev::ex2(sc[sub * 8 + j] - m_run);
        if (c <= rr) slo += p; else shi += p;
      }
    slo += __shfl_xor_sync(0xffffffffu, slo, 1);
    slo += __shfl_xor_sync(0xffffffffu, slo, 2);
    shi += __shfl_xor_sync(0xffffffffu, shi, 1);
    shi += __shfl_xor_sync(0xffffffffu, shi, 2);
    lo[u] = slo;
    hi[u] = shi;
    l_run += slo + shi;
  }
  // write this chunk: lane `part` writes tiles 2*part, 2*part+1
  const size_t row = (size_t)h * kProxyRows + r;
#pragma unroll
  for (int u = 0; u < kChunkTiles; ++u) {
    const int t = chunk * kChunkTiles + u;
    if ((u >> 1) == part && t < a.nb) {
      a.part_lo[row * a.nb + t] = lo[u];
      a.part_hi[row * a.nb + t] = hi[u];
    }
  }
  if (part == 0) a.chunk_ml[row * a.n_chunks + chunk] = make_float2(m_run, l_run);
}

// Row normalisers: M_i = max over chunks, L_i = sum l * 2^(m - M); chunk
// weight 2^(m - M) / (L_i * |Q-hat|) turns stored partials into column means.
// One warp per proxy row, lanes over chunks.
__global__ void __launch_bounds__(256) proxy_row_weights_kernel(const float2* __restrict__ ml, float* __restrict__ w,
                                                                int rows, int n_chunks, int32_t* status) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float2* p = ml + (size_t)row * n_chunks;
  float M = -INFINITY;
  for (int c = lane; c < n_chunks; c += 32) M = fmaxf(M, p[c].x);
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float L = 0.f;
  for (int c = lane; c < n_chunks; c += 32) L += p[c].y * dev::ex2(p[c].x - M);
  for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
  if (lane == 0 && (!(L > 0.f) || !isfinite(L) || !isfinite(M)))
    dev::report(status, CRISP_ERR_NONFINITE, row / kProxyRows);
  const float inv = 1.f / (L * (float)kProxyRows);
  for (int c = lane; c < n_chunks; c += 32) w[(size_t)row * n_chunks + c] = dev::ex2(p[c].x - M) * inv;
}

// Column-block masses p_v[t] and the two diagonal halves of every tile.
__global__ void proxy_tile_sums_kernel(const float* __restrict__ lo, const float* __restrict__ hi,
                                       const float* __restrict__ w, float* __restrict__ p_v,
                                       float* __restrict__ ta, float* __restrict__ tb, int nb, int n_chunks) {
  const int h = blockIdx.y;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= nb) return;
  float A = 0.f, Bs = 0.f;
  for (int r = 0; r < kProxyRows; ++r) {
    const size_t row = (size_t)h * kProxyRows + r;
    const float wt = w[row * n_chunks + t / kChunkTiles];
    A = fmaf(lo[row * nb + t], wt, A);
    Bs = fmaf(hi[row * nb + t], wt, Bs);
  }
  p_v[(size_t)h * nb + t] = A + Bs;
  ta[(size_t)h * nb + t] = A;
  tb[(size_t)h * nb + t] = Bs;
}

}  // namespace

cudaError_t launch_proxy_simt(const void* q, const void* k, const Shape& s, char* ws, const WsLayout& L,
                              cudaStream_t st) {
  ProxyArgs a;
  a.n = s.n;
  a.nb = s.nb;
  a.group = s.group;
  a.n_chunks = s.n_chunks;
  a.scale_log2 = s.scale_log2;
  a.part_lo = reinterpret_cast<float*>(ws + L.part_lo);
  a.part_hi = reinterpret_cast<float*>(ws + L.part_hi);
  a.chunk_ml = reinterpret_cast<float2*>(ws + L.chunk_ml);
  a.status = reinterpret_cast<int32_t*>(ws + L.status);
  dim3 grid(s.n_chunks, s.h_q);
  if (s.fp32)
    proxy_simt_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(q), static_cast<const float*>(k), a);
  else
    proxy_simt_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                                           static_cast<const __nv_bfloat16*>(k), a);
  return cudaGetLastError();
}

cudaError_t launch_finalize(const Shape& s, char* ws, const WsLayout& L, const IndexPtrs& ix, cudaStream_t st) {
  const float2* ml = reinterpret_cast<const float2*>(ws + L.chunk_ml);
  float* w = reinterpret_cast<float*>(ws + L.chunk_w);
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  const int rows = s.h_q * kProxyRows;
  proxy_row_weights_kernel<<<(rows + 7) / 8, 256, 0, st>>>(ml, w, rows, s.n_chunks, status);
  dim3 grid((s.nb + 127) / 128, s.h_q);
  proxy_tile_sums_kernel<<<grid, 128, 0, st>>>(reinterpret_cast<const float*>(ws + L.part_lo),
                                               reinterpret_cast<const float*>(ws + L.part_hi), w, ix.p_v,
                                               reinterpret_cast<float*>(ws + L.tile_a),
                                               reinterpret_cast<float*>(ws + L.tile_b), s.nb, s.n_chunks);
  return cudaGetLastError();
}

}  // namespace crisp
