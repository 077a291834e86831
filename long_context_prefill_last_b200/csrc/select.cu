// Route (CRISP summary page, Eq. (2) and the rule under it) and sink-aware
// VS selection (Eq. (3), Eq. (4), Algorithm 3) for every query head.
#include "internal.h"
#include "ptx.cuh"

namespace crisp {
namespace {

struct SelectArgs {
  int nb, words, group, force_route;
  float tau, alpha;
  const float* ta;
  const float* tb;
  int32_t* kv_pe;
  IndexPtrs ix;
};

// Block-wide exclusive scan of per-thread flags (0/1); returns the exclusive
// prefix of this thread and writes the block total to *total.
__device__ int block_excl_scan(int flag, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) warp_sums[wid] = __popc(bal);
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int w = 0; w < nw; ++w) {
      const int v = warp_sums[w];
      warp_sums[w] = acc;
      acc += v;
    }
    warp_sums[nw] = acc;
  }
  __syncthreads();
  const int res = warp_sums[wid] + in_warp;
  *total = warp_sums[nw];
  __syncthreads();
  return res;
}

// One CTA (1024 threads) per query head.
__global__ void __launch_bounds__(1024) vs_select_kernel(SelectArgs a) {
  __shared__ int warp_sums[33];
  __shared__ double s_mu[2];
  __shared__ int s_route;
  const int h = blockIdx.x;
  const int nb = a.nb, I = nb - 1;
  float* p_v = a.ix.p_v + (size_t)h * nb;
  float* p_s = a.ix.p_s + (size_t)h * nb;
  const float* ta = a.ta + (size_t)h * nb;
  const float* tb = a.tb + (size_t)h * nb;
  // diagonal-block masses: p_s[b] = (c <= r part of tile I-b) + (c > r part of tile I-b-1)
  for (int b = threadIdx.x; b < nb; b += blockDim.x) p_s[b] = ta[I - b] + (b < I ? tb[I - b - 1] : 0.f);
  __syncthreads();
  if (threadIdx.x == 0) {
    // Eq. (2): S_anchor = sinks (column block 0 since w_sink = B) union the
    // recency window (offset block 0 since w_local = B); disjoint for n >= 512.
    const float c = p_v[0] + p_s[0];
    int route = (c >= a.tau) ? 0 : 1;
    if (a.force_route == 0 || a.force_route == 1) route = a.force_route;
    a.ix.c_struct[h] = c;
    a.ix.route[h] = route;
    if (route == 1) atomicOr(&a.kv_pe[h / a.group], 1);
    s_route = route;
    // Eq. (3): noise floor over the non-retained blocks, per direction
    const double mv = fmax(1.0 - (double)p_v[0] - (double)p_v[nb - 1], 0.0) / (double)(nb - 2);
    const double ms = fmax(1.0 - (double)p_s[0] - (double)p_s[nb - 1], 0.0) / (double)(nb - 2);
    s_mu[0] = mv;
    s_mu[1] = ms;
    a.ix.mu[2 * h] = (float)mv;
    a.ix.mu[2 * h + 1] = (float)ms;
    a.ix.pe_count[h] = 0;
    a.ix.pe_cut[h] = 0.f;
  }
  __syncthreads();
  // Eq. (4): keep block j iff p_j > alpha * mu; first and last always kept.
  for (int dir = 0; dir < 2; ++dir) {
    const float* p = dir == 0 ? p_v : p_s;
    const double thr = (double)a.alpha * s_mu[dir];
    uint32_t* mask = a.ix.vs_mask + ((size_t)h * 2 + dir) * a.words;
    int32_t* idx = (dir == 0 ? a.ix.v_idx : a.ix.s_idx) + (size_t)h * nb;
    int base = 0;
    for (int b0 = 0; b0 < a.words * 32; b0 += blockDim.x) {
      const int b = b0 + threadIdx.x;
      int sel = 0;
      if (b < nb) sel = ((double)p[b] > thr) || b == 0 || b == nb - 1;
      const unsigned bal = __ballot_sync(0xffffffffu, sel);
      if ((threadIdx.x & 31) == 0 && (b >> 5) < a.words) mask[b >> 5] = bal;
      int tot;
      const int pos = block_excl_scan(sel, warp_sums, &tot);
      if (sel) idx[base + pos] = b;
      base += tot;
    }
    if (threadIdx.x == 0) (dir == 0 ? a.ix.nv : a.ix.ns)[h] = base;
  }
}

}  // namespace

cudaError_t launch_vs_select(const Shape& s, char* ws, const WsLayout& L, const IndexPtrs& ix, cudaStream_t st) {
  SelectArgs a;
  a.nb = s.nb;
  a.words = s.words;
  a.group = s.group;
  a.force_route = s.force_route;
  a.tau = s.tau;
  a.alpha = s.alpha;
  a.ta = reinterpret_cast<const float*>(ws + L.tile_a);
  a.tb = reinterpret_cast<const float*>(ws + L.tile_b);
  a.kv_pe = reinterpret_cast<int32_t*>(ws + L.kv_pe);
  a.ix = ix;
  vs_select_kernel<<<s.h_q, 1024, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace crisp
