// Pooled estimation (CRISP summary page, Algorithm 4, "GlobalAdaptive"):
// block-mean pooling of Q and K, A-bar = softmax(Q-bar K-bar^T * sm_scale)
// over c <= r, normalisation of the flattened causal map by its total (N_b,
// one per row), and the gamma-cumulative cut: keep the largest entries
// (ties by ascending flat index r*N_b + c) until their mass reaches gamma.
// The diagonal block is always kept.
//
// The cut is found without sorting: a three-level radix select over the
// fp32 bit patterns of the (positive) entries, with per-bucket counts and
// float64 mass. Only heads routed PE do any work; the rest exit at once.
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace crisp {
namespace {

struct PeArgs {
  int n, nb, words, group, h_q, h_kv;
  long long tri, tri_stride;
  float scale_log2;
  float gamma;
  const int32_t* route;
  const int32_t* kv_pe;
  float* qbar;
  float* kbar;
  float* tri_buf;
  float4* tri_stats;   // [h_q][nb][n_ct] per-tile row (max, sum of 2^(l - max), min, 0)
  int n_ct;            // 64-column tiles per row
  PeHist* hist;
  PeState* state;
  uint32_t* tie_rows;
  uint32_t* pe_mask;
  int64_t* pe_count;
  float* pe_cut;
  int32_t* status;
};

__device__ __forceinline__ long long tri_off(int r) { return (long long)r * (r + 1) / 2; }

__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 16 bytes of T widened to fp32.
template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&o)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void load(const float* p, float (&o)[4]) {
    const float4 u = *reinterpret_cast<const float4*>(p);
    o[0] = u.x;
    o[1] = u.y;
    o[2] = u.z;
    o[3] = u.w;
  }
};

// Block mean of 128 rows of x[head] -> out[head][b][:] (fp32). One CTA per
// (block, head); 16-byte loads, 128 / N threads per row, N rows at a time.
template <typename T>
__global__ void __launch_bounds__(128) pool_kernel(const T* __restrict__ x, float* __restrict__ out, int n, int nb,
                                                   const int32_t* __restrict__ flag) {
  const int b = blockIdx.x, head = blockIdx.y;
  if (flag[head] == 0) return;   // route (query heads) or PE-group flag (KV heads)
  constexpr int N = Vec16<T>::N;
  constexpr int TPR = kHeadDim / N;   // threads per row
  constexpr int RP = 128 / TPR;       // rows in parallel
  __shared__ float red[RP][kHeadDim];
  const int tid = threadIdx.x, rg = tid / TPR, c0 = (tid % TPR) * N;
  float acc[N];
#pragma unroll
  for (int j = 0; j < N; ++j) acc[j] = 0.f;
  const T* base = x + ((size_t)head * n + (size_t)b * kBlock) * kHeadDim + c0;
#pragma unroll 4
  for (int row = rg; row < kBlock; row += RP) {
    float v[N];
    Vec16<T>::load(base + (size_t)row * kHeadDim, v);
#pragma unroll
    for (int j = 0; j < N; ++j) acc[j] += v[j];
  }
#pragma unroll
  for (int j = 0; j < N; ++j) red[rg][c0 + j] = acc[j];
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int g = 0; g < RP; ++g) s += red[g][tid];
  out[((size_t)head * nb + b) * kHeadDim + tid] = s * (1.f / kBlock);
}

// Pooled logits (log2 domain) of one 128 x 128 tile (rt, ct), ct <= rt, of
// the block-causal triangle. Thread (ty, tx) holds an 8 x 8 register tile:
// rows ty*4 + {0..3} and 64 + ty*4 + {0..3}, columns tx*4 + {0..3} and
// 64 + tx*4 + {0..3}. Both operand tiles sit transposed in shared memory
// ([d][block], row stride 132 floats), so each step over d reads four float4
// (contiguous across the threads of a row) for 64 FMAs. The statistics the
// row softmax needs are kept per 64-column half (kLT).
constexpr int kLT = 64;        // columns per statistics tile
constexpr int kLT2 = 128;      // blocks per CTA tile side
constexpr int kLStride = 132;  // floats per transposed row
// One tile ti of query head h (routed PE).
__device__ __forceinline__ void pe_logits_tile(const PeArgs& a, int h, int ti, float* lsm) {
  const int g = h / a.group;
  // linear lower-triangle tile index -> (rt, ct)
  int rt = (int)((sqrtf(8.f * (float)ti + 1.f) - 1.f) * 0.5f);
  while ((rt + 1) * (rt + 2) / 2 <= ti) ++rt;
  while (rt * (rt + 1) / 2 > ti) --rt;
  const int ct = ti - rt * (rt + 1) / 2;
  const int r0 = rt * kLT2, c0 = ct * kLT2;
  float* qT = lsm;                        // [128][kLStride]
  float* kT = lsm + kHeadDim * kLStride;  // [128][kLStride]
  const int tid = threadIdx.x;
  for (int e = tid; e < kLT2 * kHeadDim; e += 256) {
    const int rr = e >> 7, dd = e & 127;
    qT[dd * kLStride + rr] =
        (r0 + rr < a.nb) ? a.qbar[((size_t)h * a.nb + r0 + rr) * kHeadDim + dd] * a.scale_log2 : 0.f;
    kT[dd * kLStride + rr] = (c0 + rr < a.nb) ? a.kbar[((size_t)g * a.nb + c0 + rr) * kHeadDim + dd] : 0.f;
  }
  __syncthreads();
  const int ty = tid >> 4, tx = tid & 15;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
#pragma unroll 2
  for (int dd = 0; dd < kHeadDim; ++dd) {
    const float* qd = qT + dd * kLStride;
    const float* kd = kT + dd * kLStride;
    const float4 q0 = *reinterpret_cast<const float4*>(qd + ty * 4);
    const float4 q1 = *reinterpret_cast<const float4*>(qd + 64 + ty * 4);
    const float4 k0 = *reinterpret_cast<const float4*>(kd + tx * 4);
    const float4 k1 = *reinterpret_cast<const float4*>(kd + 64 + tx * 4);
    const float qa[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    const float ka[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(qa[i], ka[j], acc[i][j]);
  }
  // per row and 64-column half: max, sum of 2^(l - max) and min over the kept
  // columns c <= r (the 16 threads of a row reduce by shuffles); then the row
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = r0 + (i >> 2) * 64 + ty * 4 + (i & 3);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float m = -INFINITY, mn = INFINITY;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int c = c0 + half * 64 + tx * 4 + jj;
        if (c <= r) {
          m = fmaxf(m, acc[i][half * 4 + jj]);
          mn = fminf(mn, acc[i][half * 4 + jj]);
        }
      }
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) {
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      }
      float sum = 0.f;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int c = c0 + half * 64 + tx * 4 + jj;
        if (c <= r) sum += dev::ex2(acc[i][half * 4 + jj] - m);
      }
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const int c64 = 2 * ct + half;   // statistics tile of this half
      if (tx == 0 && r < a.nb && c64 * kLT < a.nb && c64 * kLT <= r)
        a.tri_stats[((size_t)h * a.nb + r) * a.n_ct + c64] = make_float4(m, sum, mn, 0.f);
    }
    if (r >= a.nb) continue;
    float* row = a.tri_buf + (size_t)h * a.tri_stride + tri_off(r);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = c0 + (j >> 2) * 64 + tx * 4 + (j & 3);
      if (c <= r) row[c] = acc[i][j];
    }
  }
}

// A grid-stride loop over (query head, triangle tile) items: heads not
// routed PE cost one iteration, not a CTA launch (a launched CTA reserves
// 132 KB of shared memory, one per SM, even when it exits at once).
__global__ void __launch_bounds__(256) pe_logits_kernel(PeArgs a, int n_tri_tiles) {
  extern __shared__ __align__(16) float lsm[];
  for (long long item = blockIdx.x; item < (long long)a.h_q * n_tri_tiles; item += gridDim.x) {
    const int h = (int)(item / n_tri_tiles);
    if (a.route[h] != 1) continue;   // uniform over the CTA
    __syncthreads();                 // the previous item's reads of lsm are done
    pe_logits_tile(a, h, (int)(item % n_tri_tiles), lsm);
  }
}

__device__ __forceinline__ void hist_flush(PeHist* hist, uint32_t bucket, unsigned long long cnt, double mass) {
  if (cnt == 0) return;
  atomicAdd(&hist->count[bucket], cnt);
  atomicAdd(&hist->mass[bucket], mass);
}

constexpr int kRowsPerCta = 8;  // one warp per row
// Level-0 buckets (bits 31..20) of the values in [0, 1): every entry of the
// normalised map is at most 1 / N_b, so its bucket is below 0x3F8.
constexpr int kL0Low = 1024;

constexpr int kWin = 64;   // level-0 buckets of a row's window in the per-warp histogram

// Row softmax of the pooled logits, divided by N_b (the flattened map's
// total), written in place; level-0 histogram (bits 31..20) with float64
// mass. One warp per row; the row maximum and normaliser come from the
// logits kernel's per-tile statistics, so the row is read once. Each lane
// merges runs of equal buckets; a row whose values span fewer than kWin
// buckets gathers them in its warp's own window (lanes of one warp mostly
// hit one bucket, so windows keep contention inside a warp), a wider row
// (a heavy-tailed map) in the CTA's histogram of all level-0 buckets below
// 1.0. Non-empty buckets reach the global histogram with one atomic each.
__global__ void __launch_bounds__(256) pe_softmax_kernel(PeArgs a) {
  const int h = blockIdx.y;
  if (a.route[h] != 1) return;   // uniform over the CTA
  __shared__ unsigned long long scount[kL0Low];
  __shared__ double smass[kL0Low];
  __shared__ unsigned long long wcount[kRowsPerCta][kWin];
  __shared__ double wmass[kRowsPerCta][kWin];
  for (int i = threadIdx.x; i < kL0Low; i += blockDim.x) {
    scount[i] = 0;
    smass[i] = 0.0;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = lane; i < kWin; i += 32) {
    wcount[warp][i] = 0;
    wmass[warp][i] = 0.0;
  }
  __syncthreads();
  const int r = blockIdx.x * kRowsPerCta + warp;
  PeHist* hist = a.hist + h;
  uint32_t b_lo = 0;
  bool window = false;
  if (r < a.nb) {
    float* row = a.tri_buf + (size_t)h * a.tri_stride + tri_off(r);
    // row maximum and normaliser from the logits kernel's per-tile statistics
    const float4* st = a.tri_stats + ((size_t)h * a.nb + r) * a.n_ct;
    const int n_t = r / kLT + 1;   // column tiles holding c <= r
    float m = -INFINITY, mn = INFINITY;
    for (int i = lane; i < n_t; i += 32) {
      m = fmaxf(m, st[i].x);
      mn = fminf(mn, st[i].z);
    }
    m = warp_max(m);
    mn = warp_min(mn);
    float s = 0.f;
    for (int i = lane; i < n_t; i += 32) {
      const float4 e = st[i];
      s += e.y * dev::ex2(e.x - m);
    }
    s = warp_sum(s);
    const float inv = 1.f / (s * (float)a.nb);
    const uint32_t b_hi = __float_as_uint(inv) >> 20;                       // bucket of the row maximum
    b_lo = __float_as_uint(dev::ex2(mn - m) * inv) >> 20;                   // bucket of the row minimum
    window = b_hi >= b_lo && b_hi - b_lo < (uint32_t)kWin;
    uint32_t cur = 0xffffffffu;
    unsigned long long cnt = 0;
    double mass = 0.0;
    auto flush = [&]() {
      if (!cnt) return;
      if (window) {
        atomicAdd(&wcount[warp][cur - b_lo], cnt);
        atomicAdd(&wmass[warp][cur - b_lo], mass);
      } else if (cur < (uint32_t)kL0Low) {
        atomicAdd(&scount[cur], cnt);
        atomicAdd(&smass[cur], mass);
      } else {
        hist_flush(hist, cur, cnt, mass);
      }
    };
    for (int c = lane; c <= r; c += 32) {
      const float v = dev::ex2(row[c] - m) * inv;
      row[c] = v;
      const uint32_t bucket = __float_as_uint(v) >> 20;
      if (bucket != cur) {
        flush();
        cur = bucket;
        cnt = 0;
        mass = 0.0;
      }
      ++cnt;
      mass += (double)v;
    }
    flush();
  }
  __syncthreads();
  if (window) {   // the warp's window into the global histogram
    for (int i = lane; i < kWin; i += 32)
      if (wcount[warp][i]) hist_flush(hist, b_lo + (uint32_t)i, wcount[warp][i], wmass[warp][i]);
  }
  for (int i = threadIdx.x; i < kL0Low; i += blockDim.x)
    if (scount[i]) hist_flush(hist, (uint32_t)i, scount[i], smass[i]);
}

// Histogram of the entries whose key matches the prefix found so far
// (level 1: bits 19..8 under the 12-bit prefix; level 2: bits 7..0 under the
// 24-bit prefix). float4 sweeps over the head's triangle (stride padded to
// 64); each CTA gathers its part in shared memory (dynamic, 16 bytes per
// bucket) and adds its non-empty buckets to the global histogram.
__global__ void __launch_bounds__(256) pe_hist_kernel(PeArgs a, int level) {
  const int h = blockIdx.y;
  if (a.route[h] != 1) return;
  const PeState* st = a.state + h;
  if (st->all) return;   // uniform over the CTA
  extern __shared__ __align__(16) unsigned char hsm[];
  const int nbk = level == 1 ? kHistL1 : kHistL2;
  unsigned long long* scount = reinterpret_cast<unsigned long long*>(hsm);
  double* smass = reinterpret_cast<double*>(hsm + (size_t)nbk * sizeof(unsigned long long));
  for (int i = threadIdx.x; i < nbk; i += blockDim.x) {
    scount[i] = 0;
    smass[i] = 0.0;
  }
  __syncthreads();
  const uint32_t prefix = st->prefix;
  const int shift_p = level == 1 ? 20 : 8;
  const int shift_b = level == 1 ? 8 : 0;
  const uint32_t bmask = level == 1 ? 0xFFFu : 0xFFu;
  const float4* tri4 = reinterpret_cast<const float4*>(a.tri_buf + (size_t)h * a.tri_stride);
  const long long n4 = (a.tri + 3) / 4;
  for (long long p = (long long)blockIdx.x * blockDim.x + threadIdx.x; p < n4; p += (long long)gridDim.x * blockDim.x) {
    const float4 v4 = tri4[p];
    const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (4 * p + i >= a.tri) break;
      const uint32_t key = __float_as_uint(vv[i]);
      if ((key >> shift_p) == prefix) {
        const uint32_t b = (key >> shift_b) & bmask;
        atomicAdd(&scount[b], 1ull);
        atomicAdd(&smass[b], (double)vv[i]);
      }
    }
  }
  __syncthreads();
  PeHist* hist = a.hist + h;
  for (int i = threadIdx.x; i < nbk; i += blockDim.x)
    if (scount[i]) hist_flush(hist, (uint32_t)i, scount[i], smass[i]);
}

// Walk the buckets of the current level from the largest key down, carrying
// the mass above; pick the bucket where the cumulative mass reaches gamma.
// One CTA (1024 threads) per head. Clears the histogram for the next level.
__global__ void __launch_bounds__(1024) pe_find_kernel(PeArgs a, int level) {
  const int h = blockIdx.x;
  if (a.route[h] != 1) return;
  PeState* st = a.state + h;
  PeHist* hist = a.hist + h;
  const int nbk = level == 2 ? kHistL2 : kHistL0;
  const int per = (nbk + 1023) / 1024;
  __shared__ double tsum[1024];
  __shared__ int s_found;
  __shared__ double s_above_new;
  __shared__ int s_bucket;
  const int tid = threadIdx.x;
  if (tid == 0) {
    if (level == 0) {
      st->s_above = 0.0;
      st->prefix = 0;
      st->all = a.gamma >= 1.f ? 1u : 0u;
    }
    s_found = 0;
  }
  __syncthreads();
  const bool all = st->all != 0;
  // thread tid owns descending buckets [nbk-1 - tid*per, ... - per + 1]
  double my = 0.0;
  for (int u = 0; u < per; ++u) {
    const int b = nbk - 1 - (tid * per + u);
    if (b >= 0) my += hist->mass[b];
  }
  tsum[tid] = my;
  __syncthreads();
  // inclusive scan over threads (descending bucket order)
  for (int off = 1; off < 1024; off <<= 1) {
    const double v = tid >= off ? tsum[tid - off] : 0.0;
    __syncthreads();
    tsum[tid] += v;
    __syncthreads();
  }
  if (level == 0 && tid == 0) st->total = tsum[1023];
  __syncthreads();
  const double base = st->s_above;
  const double gamma = (double)a.gamma;
  if (!all) {
    const double before = base + (tid > 0 ? tsum[tid - 1] : 0.0);
    const double after = base + tsum[tid];
    if (before < gamma && after >= gamma) {
      double acc = before;
      int last_b = -1;
      double last_above = 0.0;
      for (int u = 0; u < per; ++u) {
        const int b = nbk - 1 - (tid * per + u);
        if (b < 0) break;
        if (hist->count[b] == 0) continue;
        last_b = b;
        last_above = acc;
        const double nxt = acc + hist->mass[b];
        if (nxt >= gamma) break;
        acc = nxt;
      }
      if (last_b >= 0) {   // the crossing bucket (or, after rounding, the lowest one of this thread)
        s_bucket = last_b;
        s_above_new = last_above;
        s_found = 1;
      }
    }
  }
  __syncthreads();
  if (!all && !s_found && level > 0 && tid == 0) {
    // Summation order can leave the children of the crossing bucket a hair
    // short of gamma; the crossing then lies in the lowest non-empty child.
    for (int b = 0; b < nbk; ++b) {
      if (hist->count[b] > 0) {
        s_bucket = b;
        s_above_new = base + (tsum[1023] - hist->mass[b]);
        s_found = 1;
        break;
      }
    }
  }
  __syncthreads();
  if (tid == 0 && !all) {
    if (!s_found) {
      st->all = 1u;   // the cumulative mass never reaches gamma: keep everything
    } else {
      const int bits = level == 2 ? 8 : 12;
      st->s_above = s_above_new;
      st->prefix = (st->prefix << bits) | (uint32_t)s_bucket;
      if (level == 2) {
        const uint32_t key = st->prefix;
        const double v = (double)__uint_as_float(key);
        const unsigned long long nt = hist->count[s_bucket];
        double need = (gamma - st->s_above) / v;
        unsigned long long t = need <= 1.0 ? 1ull : (unsigned long long)ceil(need);
        while (t > 1 && st->s_above + (double)(t - 1) * v >= gamma) --t;
        while (t < nt && st->s_above + (double)t * v < gamma) ++t;
        if (t > nt) t = nt;
        st->cut_key = key;
        st->n_ties = nt;
        st->t_keep = t;
      }
    }
  }
  __syncthreads();
  for (int b = tid; b < kHistL0; b += 1024) {
    hist->count[b] = 0;
    hist->mass[b] = 0.0;
  }
}

// Ties needed in part only: count entries equal to the cut value per row (one warp per row).
__global__ void __launch_bounds__(256) pe_tie_count_kernel(PeArgs a) {
  const int h = blockIdx.y;
  if (a.route[h] != 1) return;
  const PeState* st = a.state + h;
  if (st->all || st->t_keep >= st->n_ties) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * kRowsPerCta + warp;
  if (r >= a.nb) return;
  const float* row = a.tri_buf + (size_t)h * a.tri_stride + tri_off(r);
  uint32_t cnt = 0;
  for (int c = lane; c <= r; c += 32) cnt += (__float_as_uint(row[c]) == st->cut_key) ? 1u : 0u;
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) a.tie_rows[(size_t)h * a.nb + r] = cnt;
}

// Exclusive scan of the per-row tie counts (one CTA of 1024 threads per head).
__global__ void __launch_bounds__(1024) pe_tie_scan_kernel(PeArgs a) {
  const int h = blockIdx.x;
  if (a.route[h] != 1) return;
  const PeState* st = a.state + h;
  if (st->all || st->t_keep >= st->n_ties) return;
  __shared__ uint32_t part[1024];
  uint32_t* rows = a.tie_rows + (size_t)h * a.nb;
  const int per = (a.nb + 1023) / 1024;
  const int lo = threadIdx.x * per, hi = min(a.nb, lo + per);
  uint32_t s = 0;
  for (int r = lo; r < hi; ++r) s += rows[r];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const uint32_t v = threadIdx.x >= off ? part[threadIdx.x - off] : 0u;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  uint32_t acc = threadIdx.x > 0 ? part[threadIdx.x - 1] : 0u;
  for (int r = lo; r < hi; ++r) {
    const uint32_t v = rows[r];
    rows[r] = acc;
    acc += v;
  }
}

// Write the PE mask row by row (one warp per row): keep (r, c), c <= r, when
// its value is above the cut, or equal to it and among the first t_keep ties
// in flat order, or c == r; or everything when the cut keeps all.
__global__ void __launch_bounds__(256) pe_mask_kernel(PeArgs a) {
  const int h = blockIdx.y;
  if (a.route[h] != 1) return;
  const PeState* st = a.state + h;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * kRowsPerCta + warp;
  __shared__ unsigned long long kept_cta;
  if (threadIdx.x == 0) kept_cta = 0;
  __syncthreads();
  if (r < a.nb) {
    const bool all = st->all != 0;
    const uint32_t cut = st->cut_key;
    const bool partial_ties = !all && st->t_keep < st->n_ties;
    const unsigned long long t_keep = st->t_keep;
    unsigned long long tie_base = partial_ties ? a.tie_rows[(size_t)h * a.nb + r] : 0ull;
    const float* row = a.tri_buf + (size_t)h * a.tri_stride + tri_off(r);
    uint32_t* mrow = a.pe_mask + ((size_t)h * a.nb + r) * a.words;
    uint32_t kept = 0;
    for (int w = 0; w < a.words; ++w) {
      const int c = w * 32 + lane;
      int keep = 0, tie = 0;
      if (c <= r) {
        const uint32_t key = __float_as_uint(row[c]);
        tie = (!all && key == cut) ? 1 : 0;
        keep = all || c == r || key > cut || (tie && !partial_ties);
      }
      if (partial_ties) {
        const unsigned tb = __ballot_sync(0xffffffffu, tie);
        const unsigned long long rank = tie_base + __popc(tb & ((1u << lane) - 1u));
        if (tie && rank < t_keep) keep = 1;
        tie_base += __popc(tb);
      }
      const unsigned bal = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) mrow[w] = bal;
      kept += __popc(bal);
    }
    if (lane == 0) atomicAdd(&kept_cta, (unsigned long long)kept);
    if (lane == 0 && r == 0) a.pe_cut[h] = all ? 0.f : __uint_as_float(cut);
  }
  __syncthreads();
  if (threadIdx.x == 0 && kept_cta) atomicAdd(reinterpret_cast<unsigned long long*>(a.pe_count + h), kept_cta);
}

}  // namespace

cudaError_t launch_pe(const void* q, const void* k, const Shape& s, char* ws, const WsLayout& L,
                      const IndexPtrs& ix, cudaStream_t st) {
  PeArgs a;
  a.n = s.n;
  a.nb = s.nb;
  a.words = s.words;
  a.group = s.group;
  a.h_q = s.h_q;
  a.h_kv = s.h_kv;
  a.tri = s.tri;
  a.tri_stride = s.tri_stride;
  a.scale_log2 = s.scale_log2;
  a.gamma = s.gamma;
  a.route = ix.route;
  a.kv_pe = reinterpret_cast<const int32_t*>(ws + L.kv_pe);
  a.qbar = reinterpret_cast<float*>(ws + L.qbar);
  a.kbar = reinterpret_cast<float*>(ws + L.kbar);
  a.tri_buf = reinterpret_cast<float*>(ws + L.tri);
  a.tri_stats = reinterpret_cast<float4*>(ws + L.tri_stats);
  a.n_ct = (s.nb + kLT - 1) / kLT;
  a.hist = reinterpret_cast<PeHist*>(ws + L.hist);
  a.state = reinterpret_cast<PeState*>(ws + L.pe_state);
  a.tie_rows = reinterpret_cast<uint32_t*>(ws + L.tie_rows);
  a.pe_mask = ix.pe_mask;
  a.pe_count = ix.pe_count;
  a.pe_cut = ix.pe_cut;
  a.status = reinterpret_cast<int32_t*>(ws + L.status);

  cudaError_t e = cudaMemsetAsync(a.hist, 0, sizeof(PeHist) * s.h_q, st);
  if (e != cudaSuccess) return e;
  // the query-head pooling is gated by the route (1 = PE); the key pooling
  // by the per-group PE flag
  if (s.fp32) {
    pool_kernel<float><<<dim3(s.nb, s.h_q), 128, 0, st>>>(static_cast<const float*>(q), a.qbar, s.n, s.nb, ix.route);
    pool_kernel<float><<<dim3(s.nb, s.h_kv), 128, 0, st>>>(static_cast<const float*>(k), a.kbar, s.n, s.nb, a.kv_pe);
  } else {
    pool_kernel<__nv_bfloat16><<<dim3(s.nb, s.h_q), 128, 0, st>>>(static_cast<const __nv_bfloat16*>(q), a.qbar,
                                                                  s.n, s.nb, ix.route);
    pool_kernel<__nv_bfloat16><<<dim3(s.nb, s.h_kv), 128, 0, st>>>(static_cast<const __nv_bfloat16*>(k), a.kbar,
                                                                   s.n, s.nb, a.kv_pe);
  }
  const size_t lsmem = 2 * kHeadDim * kLStride * sizeof(float);
  e = cudaFuncSetAttribute(pe_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)lsmem);
  if (e != cudaSuccess) return e;
  const int nt = (s.nb + kLT2 - 1) / kLT2;
  {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int n_tri_tiles = nt * (nt + 1) / 2;
    const long long items = (long long)s.h_q * n_tri_tiles;
    pe_logits_kernel<<<(int)std::min<long long>(items, sms), 256, lsmem, st>>>(a, n_tri_tiles);
  }
  const int row_ctas = (s.nb + kRowsPerCta - 1) / kRowsPerCta;
  pe_softmax_kernel<<<dim3(row_ctas, s.h_q), 256, 0, st>>>(a);
  pe_find_kernel<<<s.h_q, 1024, 0, st>>>(a, 0);
  const int hist_ctas = (int)std::min<long long>(296, (s.tri / 4 + 255) / 256 + 1);
  const size_t hsm1 = (size_t)kHistL1 * 16, hsm2 = (size_t)kHistL2 * 16;
  e = cudaFuncSetAttribute(pe_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hsm1);
  if (e != cudaSuccess) return e;
  pe_hist_kernel<<<dim3(hist_ctas, s.h_q), 256, hsm1, st>>>(a, 1);
  pe_find_kernel<<<s.h_q, 1024, 0, st>>>(a, 1);
  pe_hist_kernel<<<dim3(hist_ctas, s.h_q), 256, hsm2, st>>>(a, 2);
  pe_find_kernel<<<s.h_q, 1024, 0, st>>>(a, 2);
  pe_tie_count_kernel<<<dim3(row_ctas, s.h_q), 256, 0, st>>>(a);
  pe_tie_scan_kernel<<<s.h_q, 1024, 0, st>>>(a);
  pe_mask_kernel<<<dim3(row_ctas, s.h_q), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace crisp
