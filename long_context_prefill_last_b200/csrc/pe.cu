// Pooled estimation (CRISP summary page, Algorithm 4, "GlobalAdaptive") on
// the 5th-generation tensor cores.
//
// What is computed, per query head routed PE: block means Q-bar, K-bar of Q
// and K (B = 128 rows), the pooled map A-bar = softmax over c <= r of
// sm_scale * Q-bar_r . K-bar_c, its flattened causal entries divided by their
// total (N_b, one per row), and the gamma-cumulative cut: the largest entries
// (ties by ascending flat index r*N_b + c) are kept until their mass reaches
// gamma. The diagonal block is always kept.
//
// How: the cut is found by a three-level radix select over the fp32 bit
// patterns of the (positive) entries, with per-bucket counts and mass in
// 64-bit fixed point (exact, so the sums do not depend on their order), and
// the map is never stored. Every pass evaluates an entry with the same
// expression, 2^(logit - row max) * row normaliser, so all see the same
// bits. Every pass recomputes the pooled logits it needs on the tensor
// cores: Q-bar * scale and K-bar are split into
// bf16 hi + lo parts and S = Qh.Kh^T + Ql.Kh^T + Qh.Kl^T (the lo.lo term is
// below fp32 rounding), with Q-bar held in tensor memory as the A operand
// and K-bar tiles fed by TMA. The passes:
//   1. stats + level-0: per 128-row stripe of the map, one sweep computes
//      each row's maximum and normaliser (online softmax), a second sweep
//      the entries, their level-0 histogram (bits 31..20) and, per tile, the
//      smallest and largest key;
//   2. level 1 (bits 19..8) and level 2 (bits 7..0): only tiles whose key
//      range meets the prefix found so far are recomputed, in segments of a
//      few tiles spread over the SMs;
//   3. ties (only when the cut keeps part of the entries equal to it): each
//      row's count of entries equal to the cut per tile, then a scan in flat
//      order (row by row, tile by tile) gives every tile's rank offset;
//   4. masks: a fill kernel writes the tiles entirely above (below) the cut
//      without recomputation; the sweep recomputes the tiles the cut crosses.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace crisp {
namespace {

enum PeMode : int { kStatsHist0 = 0, kHist1 = 1, kHist2 = 2, kTies = 3, kMask = 4 };

struct PeArgs {
  int nb, nt, words, group, h_q;
  float gamma;
  const int32_t* route;
  const __nv_bfloat16* qhi;   // [h_q][nb][128]  bf16(Q-bar * scale_log2)
  const __nv_bfloat16* qlo;   // [h_q][nb][128]  bf16(Q-bar * scale_log2 - qhi)
  float2* row_stat;           // [h_q][nb]        (row maximum, 1 / (row sum * N_b)), log2 domain
  uint2* tile_kr;             // [h_q][nt][nt][4] (min key, max key) per 32-row quarter of a tile
  uint32_t* tie_cnt;          // [h_q][nb][nt]    ties of the row per tile, then (tie scan) in the tiles before it
  uint32_t* tie_row;          // [h_q][nb]        ties per row, then exclusive offsets in flat order
  PeHist* hist;
  PeState* state;
  uint32_t* pe_mask;
  int64_t* pe_count;
  float* pe_cut;
  int32_t* status;
};

// ------------------------------------------------------------------ pooling

// Block means of Q (query heads routed PE) and K (KV groups with a PE head),
// written as bf16 hi/lo pairs; Q-bar is scaled by sm_scale * log2(e) first so
// the logits come out in the log2 domain. Persistent grid over (head, block)
// items; one 128 x 128 block per CTA iteration, every load issued before the
// first add (32 KB in flight per CTA).
template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&o)[8]) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
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
    const float4 u = __ldcs(reinterpret_cast<const float4*>(p));
    o[0] = u.x;
    o[1] = u.y;
    o[2] = u.z;
    o[3] = u.w;
  }
};

constexpr int kPoolThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kPoolThreads) pe_pool_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                               int n, int nb, int nb_pad, int h_q, int h_kv,
                                                               float scale, const int32_t* __restrict__ route,
                                                               const int32_t* __restrict__ kv_pe,
                                                               __nv_bfloat16* __restrict__ qhi,
                                                               __nv_bfloat16* __restrict__ qlo,
                                                               __nv_bfloat16* __restrict__ khi,
                                                               __nv_bfloat16* __restrict__ klo) {
  constexpr int N = Vec16<T>::N;
  constexpr int TPR = kHeadDim / N;            // threads per row
  constexpr int RP = kPoolThreads / TPR;       // rows in parallel
  constexpr int IT = kBlock / RP;              // rows per thread
  __shared__ float red[RP][kHeadDim + 1];
  const int tid = threadIdx.x, rg = tid / TPR, c0 = (tid % TPR) * N;
  // items: query heads x N_b blocks, then KV heads x nb_pad blocks (K-bar rows
  // past N_b are written as zeros so its TMA boxes never leave the tensor)
  const long long q_items = (long long)h_q * nb;
  const long long items = q_items + (long long)h_kv * nb_pad;
  const long long G = gridDim.x;
  for (long long it = blockIdx.x; it < items; it += G) {
    const bool is_q = it < q_items;
    const int hh = is_q ? (int)(it / nb) : (int)((it - q_items) / nb_pad);
    const int b = is_q ? (int)(it % nb) : (int)((it - q_items) % nb_pad);
    const bool want = is_q ? route[hh] == 1 : kv_pe[hh] != 0;
    if (!want) {   // uniform over the CTA: jump to this CTA's first item of the next head
      const long long next = is_q ? (long long)(hh + 1) * nb : q_items + (long long)(hh + 1) * nb_pad;
      it += ((next - it + G - 1) / G - 1) * G;
      continue;
    }
    float acc[N];
#pragma unroll
    for (int j = 0; j < N; ++j) acc[j] = 0.f;
    if (b < nb) {
      const T* base = (is_q ? q : k) + ((size_t)hh * n + (size_t)b * kBlock) * kHeadDim + c0;
      float v[IT][N];
#pragma unroll
      for (int i = 0; i < IT; ++i) Vec16<T>::load(base + (size_t)(rg + i * RP) * kHeadDim, v[i]);
#pragma unroll
      for (int j = 0; j < N; ++j) {
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < IT; ++i) s += v[i][j];
        acc[j] = s;
      }
    }
    __syncthreads();   // the previous item's reads of red are done
#pragma unroll
    for (int j = 0; j < N; ++j) red[rg][c0 + j] = acc[j];
    __syncthreads();
    if (tid < kHeadDim) {
      float s = 0.f;
#pragma unroll
      for (int g = 0; g < RP; ++g) s += red[g][tid];
      const float x = s * (1.f / kBlock) * (is_q ? scale : 1.f);
      const __nv_bfloat16 hi = __float2bfloat16_rn(x);
      const __nv_bfloat16 lo = __float2bfloat16_rn(x - __bfloat162float(hi));
      const size_t o = ((size_t)hh * (is_q ? nb : nb_pad) + b) * kHeadDim + tid;
      (is_q ? qhi : khi)[o] = hi;
      (is_q ? qlo : klo)[o] = lo;
    }
  }
}

// ------------------------------------------------------------------ the tensor-core sweep

// warp 0 TMA, warp 1 TMEM + MMA, warps 2-3 idle, warps 4..11 two epilogue
// warpgroups; the first warpgroup gives registers to the epilogue ones
// (setmaxnreg 64 / 216 / 216; 128*64 + 256*216 <= 384*168, the launch allocation)
constexpr int kThreads = 384;
constexpr int kRegsControl = 64;
constexpr int kRegsEpilogue = 216;
static_assert(128 * kRegsControl + 256 * kRegsEpilogue <= kThreads * 168, "register split exceeds the launch");
constexpr int kStages = 2;
constexpr uint32_t kTileBytes = 128 * 128 * 2;   // one bf16 128 x 128 tile (two 64-column halves)
constexpr uint32_t kHalfBytes = 128 * 128;
constexpr int kHistMax = kHistL1;                // largest per-CTA histogram (level 1)
constexpr uint32_t OFF_K = 0;                                      // [stage][hi, lo] K-bar tiles
constexpr uint32_t OFF_HCNT = OFF_K + kStages * 2 * kTileBytes;    // u32 [kHistMax]
constexpr uint32_t OFF_HMASS = OFF_HCNT + kHistMax * 4;            // u64 [kHistMax] fixed-point mass (level 0),
                                                                   // u32 [kHistMax] low-bit sums (level 1)
constexpr uint32_t OFF_XCH = OFF_HMASS + kHistMax * 8;             // float2 [128]: row statistics exchange
constexpr uint32_t OFF_ROW = OFF_XCH + 128 * 8;                    // float2 [128]: (m, inv) of the stripe's rows
constexpr uint32_t OFF_LIVE = OFF_ROW + 128 * 8;                   // int [kMaxHeads + 1]: count, then PE heads
constexpr uint32_t OFF_BAR = OFF_LIVE + (((kMaxHeads + 1) * 4 + 7) & ~7);
enum {
  B_KFULL = 0,
  B_KEMPTY = B_KFULL + kStages,
  B_SFULL = B_KEMPTY + kStages,   // [2]
  B_SEMPTY = B_SFULL + 2,         // [2], 128 arrivals (one warpgroup)
  B_QFULL = B_SEMPTY + 2,         // [2], 256 arrivals (both warpgroups)
  B_QEMPTY = B_QFULL + 2,         // [2], MMA commit after a stripe's last tile
  B_EPI = B_QEMPTY + 2,           // epilogue-wide sync, 256 arrivals
  B_DRAIN = B_EPI + 1,
  B_COUNT = B_DRAIN + 1
};
constexpr uint32_t OFF_ABORT = OFF_BAR + 8 * B_COUNT;
constexpr uint32_t OFF_TMEMPTR = OFF_ABORT + 4;
constexpr uint32_t kSmemBytes = OFF_TMEMPTR + 4 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
// TMEM: S[0] cols [0,128), S[1] [128,256); Q[b] at 256 + 128 b: hi [0,64), lo [64,128)
constexpr uint32_t kTmemCols = 512;

__device__ __forceinline__ uint32_t bar_addr(uint32_t base, int i) { return base + OFF_BAR + 8u * i; }

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int32_t* status,
                                          int where) {
  const bool ok = dev::mbar_wait(bar, parity, abort_flag, status, where);
  return __all_sync(0xffffffffu, ok);
}

// Work items. The statistics pass takes whole 128-row stripes (its per-row
// running maximum and sum need every tile of a row); the later passes split a
// stripe into segments of 8 tiles, since the tiles they recompute sit in the
// few stripes whose rows straddle the prefix or the cut, and whole stripes
// would leave those to a handful of CTAs (2-tile segments measured slower:
// every item pays for its key ranges and its Q-bar load).
__device__ __forceinline__ bool segmented(int mode) { return mode != kStatsHist0; }
__device__ __forceinline__ int seg_tiles(int) { return 8; }

struct Item {
  int h, rt;    // query head, row tile (stripe)
  int c0, c1;   // tiles c0..c1 of the stripe
  bool last;    // the segment holding the diagonal tile
};

// Item k of CTA b: a snake over the items of the heads routed PE (`live`,
// n_live of them), ordered stripe rt descending, then segment, then head.
__device__ __forceinline__ bool item_of(const PeArgs& a, const int* live, int n_live, int mode, int b, int k,
                                        Item& it) {
  const int G = gridDim.x;   // items per head <= 64 * 8, so every index fits an int
  const int seg = segmented(mode) ? seg_tiles(mode) : 64;
  int idx = (k & 1) ? (k + 1) * G - 1 - b : k * G + b;
  for (int rt = a.nt - 1; rt >= 0; --rt) {
    const int cnt = (rt / seg + 1) * n_live;
    if (idx < cnt) {
      const int sg = idx / n_live;
      it.h = live[idx - sg * n_live];
      it.rt = rt;
      it.c0 = sg * seg;
      it.c1 = min(rt, it.c0 + seg - 1);
      it.last = it.c1 == rt;
      return true;
    }
    idx -= cnt;
  }
  return false;
}

struct PassCtx {
  int mode;
  uint32_t lo_key, hi_key;   // keys a tile must reach to be recomputed
  uint32_t cut;              // level-2 result (ties, mask)
  bool all;                  // the cut keeps every entry
  bool partial_ties;
  unsigned long long t_keep;
  uint32_t prefix;
};

// Whether head h takes part in this pass, and its pass parameters.
__device__ __forceinline__ bool head_live(const PeArgs& a, int mode, int h, PassCtx& c) {
  if (a.route[h] != 1) return false;
  c.mode = mode;
  if (mode == kStatsHist0) return true;
  const PeState* st = a.state + h;
  c.all = st->all != 0;
  c.cut = st->cut_key;
  c.prefix = st->prefix;
  c.t_keep = st->t_keep;
  c.partial_ties = !c.all && st->t_keep < st->n_ties;
  if (mode == kHist1) {
    c.lo_key = c.prefix << 20;
    c.hi_key = c.lo_key | 0xFFFFFu;
    return !c.all;
  }
  if (mode == kHist2) {
    c.lo_key = c.prefix << 8;
    c.hi_key = c.lo_key | 0xFFu;
    return !c.all;
  }
  c.lo_key = c.hi_key = c.cut;
  if (mode == kTies) return c.partial_ties;
  return true;   // kMask
}

// Key range of tile (rt, ct) of head h recorded by the level-0 sweep.
__device__ __forceinline__ void tile_range(const PeArgs& a, int h, int rt, int ct, uint32_t& kmin, uint32_t& kmax) {
  const uint2* p = a.tile_kr + (((size_t)h * a.nt + rt) * a.nt + ct) * 4;
  kmin = 0xFFFFFFFFu;
  kmax = 0u;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint2 e = p[q];
    kmin = min(kmin, e.x);
    kmax = max(kmax, e.y);
  }
}

// Whether tile (rt, ct) is recomputed on the tensor cores in this pass.
__device__ __forceinline__ bool tile_active(const PeArgs& a, const PassCtx& c, int h, int rt, int ct) {
  if (c.mode == kStatsHist0) return true;
  if (c.mode == kMask && c.all) return false;
  uint32_t kmin, kmax;
  tile_range(a, h, rt, ct, kmin, kmax);
  return kmin <= c.hi_key && kmax >= c.lo_key;
}

// The tiles c0 <= ct <= c1 of item `it` recomputed in this pass, as a bit
// mask (N_b <= 8192, so at most 64 tiles). Evaluated by a whole warp, one
// tile per lane, so the key ranges are read in one round.
__device__ __forceinline__ uint64_t stripe_mask(const PeArgs& a, const PassCtx& c, const Item& it, int lane) {
  const bool a0 = lane >= it.c0 && lane <= it.c1 && tile_active(a, c, it.h, it.rt, lane);
  const bool a1 = lane + 32 >= it.c0 && lane + 32 <= it.c1 && tile_active(a, c, it.h, it.rt, lane + 32);
  return (uint64_t)__ballot_sync(0xffffffffu, a0) | ((uint64_t)__ballot_sync(0xffffffffu, a1) << 32);
}

__device__ __forceinline__ int sweeps_of(int mode) { return mode == kStatsHist0 ? 2 : 1; }

// Epilogue-wide barrier (256 threads) with a bounded wait.
__device__ __forceinline__ bool epi_sync(uint32_t sbase, uint32_t& phase, volatile int* abort_flag,
                                         int32_t* status) {
  dev::mbar_arrive(bar_addr(sbase, B_EPI));
  const bool ok = warp_wait(bar_addr(sbase, B_EPI), phase, abort_flag, status, 40);
  phase ^= 1u;
  return ok;
}

// Mass is kept in fixed point, units of 2^-62 (entries are at most 1/4).
// bucket_mass gives the summed mass of `cnt` entries whose keys agree with
// `key_base` on every bit above some low bits (zero in key_base) and whose low
// bits add up to `low`. A positive normal float is (2^23 + mantissa) *
// 2^(exponent - 150), so the sum is (cnt * (2^23 + high mantissa bits) + low)
// * 2^(exponent - 150): integer arithmetic, exact for entries of at least
// 2^-38 (then every entry is a whole number of units); smaller ones are
// truncated to whole units and subnormal ones count 0. Histograms keep
// (count, low-bit sum) per bucket in 32-bit integers and convert once.
__device__ __forceinline__ unsigned long long bucket_mass(uint32_t key_base, uint32_t cnt, unsigned long long low) {
  const int e = (int)(key_base >> 23);
  if (e == 0) return 0ull;
  const unsigned long long x = (unsigned long long)cnt * (0x800000u | (key_base & 0x7FFFFFu)) + low;
  return e >= 88 ? x << (e - 88) : x >> (88 - e);
}

__device__ __forceinline__ void hist_add(uint32_t* cnt, unsigned long long* mass, uint32_t b, uint32_t c,
                                         unsigned long long m) {
  atomicAdd(&cnt[b], c);
  atomicAdd(&mass[b], m);
}

__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
pe_sweep_kernel(const __grid_constant__ CUtensorMap tm_khi, const __grid_constant__ CUtensorMap tm_klo, PeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = dev::smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + OFF_ABORT);
  uint32_t* tmem_ptr_smem = reinterpret_cast<uint32_t*>(sgen + OFF_TMEMPTR);
  uint32_t* hcnt = reinterpret_cast<uint32_t*>(sgen + OFF_HCNT);
  unsigned long long* hmass = reinterpret_cast<unsigned long long*>(sgen + OFF_HMASS);
  uint32_t* hlow = reinterpret_cast<uint32_t*>(sgen + OFF_HMASS);   // level 1: low-bit sums in hmass's space
  float2* xch = reinterpret_cast<float2*>(sgen + OFF_XCH);
  float2* rows_sm = reinterpret_cast<float2*>(sgen + OFF_ROW);
  int* live_sm = reinterpret_cast<int*>(sgen + OFF_LIVE);
  const int* live = live_sm + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbk = MODE == kHist1 ? kHistL1 : MODE == kHist2 ? kHistL2 : 1024;

  if (threadIdx.x == 0) {
    *abort_flag = dev::load_volatile(a.status) != 0 ? 1 : 0;
    for (int s = 0; s < kStages; ++s) {
      dev::mbar_init(bar_addr(sbase, B_KFULL + s), 1);
      dev::mbar_init(bar_addr(sbase, B_KEMPTY + s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      dev::mbar_init(bar_addr(sbase, B_SFULL + x), 1);
      dev::mbar_init(bar_addr(sbase, B_SEMPTY + x), 128);
      dev::mbar_init(bar_addr(sbase, B_QFULL + x), 256);
      dev::mbar_init(bar_addr(sbase, B_QEMPTY + x), 1);
    }
    dev::mbar_init(bar_addr(sbase, B_EPI), 256);
    dev::mbar_init(bar_addr(sbase, B_DRAIN), 1);
    dev::fence_mbar_init();
  }
  for (int i = threadIdx.x; i < kHistMax; i += kThreads) {
    hcnt[i] = 0u;
    hmass[i] = 0ull;
  }
  if (warp == 0) {   // the heads routed PE, in order
    int cnt = 0;
    for (int h0 = 0; h0 < a.h_q; h0 += 32) {
      const bool pe = h0 + lane < a.h_q && a.route[h0 + lane] == 1;
      const uint32_t bal = __ballot_sync(0xffffffffu, pe);
      if (pe) live_sm[1 + cnt + __popc(bal & ((1u << lane) - 1u))] = h0 + lane;
      cnt += __popc(bal);
    }
    if (lane == 0) live_sm[0] = cnt;
  }
  __syncthreads();
  const int n_live = live_sm[0];
  // an earlier kernel failed, or no head is routed PE: nothing to do
  // (uniform, before TMEM is taken)
  if (*abort_flag || n_live == 0) return;
  if (warp == 1) {
    dev::tmem_alloc(dev::smem_u32(tmem_ptr_smem), kTmemCols);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = *tmem_ptr_smem;

  if (warp < 4) dev::regs_release<kRegsControl>();
  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // the whole warp walks the stripes (tile masks); lane 0 issues the copies
    if (lane == 0) {
      dev::prefetch_tmap(&tm_khi);
      dev::prefetch_tmap(&tm_klo);
    }
    int kt = 0;
    bool ok = true;
    PassCtx c;
    Item item;
    for (int it = 0; ok && item_of(a, live, n_live, MODE, blockIdx.x, it, item); ++it) {
      if (!head_live(a, MODE, item.h, c)) continue;
      const uint64_t act = stripe_mask(a, c, item, lane);
      const int g = item.h / a.group;
      for (int sw = 0; ok && sw < sweeps_of(MODE); ++sw) {
        for (uint64_t m = act; ok && m; m &= m - 1) {
          const int ct = __ffsll((long long)m) - 1;
          const int s = kt % kStages;
          if (lane == 0) {
            ok = dev::mbar_wait(bar_addr(sbase, B_KEMPTY + s), ((kt / kStages) & 1) ^ 1, abort_flag, a.status, 41);
            if (ok) {
              const uint32_t bk = bar_addr(sbase, B_KFULL + s);
              const uint32_t dst = sbase + OFF_K + s * 2 * kTileBytes;
              dev::mbar_arrive_expect_tx(bk, 2 * kTileBytes);
              dev::tma_load_3d(dst, &tm_khi, bk, 0, ct * 128, g);
              dev::tma_load_3d(dst + kHalfBytes, &tm_khi, bk, 64, ct * 128, g);
              dev::tma_load_3d(dst + kTileBytes, &tm_klo, bk, 0, ct * 128, g);
              dev::tma_load_3d(dst + kTileBytes + kHalfBytes, &tm_klo, bk, 64, ct * 128, g);
            }
          }
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (ok) ++kt;
        }
      }
    }
    if (!ok && lane == 0) {   // let the copies in flight land before the CTA exits
      for (int s = 0; s < kStages && s < kt; ++s) {
        const int last = kt - 1 - ((kt - 1 - s) % kStages);
        dev::mbar_drain(bar_addr(sbase, B_KFULL + s), (last / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // the whole warp walks the items and waits (descriptors stay
    // warp-uniform); one elected lane issues every tcgen05.mma and commit
    const uint32_t idesc = dev::umma_idesc_bf16(128, 128, false);
    const uint64_t KD0 = dev::smem_desc_sw128(sbase + OFF_K, 16, 1024);
    int kt = 0, j = 0, qi = 0;
    bool ok = true;
    PassCtx c;
    Item item;
    for (int it = 0; ok && item_of(a, live, n_live, MODE, blockIdx.x, it, item); ++it) {
      if (!head_live(a, MODE, item.h, c)) continue;
      const uint64_t act = stripe_mask(a, c, item, lane);
      if (act == 0) continue;
      if (!warp_wait(bar_addr(sbase, B_QFULL + (qi & 1)), (qi >> 1) & 1, abort_flag, a.status, 42)) {
        ok = false;
        break;
      }
      dev::tc_fence_after();
      const uint32_t qcol = tmem + 256u + (uint32_t)(qi & 1) * 128u;
      for (int sw = 0; ok && sw < sweeps_of(MODE); ++sw) {
        for (uint64_t m = act; ok && m; m &= m - 1) {
          const int s = kt % kStages, buf = j & 1;
          ok = warp_wait(bar_addr(sbase, B_KFULL + s), (kt / kStages) & 1, abort_flag, a.status, 43);
          if (ok && j >= 2)
            ok = warp_wait(bar_addr(sbase, B_SEMPTY + buf), ((j - 2) >> 1) & 1, abort_flag, a.status, 44);
          if (ok) {
            dev::tc_fence_after();
            // K-bar hi then lo of stage s (each a whole tile further in the start-address field)
            const uint64_t kh = KD0 + (uint64_t)(s * 2 * (kTileBytes >> 4)), kl = kh + (kTileBytes >> 4);
            const uint32_t d = tmem + (uint32_t)buf * 128u;
            dev::umma_ts8k_w(d, qcol, kh, idesc, 0u);        // Qh . Kh
            dev::umma_ts8k_w(d, qcol + 64, kh, idesc, 1u);   // Ql . Kh
            dev::umma_ts8k_w(d, qcol, kl, idesc, 1u);        // Qh . Kl
            dev::umma_commit_w(bar_addr(sbase, B_SFULL + buf));
            dev::umma_commit_w(bar_addr(sbase, B_KEMPTY + s));
          }
          ++kt;
          ++j;
        }
      }
      dev::umma_commit_w(bar_addr(sbase, B_QEMPTY + (qi & 1)));   // this stripe's Q-bar is no longer read
      ++qi;
    }
    // every MMA issued completes before TMEM is released
    dev::umma_commit_w(bar_addr(sbase, B_DRAIN));
    dev::mbar_drain(bar_addr(sbase, B_DRAIN), 0);
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- epilogue warpgroups
    dev::regs_acquire<kRegsEpilogue>();
    const int wg = (warp - 4) >> 2;               // 0 or 1: the tiles j with j % 2 == wg
    const int quarter = warp & 3;                 // TMEM lane quarter of this warp
    const int lr = quarter * 32 + lane;           // row inside the tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    uint32_t epi_phase = 0;
    int j = 0, qi = 0;
    bool ok = true;
    PassCtx c;
    Item item;

    // write the Q-bar rows of stripe (hq, rtq) into TMEM buffer `buf` (this
    // warpgroup's half: hi for warpgroup 0, lo for 1); q = its index among the
    // stripes with tensor-core work
    auto write_q = [&](int hq, int rtq, int q) -> bool {
      const int buf = q & 1;
      if (q >= 2 && !warp_wait(bar_addr(sbase, B_QEMPTY + buf), ((q - 2) >> 1) & 1, abort_flag, a.status, 45))
        return false;
      dev::tc_fence_after();
      const int r = rtq * 128 + lr;
      const __nv_bfloat16* src = (wg == 0 ? a.qhi : a.qlo) + ((size_t)hq * a.nb + r) * kHeadDim;
      const uint32_t col = tmem + lane_base + 256u + (uint32_t)buf * 128u + (uint32_t)wg * 64u;
#pragma unroll
      for (int part = 0; part < 4; ++part) {
        uint32_t w[16];
        if (r < a.nb) {
          const uint4* p = reinterpret_cast<const uint4*>(src + part * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            const uint4 u = p[x];
            w[4 * x] = u.x;
            w[4 * x + 1] = u.y;
            w[4 * x + 2] = u.z;
            w[4 * x + 3] = u.w;
          }
        } else {
#pragma unroll
          for (int x = 0; x < 16; ++x) w[x] = 0u;
        }
        dev::tmem_st16(col + part * 16, w);
      }
      dev::tmem_wait_st();
      dev::tc_fence_before();
      dev::mbar_arrive(bar_addr(sbase, B_QFULL + buf));
      return true;
    };
    // next item after item `it` with tensor-core work, for the Q prefetch
    auto next_active = [&](int it, int& hn, int& rtn) -> bool {
      PassCtx cn;
      Item in;
      for (int k = it + 1; item_of(a, live, n_live, MODE, blockIdx.x, k, in); ++k)
        if (head_live(a, MODE, in.h, cn) && stripe_mask(a, cn, in, lane) != 0) {
          hn = in.h;
          rtn = in.rt;
          return true;
        }
      return false;
    };
    // Quarter q (columns [32q, 32q + 32)) of the S tile j into x; the first
    // quarter waits for the tile, the last releases its buffer once loaded.
    auto load_q = [&](int qq, float (&x)[32]) -> bool {
      const int buf = j & 1;
      if (qq == 0) {
        if (!warp_wait(bar_addr(sbase, B_SFULL + buf), (j >> 1) & 1, abort_flag, a.status, 46)) return false;
        dev::tc_fence_after();
      }
      dev::tmem_ld32(tmem + lane_base + (uint32_t)buf * 128u + (uint32_t)qq * 32u,
                     reinterpret_cast<uint32_t (&)[32]>(x));
      dev::tmem_wait_ld();
      if (qq == 3) {
        dev::tc_fence_before();
        dev::mbar_arrive(bar_addr(sbase, B_SEMPTY + buf));
      }
      return true;
    };
    // add the CTA's histogram of head hh to the head's global one and clear
    // it; levels 1 and 2 turn (count, low-bit sum) into mass here
    auto flush_hist = [&](int hh) -> bool {
      if (!epi_sync(sbase, epi_phase, abort_flag, a.status)) return false;
      PeHist* gh = a.hist + hh;
      for (int i = threadIdx.x - 128; i < nbk; i += 256) {
        const uint32_t cnt = hcnt[i];
        if (cnt) {
          unsigned long long m;
          if (MODE == kHist1) {
            m = bucket_mass((c.prefix << 20) | ((uint32_t)i << 8), cnt, hlow[i]);
            hlow[i] = 0u;
          } else if (MODE == kHist2) {
            m = bucket_mass((c.prefix << 8) | (uint32_t)i, cnt, 0ull);
          } else {
            m = hmass[i];
            hmass[i] = 0ull;
          }
          atomicAdd(&gh->count[i], (unsigned long long)cnt);
          atomicAdd(&gh->mass[i], m);
          hcnt[i] = 0u;
        }
      }
      return epi_sync(sbase, epi_phase, abort_flag, a.status);
    };

    {   // the first stripe with tensor-core work
      int h0, rt0;
      if (next_active(-1, h0, rt0)) ok = write_q(h0, rt0, 0);
    }
    for (int it = 0; ok && item_of(a, live, n_live, MODE, blockIdx.x, it, item); ++it) {
      const int h = item.h, rt = item.rt;
      if (!head_live(a, MODE, h, c)) continue;
      const uint64_t act_mask = stripe_mask(a, c, item, lane);
      const int n_act = __popcll(act_mask);
      if (n_act > 0) {
        int hn, rtn;
        if (next_active(it, hn, rtn) && !write_q(hn, rtn, qi + 1)) {
          ok = false;
          break;
        }
      }
      const int r = rt * 128 + lr;
      const bool row_ok = r < a.nb;
      const int ncol = row_ok ? r - rt * 128 : -1;     // last valid column of the diagonal tile
      // last valid column of tile ct: every column before the diagonal tile
      // (c <= r < N_b), up to the diagonal in it, none in a padding row
      auto last_of = [&](int ct) { return !row_ok ? -1 : (ct < rt ? 127 : ncol); };
      float x[32];
      if (MODE == kStatsHist0) {
        // sweep 1: this warpgroup's tiles, running maximum and normaliser per row
        float m = -INFINITY, l = 0.f;
        for (int ct = 0; ct <= rt; ++ct, ++j) {
          if ((j & 1) != wg) continue;
          const int last = last_of(ct);
#pragma unroll 1
          for (int qq = 0; qq < 4; ++qq) {
            if (!load_q(qq, x)) {
              ok = false;
              break;
            }
            const int lastc = last - 32 * qq;   // valid: i <= lastc
            float hm = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i) hm = i <= lastc ? fmaxf(hm, x[i]) : hm;
            const float mn = fmaxf(m, hm);
            l *= mn == m ? 1.f : dev::ex2(m - mn);
            m = mn;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[i & 3] += dev::ex2(i <= lastc ? x[i] - m : -INFINITY);
            l += (acc[0] + acc[1]) + (acc[2] + acc[3]);
          }
          if (!ok) break;
        }
        if (!ok) break;
        // the two warpgroups' statistics of each row, combined
        if (wg == 1) xch[lr] = make_float2(m, l);
        if (!epi_sync(sbase, epi_phase, abort_flag, a.status)) {
          ok = false;
          break;
        }
        if (wg == 0) {
          const float2 o = xch[lr];
          const float M = fmaxf(m, o.x);
          const float L = (m == -INFINITY ? 0.f : l * dev::ex2(m - M)) + (o.x == -INFINITY ? 0.f : o.y * dev::ex2(o.x - M));
          const float2 st = make_float2(M, 1.f / (L * (float)a.nb));
          rows_sm[lr] = st;
          if (row_ok) a.row_stat[(size_t)h * a.nb + r] = st;
        }
        if (!epi_sync(sbase, epi_phase, abort_flag, a.status)) {
          ok = false;
          break;
        }
        const float2 st = rows_sm[lr];
        // A row's largest entry is its normaliser inv (at l = m), so its
        // entries fall in level-0 buckets at or below that of inv, in a
        // near-uniform row in that bucket or the next ones down. Counts and
        // low-bit sums of those three buckets are kept per row in registers
        // (predicated adds) and merged, once per tile, over the lanes whose
        // rows share the bucket; the entries further down go to the shared
        // histogram as they come.
        const uint32_t b_base = row_ok ? (__float_as_uint(st.y) >> 20) : 0u;
        const uint32_t b_grp = __match_any_sync(0xffffffffu, b_base);   // lanes with the same row bucket
        // sweep 2: entries, level-0 histogram, tile key ranges
        for (int ct = 0; ct <= rt; ++ct, ++j) {
          if ((j & 1) != wg) continue;
          const int last = last_of(ct);
          uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
          // per window: entry count and the sum of the low 20 key bits
          // (at most 128 * 2^20 per thread and tile)
          uint32_t c0 = 0, c1 = 0, c2 = 0;
          uint32_t l0 = 0, l1 = 0, l2 = 0;
#pragma unroll 1
          for (int qq = 0; qq < 4; ++qq) {
            if (!load_q(qq, x)) {
              ok = false;
              break;
            }
            const int lastc = last - 32 * qq;
            bool far = false;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const bool valid = i <= lastc;
              const float v = dev::ex2(valid ? x[i] - st.x : -INFINITY) * st.y;
              const uint32_t key = __float_as_uint(v);
              kmin = valid ? min(kmin, key) : kmin;
              kmax = max(kmax, key);   // masked entries are 0.0f (key 0)
              const uint32_t off = valid ? b_base - (key >> 20) : 0xFFFFFFFFu;
              const uint32_t low = key & 0xFFFFFu;
              c0 += off == 0 ? 1u : 0u;
              l0 += off == 0 ? low : 0u;
              c1 += off == 1 ? 1u : 0u;
              l1 += off == 1 ? low : 0u;
              c2 += off == 2 ? 1u : 0u;
              l2 += off == 2 ? low : 0u;
              far = far || (valid && off > 2u);
            }
            if (__any_sync(0xffffffffu, far)) {
              // entries below the window: the lanes of a column that share a
              // bucket are merged first (count, low-bit sum), so a column whose
              // rows agree costs one shared atomic instead of 32
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const bool valid = i <= lastc;
                const uint32_t key = __float_as_uint(dev::ex2(valid ? x[i] - st.x : -INFINITY) * st.y);
                const bool out = valid && b_base - (key >> 20) > 2u;
                const uint32_t outs = __ballot_sync(0xffffffffu, out);
                if (out) {
                  const uint32_t b = key >> 20;
                  const uint32_t grp = __match_any_sync(outs, b);
                  const uint32_t lsum = __reduce_add_sync(grp, key & 0xFFFFFu);
                  const uint32_t cnt = __popc(grp);
                  if (lane == __ffs(grp) - 1) hist_add(hcnt, hmass, b, cnt, bucket_mass(b << 20, cnt, lsum));
                }
              }
            }
          }
          if (!ok) break;
          {
            // the rows of b_grp share b_base: sum their windows (the low-bit
            // sums in 16-bit halves, so 32 lanes cannot overflow) and let the
            // group's first lane add them
            const uint32_t cs[3] = {__reduce_add_sync(b_grp, c0), __reduce_add_sync(b_grp, c1),
                                    __reduce_add_sync(b_grp, c2)};
            const unsigned long long ls[3] = {
                ((unsigned long long)__reduce_add_sync(b_grp, l0 >> 16) << 16) + __reduce_add_sync(b_grp, l0 & 0xFFFFu),
                ((unsigned long long)__reduce_add_sync(b_grp, l1 >> 16) << 16) + __reduce_add_sync(b_grp, l1 & 0xFFFFu),
                ((unsigned long long)__reduce_add_sync(b_grp, l2 >> 16) << 16) + __reduce_add_sync(b_grp, l2 & 0xFFFFu)};
            if (lane == __ffs(b_grp) - 1) {
#pragma unroll
              for (int w = 0; w < 3; ++w)
                if (cs[w] && b_base >= (uint32_t)w)
                  hist_add(hcnt, hmass, b_base - w, cs[w], bucket_mass((b_base - w) << 20, cs[w], ls[w]));
            }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
            kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
          }
          if (lane == 0) a.tile_kr[(((size_t)h * a.nt + rt) * a.nt + ct) * 4 + quarter] = make_uint2(kmin, kmax);
        }
        if (!ok) break;
        if (!flush_hist(h)) {
          ok = false;
          break;
        }
      } else {
        const float2 st = row_ok ? a.row_stat[(size_t)h * a.nb + r] : make_float2(0.f, 0.f);
        uint32_t* mrow = a.pe_mask + ((size_t)h * a.nb + (row_ok ? r : 0)) * a.words;
        uint32_t* trow = a.tie_cnt + ((size_t)h * a.nb + (row_ok ? r : 0)) * a.nt;
        unsigned long long kept = 0;
        if (MODE == kTies) {
          // each row's count of entries equal to the cut, per tile; the tie
          // scan turns them into running counts in flat order
          for (int ct = item.c0; ct <= item.c1; ++ct) {
            const bool act = (act_mask >> ct) & 1ull;
            const int owner = act ? (j & 1) : (ct & 1);
            if (owner != wg) {
              if (act) ++j;
              continue;
            }
            uint32_t cnt = 0;
            if (act) {
              const int last = last_of(ct);
#pragma unroll 1
              for (int qq = 0; qq < 4; ++qq) {
                if (!load_q(qq, x)) {
                  ok = false;
                  break;
                }
                const int lastc = last - 32 * qq;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                  const bool valid = i <= lastc;
                  const uint32_t key = __float_as_uint(dev::ex2(valid ? x[i] - st.x : -INFINITY) * st.y);
                  cnt += (valid && key == c.cut) ? 1u : 0u;
                }
              }
              if (!ok) break;
              ++j;
            }
            if (row_ok) trow[ct] = cnt;
          }
          if (!ok) break;
        }
        // Levels 1 and 2 keep, per bucket of the shared histogram, the entry
        // count and (level 1) the sum of the key bits below the bucket (8
        // bits), both 32-bit shared atomics; flush_hist turns them into mass.
        for (int ct = item.c0; MODE != kTies && ct <= item.c1; ++ct) {
          const bool act = (act_mask >> ct) & 1ull;
          const int last = last_of(ct);
          const int owner = act ? (j & 1) : (ct & 1);
          if (owner != wg || !act) {   // tiles the cut does not cross: pe_mask_fill_kernel
            if (act) ++j;
            continue;
          }
          if (MODE == kHist1 || MODE == kHist2) {
#pragma unroll 1
            for (int qq = 0; qq < 4; ++qq) {
              if (!load_q(qq, x)) {
                ok = false;
                break;
              }
              const int lastc = last - 32 * qq;
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const bool valid = i <= lastc;
                const uint32_t key = __float_as_uint(dev::ex2(valid ? x[i] - st.x : -INFINITY) * st.y);
                if (MODE == kHist1) {
                  if (valid && (key >> 20) == c.prefix) {
                    atomicAdd(&hcnt[(key >> 8) & 0xFFFu], 1u);
                    atomicAdd(&hlow[(key >> 8) & 0xFFFu], key & 0xFFu);
                  }
                } else if (valid && (key >> 8) == c.prefix) {
                  atomicAdd(&hcnt[key & 0xFFu], 1u);
                }
              }
            }
            if (!ok) break;
            ++j;
          } else {   // kMask, a tile the cut crosses
            uint32_t w[4] = {0u, 0u, 0u, 0u};
            {
              unsigned long long rank =
                  c.partial_ties && row_ok ? (unsigned long long)a.tie_row[(size_t)h * a.nb + r] + trow[ct] : 0ull;
              const int diag = ct == rt ? ncol : -1;
#pragma unroll 1
              for (int qq = 0; qq < 4; ++qq) {
                if (!load_q(qq, x)) {
                  ok = false;
                  break;
                }
                const int lastc = last - 32 * qq;
                uint32_t word = 0u;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                  const bool valid = i <= lastc;
                  const uint32_t key = __float_as_uint(dev::ex2(valid ? x[i] - st.x : -INFINITY) * st.y);
                  const bool tie = valid && key == c.cut;
                  const bool keep = (valid && key > c.cut) || (tie && (!c.partial_ties || rank < c.t_keep)) ||
                                    (32 * qq + i == diag);
                  rank += tie ? 1ull : 0ull;
                  word |= keep ? 1u << i : 0u;
                }
                // w[qq] with qq a loop variable would live in local memory: select instead
                w[0] = qq == 0 ? word : w[0];
                w[1] = qq == 1 ? word : w[1];
                w[2] = qq == 2 ? word : w[2];
                w[3] = qq == 3 ? word : w[3];
              }
              if (!ok) break;
              ++j;
            }
            if (row_ok) {
              if (ct == rt) w[ncol >> 5] |= 1u << (ncol & 31);   // the diagonal block
#pragma unroll
              for (int x4 = 0; x4 < 4; ++x4) {
                const int word = ct * 4 + x4;
                if (word < a.words) {
                  mrow[word] = w[x4];
                  kept += __popc(w[x4]);
                }
              }
            }
          }
        }
        if (!ok) break;
        if ((MODE == kHist1 || MODE == kHist2) && n_act > 0) {
          if (!flush_hist(h)) {
            ok = false;
            break;
          }
        }
        if (MODE == kMask) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) kept += __shfl_xor_sync(0xffffffffu, kept, o);
          if (lane == 0 && kept) atomicAdd(reinterpret_cast<unsigned long long*>(a.pe_count + h), kept);
        }
      }
      if (n_act > 0) ++qi;
    }
    dev::tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ the cut

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
      st->n_ties = 0;
      st->t_keep = 0;
      st->cut_key = 0;
    }
    s_found = 0;
  }
  __syncthreads();
  const bool all = st->all != 0;
  // thread tid owns descending buckets [nbk-1 - tid*per, ... - per + 1]
  double my = 0.0;
  for (int u = 0; u < per; ++u) {
    const int b = nbk - 1 - (tid * per + u);
    if (b >= 0) my += (double)hist->mass[b] * kMassUnit;
  }
  tsum[tid] = my;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {   // inclusive scan over threads (descending bucket order)
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
        const double nxt = acc + (double)hist->mass[b] * kMassUnit;
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
        s_above_new = base + (tsum[1023] - (double)hist->mass[b] * kMassUnit);
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
    hist->mass[b] = 0ull;
  }
}

// Exclusive scan over rows of the per-row tie counts, for heads whose cut
// keeps part of its ties: flat order is row by row, so a tie's rank is its
// row's offset plus the ties before it in the row (kept per tile by the
// ties pass). One CTA of 1024 threads per head.
// Masks of the tiles the cut does not cross, for stripe blockIdx.x of head
// blockIdx.y: all ones for c <= r in tiles entirely above the cut (every tile
// when the cut keeps everything), zero in tiles entirely below it and past
// the diagonal tile, and the diagonal block always kept. Tiles the cut crosses
// are left to the mask sweep, which decides them with the same tile key
// ranges. Each tile is classified once; the stripe's words are then written
// row by row (coalesced). Adds the kept blocks to pe_count.
__global__ void __launch_bounds__(256) pe_mask_fill_kernel(PeArgs a) {
  const int h = blockIdx.y, rt = blockIdx.x;
  if (a.route[h] != 1) return;
  __shared__ int8_t kind[64];   // per tile ct <= rt: 1 above, 0 below, -1 crossed
  const PeState* st = a.state + h;
  const bool all = st->all != 0;
  const uint32_t cut = st->cut_key;
  if (threadIdx.x <= rt) {
    int8_t k = 1;
    if (!all) {
      uint32_t kmin, kmax;
      tile_range(a, h, rt, threadIdx.x, kmin, kmax);
      k = (kmin <= cut && kmax >= cut) ? -1 : (kmin > cut ? 1 : 0);
    }
    kind[threadIdx.x] = k;
  }
  __syncthreads();
  const int r_end = min(rt * 128 + 128, a.nb);
  unsigned long long kept = 0;
  // one warp per row, lanes over the row's words
  for (int r = rt * 128 + (threadIdx.x >> 5); r < r_end; r += 8) {
    uint32_t* mrow = a.pe_mask + ((size_t)h * a.nb + r) * a.words;
    for (int w = threadIdx.x & 31; w < a.words; w += 32) {
      const int ct = w >> 2, c0 = w * 32;
      uint32_t word = 0u;
      if (ct <= rt) {
        if (kind[ct] < 0) continue;   // crossed: the mask sweep writes it
        const uint32_t upto = r >= c0 + 31 ? 0xFFFFFFFFu : (r < c0 ? 0u : (2u << (r - c0)) - 1u);   // c <= r
        word = kind[ct] > 0 ? upto : 0u;
        if (r >= c0 && r < c0 + 32) word |= 1u << (r - c0);   // the diagonal block
      }
      mrow[w] = word;
      kept += __popc(word);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) kept += __shfl_xor_sync(0xffffffffu, kept, o);
  if ((threadIdx.x & 31) == 0 && kept) atomicAdd(reinterpret_cast<unsigned long long*>(a.pe_count + h), kept);
  if (rt == 0 && threadIdx.x == 0) a.pe_cut[h] = all ? 0.f : __uint_as_float(cut);
}

// Ties, per row of head blockIdx.y (one warp per row, lanes over tiles): the
// counts of the tiles c <= r / 128 become running counts (ties in the tiles
// before each tile) and the row's total goes to tie_row.
__global__ void __launch_bounds__(1024) pe_tie_rows_kernel(PeArgs a) {
  const int h = blockIdx.y;
  if (a.route[h] != 1) return;
  const PeState* st = a.state + h;
  if (st->all || st->t_keep >= st->n_ties) return;
  const int r = blockIdx.x * 32 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= a.nb) return;
  uint32_t* t = a.tie_cnt + ((size_t)h * a.nb + r) * a.nt;
  const int ntile = r / 128 + 1;
  uint32_t carry = 0;
  for (int c0 = 0; c0 < ntile; c0 += 32) {
    const int ct = c0 + lane;
    const uint32_t v = ct < ntile ? t[ct] : 0u;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (ct < ntile) t[ct] = carry + incl - v;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) a.tie_row[(size_t)h * a.nb + r] = carry;
}

// Ties, per head: the row totals become exclusive offsets in flat order.
__global__ void __launch_bounds__(1024) pe_tie_scan_kernel(PeArgs a) {
  const int h = blockIdx.x;
  if (a.route[h] != 1) return;
  const PeState* st = a.state + h;
  if (st->all || st->t_keep >= st->n_ties) return;
  __shared__ unsigned long long part[1024];
  uint32_t* rows = a.tie_row + (size_t)h * a.nb;
  const int per = (a.nb + 1023) / 1024;
  const int lo = threadIdx.x * per, hi = min(a.nb, lo + per);
  unsigned long long s = 0;
  for (int r = lo; r < hi; ++r) s += rows[r];
  part[threadIdx.x] = s;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const unsigned long long v = threadIdx.x >= off ? part[threadIdx.x - off] : 0ull;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  // offsets fit 32 bits: a head has at most 2^25 causal blocks
  unsigned long long acc = threadIdx.x > 0 ? part[threadIdx.x - 1] : 0ull;
  for (int r = lo; r < hi; ++r) {
    const uint32_t v = rows[r];
    rows[r] = (uint32_t)acc;
    acc += v;
  }
}

template <int MODE>
cudaError_t launch_sweep(const CUtensorMap& mh, const CUtensorMap& ml, const PeArgs& a, int grid, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(pe_sweep_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  pe_sweep_kernel<MODE><<<grid, kThreads, kSmemBytes, st>>>(mh, ml, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pe(const void* q, const void* k, const Shape& s, char* ws, const WsLayout& L,
                      const IndexPtrs& ix, cudaStream_t st) {
  PeArgs a;
  a.nb = s.nb;
  a.nt = (s.nb + 127) / 128;
  a.words = s.words;
  a.group = s.group;
  a.h_q = s.h_q;
  a.gamma = s.gamma;
  a.route = ix.route;
  auto* qhi = reinterpret_cast<__nv_bfloat16*>(ws + L.qhi);
  auto* qlo = reinterpret_cast<__nv_bfloat16*>(ws + L.qlo);
  auto* khi = reinterpret_cast<__nv_bfloat16*>(ws + L.khi);
  auto* klo = reinterpret_cast<__nv_bfloat16*>(ws + L.klo);
  a.qhi = qhi;
  a.qlo = qlo;
  a.row_stat = reinterpret_cast<float2*>(ws + L.row_stat);
  a.tile_kr = reinterpret_cast<uint2*>(ws + L.tile_kr);
  a.tie_cnt = reinterpret_cast<uint32_t*>(ws + L.tie_cnt);
  a.tie_row = reinterpret_cast<uint32_t*>(ws + L.tie_row);
  a.hist = reinterpret_cast<PeHist*>(ws + L.hist);
  a.state = reinterpret_cast<PeState*>(ws + L.pe_state);
  a.pe_mask = ix.pe_mask;
  a.pe_count = ix.pe_count;
  a.pe_cut = ix.pe_cut;
  a.status = reinterpret_cast<int32_t*>(ws + L.status);
  const int32_t* kv_pe = reinterpret_cast<const int32_t*>(ws + L.kv_pe);

  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);

  cudaError_t e = cudaMemsetAsync(a.hist, 0, sizeof(PeHist) * s.h_q, st);
  if (e != cudaSuccess) return e;
  const int pool_grid = 4 * sms;
  if (s.fp32)
    pe_pool_kernel<float><<<pool_grid, kPoolThreads, 0, st>>>(static_cast<const float*>(q),
                                                              static_cast<const float*>(k), s.n, s.nb, a.nt * 128,
                                                              s.h_q, s.h_kv, s.scale_log2, ix.route, kv_pe, qhi, qlo,
                                                              khi, klo);
  else
    pe_pool_kernel<__nv_bfloat16><<<pool_grid, kPoolThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), s.n, s.nb, a.nt * 128, s.h_q,
        s.h_kv, s.scale_log2, ix.route, kv_pe, qhi, qlo, khi, klo);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  CUtensorMap mh, ml;
  if (!make_bf16_map(&mh, khi, a.nt * 128, s.h_kv, 128) || !make_bf16_map(&ml, klo, a.nt * 128, s.h_kv, 128))
    return cudaErrorInvalidValue;
  // one CTA per SM, at most one per stripe
  const int grid = (int)std::min<long long>(sms, (long long)s.h_q * a.nt);
  if ((e = launch_sweep<kStatsHist0>(mh, ml, a, grid, st)) != cudaSuccess) return e;
  pe_find_kernel<<<s.h_q, 1024, 0, st>>>(a, 0);
  if ((e = launch_sweep<kHist1>(mh, ml, a, grid, st)) != cudaSuccess) return e;
  pe_find_kernel<<<s.h_q, 1024, 0, st>>>(a, 1);
  if ((e = launch_sweep<kHist2>(mh, ml, a, grid, st)) != cudaSuccess) return e;
  pe_find_kernel<<<s.h_q, 1024, 0, st>>>(a, 2);
  if ((e = launch_sweep<kTies>(mh, ml, a, grid, st)) != cudaSuccess) return e;
  pe_tie_rows_kernel<<<dim3((s.nb + 31) / 32, s.h_q), 1024, 0, st>>>(a);
  pe_tie_scan_kernel<<<s.h_q, 1024, 0, st>>>(a);
  pe_mask_fill_kernel<<<dim3(a.nt, s.h_q), 256, 0, st>>>(a);
  if ((e = launch_sweep<kMask>(mh, ml, a, grid, st)) != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace crisp
