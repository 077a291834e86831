// Proxy map reduction on the tensor cores (CRISP summary page, Algorithm 2):
// the last 64 queries of every query head of a KV group are scored against
// every key by tcgen05.mma (bf16 in, fp32 in TMEM), and the softmax warps
// reduce each 128-key tile straight to the two partial sums the finaliser
// needs (keys c <= r and c > r of the row's block position r), so the proxy
// map itself never reaches memory. Each key tile is read from HBM once per
// CTA and used for two 128-row M tiles (four query heads).
//
// CTA = (KV head, pair of M tiles, contiguous range of 8-tile chunks);
// 12 warps: 0 TMA producer, 1 TMEM + MMA issuer, 2..3 idle, 4..11 softmax (one
// row per thread; warps 4..7 take M tile 0, 8..11 M tile 1). The first
// warpgroup gives registers to the softmax warpgroups (setmaxnreg 64 / 216 /
// 216), which hold a 128-column row and the chunk's 16 partial sums.
// TMEM: S[m][buf] at columns (2m + buf) * 128, 512 columns in all.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace crisp {
namespace {

constexpr int kThreads = 384;
constexpr int kRegsControl = 64;
constexpr int kRegsSoftmax = 216;
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= kThreads * 168, "register split exceeds the launch");
constexpr int kStages = 4;
// Pairs in every 8 whose exponentials use the FMA-pipe polynomial instead of
// MUFU. With the chunk partials in registers the softmax is led by MUFU, and
// moving one pair in eight to the polynomial measured 8% faster on the route
// stage at 512K tokens (two in eight: 4% faster, the extra FMA-pipe
// instructions then cost more than the MUFU time they free).
constexpr int kPolyPairsPer8 = 1;
constexpr uint32_t kTileBytes = 128 * 128 * 2;
constexpr uint32_t kHalfBytes = 128 * 128;
constexpr uint32_t OFF_Q = 0;                                // 2 M tiles
constexpr uint32_t OFF_K = OFF_Q + 2 * kTileBytes;
constexpr uint32_t OFF_BAR = OFF_K + kStages * kTileBytes;
enum {
  B_Q = 0,
  B_KFULL = 1,
  B_KEMPTY = B_KFULL + kStages,
  B_SFULL = B_KEMPTY + kStages,
  B_SEMPTY = B_SFULL + 2,
  B_DRAIN = B_SEMPTY + 2,
  B_COUNT = B_DRAIN + 1
};
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + 8 * B_COUNT;
constexpr uint32_t OFF_ABORT = OFF_TMEMPTR + 4;
constexpr uint32_t kSmemBytes = OFF_ABORT + 4 + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct PtcArgs {
  int n, nb, group, n_chunks, n_mp, n_split, chunks_per_cta;
  float scale_log2;
  float* part_lo;
  float* part_hi;
  float2* chunk_ml;
  int32_t* status;
};

__device__ __forceinline__ uint32_t bar_addr(uint32_t base, int i) { return base + OFF_BAR + 8u * i; }

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int32_t* status,
                                          int where) {
  const bool ok = dev::mbar_wait(bar, parity, abort_flag, status, where);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kThreads, 1)
proxy_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k, PtcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = dev::smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + OFF_ABORT);
  uint32_t* tmem_ptr_smem = reinterpret_cast<uint32_t*>(sgen + OFF_TMEMPTR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x % a.n_split;
  const int mp = (blockIdx.x / a.n_split) % a.n_mp;
  const int g = blockIdx.x / (a.n_split * a.n_mp);
  const int c_begin = split * a.chunks_per_cta;
  const int c_end = min(a.n_chunks, c_begin + a.chunks_per_cta);
  const int t_begin = c_begin * kChunkTiles;
  const int t_end = min(a.nb, c_end * kChunkTiles);
  const int n_tiles = max(0, t_end - t_begin);
  // query heads of this CTA: local head j in [0, 4) -> group head 4*mp + j
  const int head0 = g * a.group + 4 * mp;
  const int heads_here = min(4, a.group - 4 * mp);

  if (threadIdx.x == 0) {
    *abort_flag = (dev::load_volatile(a.status) != 0 || n_tiles == 0) ? 1 : 0;
    dev::mbar_init(bar_addr(sbase, B_Q), 1);
    for (int s = 0; s < kStages; ++s) {
      dev::mbar_init(bar_addr(sbase, B_KFULL + s), 1);
      dev::mbar_init(bar_addr(sbase, B_KEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      dev::mbar_init(bar_addr(sbase, B_SFULL + b), 1);
      dev::mbar_init(bar_addr(sbase, B_SEMPTY + b), 256);
    }
    dev::mbar_init(bar_addr(sbase, B_DRAIN), 1);
    dev::fence_mbar_init();
  }
  // rows of absent heads (group not a multiple of 4) are zero
  for (int j = heads_here; j < 4; ++j) {
    const int mt = j >> 1, rowoff = (j & 1) * 64;
    for (int half = 0; half < 2; ++half) {
      uint4* p = reinterpret_cast<uint4*>(sgen + OFF_Q + mt * kTileBytes + half * kHalfBytes + rowoff * 128);
      for (int e = threadIdx.x; e < 64 * 128 / 16; e += kThreads) p[e] = make_uint4(0, 0, 0, 0);
    }
  }
  dev::fence_proxy_async_smem();
  __syncthreads();
  if (*abort_flag) return;
  if (warp == 1) {
    dev::tmem_alloc(dev::smem_u32(tmem_ptr_smem), 512);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = *tmem_ptr_smem;
  const int n_mt = heads_here > 2 ? 2 : 1;   // M tiles holding at least one head

  if (warp < 4) dev::regs_release<kRegsControl>();
  if (warp == 0) {
    if (lane == 0) {
      dev::prefetch_tmap(&tm_q);
      dev::prefetch_tmap(&tm_k);
      const uint32_t bq = bar_addr(sbase, B_Q);
      dev::mbar_arrive_expect_tx(bq, (uint32_t)heads_here * 2u * 8192u);
      for (int j = 0; j < heads_here; ++j) {
        const int mt = j >> 1, rowoff = (j & 1) * 64;
        for (int half = 0; half < 2; ++half)
          dev::tma_load_3d(sbase + OFF_Q + mt * kTileBytes + half * kHalfBytes + rowoff * 128, &tm_q, bq, half * 64,
                           a.n - kProxyRows, head0 + j);
      }
      int issued = 0;
      bool ok = true;
      for (int k = 0; k < n_tiles; ++k) {
        const int s = k % kStages;
        if (!dev::mbar_wait(bar_addr(sbase, B_KEMPTY + s), ((k / kStages) & 1) ^ 1, abort_flag, a.status, 21)) {
          ok = false;
          break;
        }
        const uint32_t bk = bar_addr(sbase, B_KFULL + s);
        dev::mbar_arrive_expect_tx(bk, kTileBytes);
        const int t = t_begin + k;
        dev::tma_load_3d(sbase + OFF_K + s * kTileBytes, &tm_k, bk, 0, t * 128, g);
        dev::tma_load_3d(sbase + OFF_K + s * kTileBytes + kHalfBytes, &tm_k, bk, 64, t * 128, g);
        ++issued;
      }
      if (!ok) {
        dev::mbar_drain(bq, 0);
        for (int s = 0; s < kStages && s < issued; ++s) {
          const int last = issued - 1 - ((issued - 1 - s) % kStages);
          dev::mbar_drain(bar_addr(sbase, B_KFULL + s), (last / kStages) & 1);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = dev::umma_idesc_bf16(128, 128, false);
      bool ok = dev::mbar_wait(bar_addr(sbase, B_Q), 0, abort_flag, a.status, 22);
      dev::tc_fence_after();
      for (int k = 0; k < n_tiles && ok; ++k) {
        const int s = k % kStages, sb = k & 1;
        if (!dev::mbar_wait(bar_addr(sbase, B_KFULL + s), (k / kStages) & 1, abort_flag, a.status, 23)) break;
        if (k >= 2 && !dev::mbar_wait(bar_addr(sbase, B_SEMPTY + sb), ((k - 2) >> 1) & 1, abort_flag, a.status, 24))
          break;
        dev::tc_fence_after();
        const uint32_t k_base = sbase + OFF_K + s * kTileBytes;
        for (int mt = 0; mt < n_mt; ++mt) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            const uint64_t ad = dev::smem_desc_sw128(sbase + OFF_Q + mt * kTileBytes + off, 16, 1024);
            const uint64_t bd = dev::smem_desc_sw128(k_base + off, 16, 1024);
            dev::umma_ss(tmem + (uint32_t)(2 * mt + sb) * 128, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
        }
        dev::umma_commit(bar_addr(sbase, B_SFULL + sb));
        dev::umma_commit(bar_addr(sbase, B_KEMPTY + s));
      }
      dev::umma_commit(bar_addr(sbase, B_DRAIN));
      dev::mbar_drain(bar_addr(sbase, B_DRAIN), 0);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax warps
    dev::regs_acquire<kRegsSoftmax>();
    const int sw = warp - 4;                 // 0..7
    const int mt = sw >> 2;                  // M tile
    const int quarter = warp & 3;            // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;       // row inside the M tile
    const int j = mt * 2 + (r >> 6);         // local head
    const int ri = r & 63;                   // proxy row of that head
    const int rr = (a.n - kProxyRows + ri) - (a.nb - 1) * kBlock;   // position inside the last block
    const bool active = j < heads_here;
    const int I = a.nb - 1;
    const float sl2 = a.scale_log2;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const size_t row = (size_t)(head0 + (active ? j : 0)) * kProxyRows + ri;
    // this thread's partials of the current 8-tile chunk, in registers (slot u
    // of tile t_begin + 8c + u; every slot index below is a compile-time constant)
    float plo[kChunkTiles], phi[kChunkTiles];
#pragma unroll
    for (int w = 0; w < kChunkTiles; ++w) plo[w] = phi[w] = 0.f;
    int k = 0;
    bool ok = true;
    float m_run = -INFINITY, l_run = 0.f;
    for (int t = t_begin; t < t_end && ok; ++t) {
      const int u = (t - t_begin) % kChunkTiles;   // chunks start at t_begin (a multiple of 8)
      const int sb = k & 1;
      if (!warp_wait(bar_addr(sbase, B_SFULL + sb), (k >> 1) & 1, abort_flag, a.status, 25)) {
        ok = false;
        break;
      }
      dev::tc_fence_after();
      float x[128];
      if (mt < n_mt) {
        dev::tmem_ld128(tmem + lane_base + (uint32_t)(2 * mt + sb) * 128, x);
        dev::tmem_wait_ld();
      }
      dev::tc_fence_before();
      dev::mbar_arrive(bar_addr(sbase, B_SEMPTY + sb));
      ++k;
      if (active) {
        if (t == I) {   // causal: keys after the query
#pragma unroll
          for (int c = 64; c < 128; ++c) x[c] = c <= rr ? x[c] : -INFINITY;
        }
        float mx[4] = {x[0], x[1], x[2], x[3]};
#pragma unroll
        for (int c = 4; c < 128; c += 8) {
          mx[0] = dev::max3(mx[0], x[c], x[c + 1]);
          mx[1] = dev::max3(mx[1], x[c + 2], x[c + 3]);
          mx[2] = dev::max3(mx[2], x[c + 4], x[c + 5]);
          mx[3] = dev::max3(mx[3], x[c + 6], x[c + 7]);
        }
        const float tmax = fmaxf(dev::max3(mx[0], mx[1], mx[2]), mx[3]) * sl2;
        if (tmax > m_run + 8.f) {   // lazy rescale of this chunk's partials (slots >= u are still 0)
          const float f = dev::ex2(m_run - tmax);
          l_run *= f;
#pragma unroll
          for (int w = 0; w < kChunkTiles; ++w) {
            plo[w] *= f;
            phi[w] *= f;
          }
          m_run = tmax;
        }
        // exponentials with packed f32x2 arguments and sums; kPolyPairsPer8
        // pairs in eight on the FMA pipe. total = all columns, hi = columns c > rr
        // (only in the upper half since rr >= 64); lo = total - hi holds at
        // least the 64 lower columns, so the subtraction is well conditioned.
        const uint64_t scale2 = dev::f2_pack(sl2, sl2), negm2 = dev::f2_pack(-m_run, -m_run);
        uint64_t tot[4] = {0ull, 0ull, 0ull, 0ull}, hi2[2] = {0ull, 0ull};
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const int c = 2 * j;
          const uint64_t e2 = dev::f2_fma(dev::f2_pack(x[c], x[c + 1]), scale2, negm2);
          float p0, p1, e0, e1;
          dev::f2_unpack(e2, e0, e1);
          if ((j & 7) >= 8 - kPolyPairsPer8) {
            dev::exp2_poly3_x2(dev::f2_pack(fmaxf(e0, -125.f), fmaxf(e1, -125.f)), p0, p1);
            if (c >= 64) {
              p0 = x[c] == -INFINITY ? 0.f : p0;
              p1 = x[c + 1] == -INFINITY ? 0.f : p1;
            }
          } else {
            p0 = dev::ex2(e0);
            p1 = dev::ex2(e1);
          }
          tot[j & 3] = dev::f2_add(tot[j & 3], dev::f2_pack(p0, p1));
          if (c >= 64) hi2[j & 1] = dev::f2_add(hi2[j & 1], dev::f2_pack(c > rr ? p0 : 0.f, c + 1 > rr ? p1 : 0.f));
        }
        float t8[8], h4[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) dev::f2_unpack(tot[q], t8[2 * q], t8[2 * q + 1]);
        dev::f2_unpack(hi2[0], h4[0], h4[1]);
        dev::f2_unpack(hi2[1], h4[2], h4[3]);
        const float stot = ((t8[0] + t8[1]) + (t8[2] + t8[3])) + ((t8[4] + t8[5]) + (t8[6] + t8[7]));
        const float shi = (h4[0] + h4[1]) + (h4[2] + h4[3]);
        const float slo = stot - shi;
#pragma unroll
        for (int w = 0; w < kChunkTiles; ++w) {
          plo[w] = w == u ? slo : plo[w];
          phi[w] = w == u ? shi : phi[w];
        }
        l_run += slo + shi;
        if (u == kChunkTiles - 1 || t == t_end - 1) {
          const int c = t / kChunkTiles;
          float* glo = a.part_lo + row * a.nb + (size_t)c * kChunkTiles;
          float* ghi = a.part_hi + row * a.nb + (size_t)c * kChunkTiles;
          if (u == kChunkTiles - 1 && (a.nb & 3) == 0) {   // a whole chunk, 16-byte aligned rows
            reinterpret_cast<float4*>(glo)[0] = make_float4(plo[0], plo[1], plo[2], plo[3]);
            reinterpret_cast<float4*>(glo)[1] = make_float4(plo[4], plo[5], plo[6], plo[7]);
            reinterpret_cast<float4*>(ghi)[0] = make_float4(phi[0], phi[1], phi[2], phi[3]);
            reinterpret_cast<float4*>(ghi)[1] = make_float4(phi[4], phi[5], phi[6], phi[7]);
          } else {
#pragma unroll
            for (int w = 0; w < kChunkTiles; ++w)
              if (w <= u) {
                glo[w] = plo[w];
                ghi[w] = phi[w];
              }
          }
          a.chunk_ml[row * a.n_chunks + c] = make_float2(m_run, l_run);
          m_run = -INFINITY;
          l_run = 0.f;
#pragma unroll
          for (int w = 0; w < kChunkTiles; ++w) plo[w] = phi[w] = 0.f;
        }
      }
    }
    dev::tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_proxy_tc(const void* q, const void* k, const Shape& s, char* ws, const WsLayout& L,
                            cudaStream_t st) {
  CUtensorMap mq, mk;
  if (!make_bf16_map(&mq, q, s.n, s.h_q, kProxyRows) || !make_bf16_map(&mk, k, s.n, s.h_kv, 128)) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  PtcArgs a;
  a.n = s.n;
  a.nb = s.nb;
  a.group = s.group;
  a.n_chunks = s.n_chunks;
  a.n_mp = (s.group + 3) / 4;
  const int units = s.h_kv * a.n_mp;
  a.n_split = std::max(1, std::min(s.n_chunks, sms / units));
  a.chunks_per_cta = (s.n_chunks + a.n_split - 1) / a.n_split;
  a.n_split = (s.n_chunks + a.chunks_per_cta - 1) / a.chunks_per_cta;
  a.scale_log2 = s.scale_log2;
  a.part_lo = reinterpret_cast<float*>(ws + L.part_lo);
  a.part_hi = reinterpret_cast<float*>(ws + L.part_hi);
  a.chunk_ml = reinterpret_cast<float2*>(ws + L.chunk_ml);
  a.status = reinterpret_cast<int32_t*>(ws + L.status);
  cudaError_t e = cudaFuncSetAttribute(proxy_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  proxy_tc_kernel<<<units * a.n_split, kThreads, kSmemBytes, st>>>(mq, mk, a);
  return cudaGetLastError();
}

}  // namespace crisp
