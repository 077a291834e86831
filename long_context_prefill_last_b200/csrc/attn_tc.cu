// Block-sparse causal attention on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in TMEM, operands staged by TMA), bf16 inputs,
// fp32 accumulation and softmax. CRISP summary page, Algorithm 1: exact
// softmax attention over exactly the selected keys; dev::tile_kind says which
// part of each 128x128 tile is selected, so VS diagonal bands are masked
// element-exactly inside a tile. The same kernel with every causal tile kept
// is the dense reference.
//
// One CTA per (query tile of 128 rows, query head); 6 warps:
//   warp 0      TMA producer: Q once, then K and V tiles through 2-stage rings
//   warp 1      TMEM allocation; one thread issues every tcgen05.mma
//   warps 2..5  softmax: one query row per thread (TMEM lane = row)
// TMEM columns: S double buffer [0,128) [128,256), O [256,384).
// Per kept tile k:  S[k%2] = Q K_k^T  ->  softmax -> P[k%2] (bf16, smem)
//                   O += P[k%2] V_k.   S(k+1) is computed while row k's
// softmax runs. O is rescaled lazily: only when a row's running maximum grows
// by more than 2^8, after the previous P V has landed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace crisp {
namespace {

constexpr int kThreads = 192;
constexpr int kStages = 2;
constexpr uint32_t kTileBytes = 128 * 128 * 2;   // one bf16 128x128 tile (two 64-column halves)
constexpr uint32_t kHalfBytes = 128 * 128;       // one half: 128 rows x 128 bytes
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_K = OFF_Q + kTileBytes;
constexpr uint32_t OFF_V = OFF_K + kStages * kTileBytes;
constexpr uint32_t OFF_P = OFF_V + kStages * kTileBytes;
constexpr uint32_t OFF_BAR = OFF_P + 2 * kTileBytes;
// barriers (8 bytes each)
enum {
  B_Q = 0,
  B_KFULL = 1,
  B_KEMPTY = B_KFULL + kStages,
  B_VFULL = B_KEMPTY + kStages,
  B_VEMPTY = B_VFULL + kStages,
  B_SFULL = B_VEMPTY + kStages,
  B_SEMPTY = B_SFULL + 2,
  B_PFULL = B_SEMPTY + 2,
  B_PVDONE = B_PFULL + 2,
  B_DRAIN = B_PVDONE + 2,
  B_COUNT = B_DRAIN + 1
};
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + 8 * B_COUNT;
constexpr uint32_t OFF_ABORT = OFF_TMEMPTR + 4;
constexpr uint32_t kSmemUsed = OFF_ABORT + 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;   // slack to align the base to 1024
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t TM_S0 = 0, TM_O = 256;
constexpr float kRescaleLog2 = 8.f;

struct TcArgs {
  int n, nb, words, group, h_q;
  float scale_log2;
  int dense;
  const int32_t* route;
  const uint32_t* vs_mask;
  const uint32_t* pe_mask;
  __nv_bfloat16* out;
  int32_t* status;
};

__device__ __forceinline__ uint32_t bar_addr(uint32_t base, int i) { return base + OFF_BAR + 8u * i; }

// Every lane waits; the warp proceeds only if all lanes saw the phase complete,
// so warp-collective tcgen05 loads and stores never run on a diverged warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int32_t* status,
                                          int where) {
  const bool ok = dev::mbar_wait(bar, parity, abort_flag, status, where);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = dev::smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + OFF_ABORT);
  uint32_t* tmem_ptr_smem = reinterpret_cast<uint32_t*>(sgen + OFF_TMEMPTR);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int lin = blockIdx.x;
  const int h = lin % a.h_q;
  const int I = (a.nb - 1) - lin / a.h_q;     // heaviest query tiles first
  const int g = h / a.group;
  const int route = a.dense ? 0 : a.route[h];
  const uint32_t* vmask = a.vs_mask + (size_t)h * 2 * a.words;
  const uint32_t* smask = vmask + a.words;
  const uint32_t* pe_row = a.pe_mask + ((size_t)h * a.nb + I) * a.words;
  const bool dense = a.dense != 0;

  if (threadIdx.x == 0) {
    // an earlier failure anywhere in the grid: this CTA does nothing
    *abort_flag = dev::load_volatile(a.status) != 0 ? 1 : 0;
    dev::mbar_init(bar_addr(sbase, B_Q), 1);
    for (int s = 0; s < kStages; ++s) {
      dev::mbar_init(bar_addr(sbase, B_KFULL + s), 1);
      dev::mbar_init(bar_addr(sbase, B_KEMPTY + s), 1);
      dev::mbar_init(bar_addr(sbase, B_VFULL + s), 1);
      dev::mbar_init(bar_addr(sbase, B_VEMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      dev::mbar_init(bar_addr(sbase, B_SFULL + b), 1);
      dev::mbar_init(bar_addr(sbase, B_SEMPTY + b), 128);
      dev::mbar_init(bar_addr(sbase, B_PFULL + b), 128);
      dev::mbar_init(bar_addr(sbase, B_PVDONE + b), 1);
    }
    dev::mbar_init(bar_addr(sbase, B_DRAIN), 1);
    dev::fence_mbar_init();
  }
  __syncthreads();
  if (*abort_flag) return;   // uniform: read after the barrier, before any TMEM is taken
  if (warp == 1) {
    dev::tmem_alloc(dev::smem_u32(tmem_ptr_smem), kTmemCols);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tmem = *tmem_ptr_smem;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      dev::prefetch_tmap(&tm_q);
      dev::prefetch_tmap(&tm_k);
      dev::prefetch_tmap(&tm_v);
      const uint32_t bq = bar_addr(sbase, B_Q);
      dev::mbar_arrive_expect_tx(bq, kTileBytes);
      dev::tma_load_3d(sbase + OFF_Q, &tm_q, bq, 0, I * 128, h);
      dev::tma_load_3d(sbase + OFF_Q + kHalfBytes, &tm_q, bq, 64, I * 128, h);
      int k = 0, prev_t = -1;
      int issued_k = 0, issued_v = 0;
      bool ok = true;
      for (int t = 0; t <= I + 1 && ok; ++t) {
        int kind = dev::kSkip;
        if (t <= I) kind = dev::tile_kind(route, vmask, smask, pe_row, dense, I, t);
        if (t <= I && kind == dev::kSkip) continue;
        if (t <= I) {   // K of tile k
          const int s = k % kStages;
          if (!dev::mbar_wait(bar_addr(sbase, B_KEMPTY + s), ((k / kStages) & 1) ^ 1, abort_flag, a.status, 1)) {
            ok = false;
            break;
          }
          const uint32_t bk = bar_addr(sbase, B_KFULL + s);
          dev::mbar_arrive_expect_tx(bk, kTileBytes);
          dev::tma_load_3d(sbase + OFF_K + s * kTileBytes, &tm_k, bk, 0, t * 128, g);
          dev::tma_load_3d(sbase + OFF_K + s * kTileBytes + kHalfBytes, &tm_k, bk, 64, t * 128, g);
          ++issued_k;
        }
        if (k >= 1) {   // V of tile k-1
          const int kv = k - 1, s = kv % kStages;
          if (!dev::mbar_wait(bar_addr(sbase, B_VEMPTY + s), ((kv / kStages) & 1) ^ 1, abort_flag, a.status, 2)) {
            ok = false;
            break;
          }
          const uint32_t bv = bar_addr(sbase, B_VFULL + s);
          dev::mbar_arrive_expect_tx(bv, kTileBytes);
          dev::tma_load_3d(sbase + OFF_V + s * kTileBytes, &tm_v, bv, 0, prev_t * 128, g);
          dev::tma_load_3d(sbase + OFF_V + s * kTileBytes + kHalfBytes, &tm_v, bv, 64, prev_t * 128, g);
          ++issued_v;
        }
        prev_t = t;
        ++k;
      }
      if (!ok) {
        // error path: let the copies already issued land before the CTA exits
        dev::mbar_drain(bq, 0);
        for (int s = 0; s < kStages; ++s) {
          const int last_k = issued_k - 1 - ((issued_k - 1 - s) % kStages + kStages) % kStages;
          if (issued_k > s && last_k >= 0) dev::mbar_drain(bar_addr(sbase, B_KFULL + s), (last_k / kStages) & 1);
          const int last_v = issued_v - 1 - ((issued_v - 1 - s) % kStages + kStages) % kStages;
          if (issued_v > s && last_v >= 0) dev::mbar_drain(bar_addr(sbase, B_VFULL + s), (last_v / kStages) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_qk = dev::umma_idesc_bf16(128, 128, false);
      const uint32_t idesc_pv = dev::umma_idesc_bf16(128, 128, true);
      bool ok = dev::mbar_wait(bar_addr(sbase, B_Q), 0, abort_flag, a.status, 3);
      dev::tc_fence_after();
      int k = 0;
      auto issue_pv = [&](int kp) -> bool {
        const int pb = kp & 1, s = kp % kStages;
        if (!dev::mbar_wait(bar_addr(sbase, B_PFULL + pb), (kp >> 1) & 1, abort_flag, a.status, 4)) return false;
        if (!dev::mbar_wait(bar_addr(sbase, B_VFULL + s), (kp / kStages) & 1, abort_flag, a.status, 5)) return false;
        dev::tc_fence_after();
        const uint32_t p_base = sbase + OFF_P + pb * kTileBytes;
        const uint32_t v_base = sbase + OFF_V + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ad = dev::smem_desc_sw128(p_base + (kk >> 2) * kHalfBytes + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = dev::smem_desc_sw128(v_base + kk * 2048, kHalfBytes, 1024);
          dev::umma_ss(tmem + TM_O, ad, bd, idesc_pv, (kp > 0 || kk > 0) ? 1u : 0u);
        }
        dev::umma_commit(bar_addr(sbase, B_PVDONE + pb));
        dev::umma_commit(bar_addr(sbase, B_VEMPTY + s));
        return true;
      };
      for (int t = 0; t <= I && ok; ++t) {
        const int kind = dev::tile_kind(route, vmask, smask, pe_row, dense, I, t);
        if (kind == dev::kSkip) continue;
        const int s = k % kStages, sb = k & 1;
        if (!dev::mbar_wait(bar_addr(sbase, B_KFULL + s), (k / kStages) & 1, abort_flag, a.status, 6)) {
          ok = false;
          break;
        }
        if (k >= 2 &&
            !dev::mbar_wait(bar_addr(sbase, B_SEMPTY + sb), ((k - 2) >> 1) & 1, abort_flag, a.status, 7)) {
          ok = false;
          break;
        }
        dev::tc_fence_after();
        const uint32_t k_base = sbase + OFF_K + s * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          const uint64_t ad = dev::smem_desc_sw128(sbase + OFF_Q + off, 16, 1024);
          const uint64_t bd = dev::smem_desc_sw128(k_base + off, 16, 1024);
          dev::umma_ss(tmem + TM_S0 + sb * 128, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        dev::umma_commit(bar_addr(sbase, B_SFULL + sb));
        dev::umma_commit(bar_addr(sbase, B_KEMPTY + s));
        if (k >= 1 && !issue_pv(k - 1)) {
          ok = false;
          break;
        }
        ++k;
      }
      if (ok && k >= 1) ok = issue_pv(k - 1);
      // all MMAs issued must complete before TMEM is released
      dev::umma_commit(bar_addr(sbase, B_DRAIN));
      dev::mbar_drain(bar_addr(sbase, B_DRAIN), 0);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int quarter = warp & 3;                 // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;            // query row inside the tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    float m_ref = -INFINITY, l = 0.f;
    int k = 0;
    bool ok = true;
    for (int t = 0; t <= I; ++t) {
      const int kind = dev::tile_kind(route, vmask, smask, pe_row, dense, I, t);
      if (kind == dev::kSkip) continue;
      const int sb = k & 1;
      if (!warp_wait(bar_addr(sbase, B_SFULL + sb), (k >> 1) & 1, abort_flag, a.status, 8)) {
        ok = false;
        break;
      }
      dev::tc_fence_after();
      float x[128];
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        dev::tmem_ld32(tmem + lane_base + TM_S0 + sb * 128 + c0, v);
        dev::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) x[c0 + j] = __uint_as_float(v[j]);
      }
      dev::tc_fence_before();
      dev::mbar_arrive(bar_addr(sbase, B_SEMPTY + sb));
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const bool keep = kind == dev::kFull || (kind == dev::kLower ? c <= r : c > r);
        x[c] = keep ? x[c] * a.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, x[c]);
      }
      const bool need = tmax > m_ref + kRescaleLog2;
      const float m_new = need ? tmax : m_ref;
      const float factor = need ? dev::ex2(m_ref - m_new) : 1.f;   // 0 when m_ref = -inf
      if (k > 0 && __any_sync(0xffffffffu, need)) {
        // O holds P V up to tile k-1: wait for it, then scale this warp's rows
        const int kp = k - 1;
        if (!warp_wait(bar_addr(sbase, B_PVDONE + (kp & 1)), (kp >> 1) & 1, abort_flag, a.status, 9)) {
          ok = false;
          break;
        }
        dev::tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t v[32];
          dev::tmem_ld32(tmem + lane_base + TM_O + c0, v);
          dev::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * factor);
          dev::tmem_st32(tmem + lane_base + TM_O + c0, v);
        }
        dev::tmem_wait_st();
        dev::tc_fence_before();
      }
      l *= factor;
      m_ref = m_new;
      const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
      // P = 2^(x - m), row sum, packed to bf16
      uint32_t pk[64];
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float p0 = dev::ex2(x[c] - m_use);
        const float p1 = dev::ex2(x[c + 1] - m_use);
        rs += p0 + p1;
        pk[c >> 1] = dev::pack_bf16x2(p0, p1);
      }
      l += rs;
      // the P buffer of tile k was read by P V of tile k-2
      if (k >= 2) {
        const int kp = k - 2;
        if (!warp_wait(bar_addr(sbase, B_PVDONE + (kp & 1)), (kp >> 1) & 1, abort_flag, a.status, 10)) {
          ok = false;
          break;
        }
      }
      uint8_t* prow = sgen + OFF_P + sb * kTileBytes + r * 128;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const int half = ch >> 3, cc = ch & 7;
        uint4 val = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        *reinterpret_cast<uint4*>(prow + half * kHalfBytes + ((cc ^ (r & 7)) << 4)) = val;
      }
      dev::fence_proxy_async_smem();
      dev::mbar_arrive(bar_addr(sbase, B_PFULL + sb));
      ++k;
    }
    // epilogue: O / l -> bf16 row of the output
    if (ok && k > 0) {
      const int kp = k - 1;
      ok = warp_wait(bar_addr(sbase, B_PVDONE + (kp & 1)), (kp >> 1) & 1, abort_flag, a.status, 11);
    }
    if (ok && k > 0) {
      dev::tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* orow = a.out + ((size_t)h * a.n + (size_t)I * 128 + r) * kHeadDim;
#pragma unroll
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t v[32];
        dev::tmem_ld32(tmem + lane_base + TM_O + c0, v);
        dev::tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          w[j] = dev::pack_bf16x2(__uint_as_float(v[2 * j]) * inv, __uint_as_float(v[2 * j + 1]) * inv);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(orow + c0 + 8 * j) = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
      }
    }
    dev::tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, void* out, const Shape& s,
                           const int32_t* route, const uint32_t* vs_mask, const uint32_t* pe_mask, bool dense,
                           int32_t* status, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_bf16_map(&mq, q, s.n, s.h_q, 128) || !make_bf16_map(&mk, k, s.n, s.h_kv, 128) || !make_bf16_map(&mv, v, s.n, s.h_kv, 128))
    return cudaErrorInvalidValue;
  TcArgs a;
  a.n = s.n;
  a.nb = s.nb;
  a.words = s.words;
  a.group = s.group;
  a.h_q = s.h_q;
  a.scale_log2 = s.scale_log2;
  a.dense = dense ? 1 : 0;
  a.route = route;
  a.vs_mask = vs_mask;
  a.pe_mask = pe_mask;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.status = status;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<<<s.nb * s.h_q, kThreads, kSmemBytes, st>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace crisp
