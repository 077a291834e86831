// Block-sparse causal attention on the 5th-generation tensor cores
// (tcgen05.mma, accumulators in TMEM, operands staged by TMA), bf16 inputs,
// fp32 accumulation and softmax. CRISP summary page, Algorithm 1: exact
// softmax attention over exactly the selected keys; dev::tile_kind says which
// part of each 128x128 tile is selected, so VS diagonal bands are masked
// element-exactly inside a tile. The same kernel with every causal tile kept
// is the dense reference.
//
// One CTA per (pair of adjacent 128-row query tiles A = I, B = I-1, query
// head); the K/V tiles of the union of their schedules stream once through
// shared memory and serve both. The grid runs KV group by KV group (heaviest
// pairs first within a group): the CTAs resident at any time then read one
// or two KV heads' keys and values, which stay in L2 between them (at
// 512K tokens this cut DRAM reads from 5.0 TB to 1.9 TB per launch). 12 warps in three warpgroups:
//   warp 0       TMA producer: Q_A, Q_B once, then K (3-stage ring) and V (2-stage ring)
//   warp 1       TMEM allocation; walks the schedule warp-wide (descriptors stay
//                warp-uniform) and one elected lane issues every tcgen05.mma
//   warps 2, 3   idle (they complete the first warpgroup)
//   warps 4..7   softmax of tile A, warps 8..11 softmax of tile B (row = TMEM lane)
// The first warpgroup gives registers to the softmax warpgroups
// (setmaxnreg: 64 / 216 / 216 per thread; 128*64 + 256*216 <= 384*168, the
// launch allocation), so a softmax thread holds its whole 128-column S row and
// reads TMEM once per tile. The softmax is issue-bound more than MUFU-bound
// (MUFU runs under half its rate), so it uses packed f32x2 arithmetic and a
// three-input max, and every exponential stays on MUFU: moving one pair in
// eight to an FMA-pipe polynomial measured 6% slower at 512K tokens.
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).
// P (bf16) is written back over the first 64 columns of S and read by the
// P.V MMA straight from TMEM. MMA issue order per kept tile u:
//     S_B(u) = Q_B K_u^T,  O_A += P_A(u) V_u,  S_A(u+1) = Q_A K_{u+1}^T,  O_B += P_B(u) V_u
// so each softmax runs while the tensor pipe does two MMAs of the other tile.
// Because MMAs complete in issue order, S_X(u) landing means O_X already holds
// P_X(u-1) V: the softmax may rescale O_X without another wait. Rescaling is
// lazy: only when a row's running maximum grows by more than 2^8.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "internal.h"
#include "ptx.cuh"
#include "tmap.h"

namespace crisp {
namespace {

constexpr int kThreads = 384;
constexpr int kRegsControl = 64;    // producer / MMA warpgroup after the split
constexpr int kRegsSoftmax = 216;   // each softmax warpgroup after the split
static_assert(128 * kRegsControl + 256 * kRegsSoftmax <= kThreads * 168, "register split exceeds the launch");
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr uint32_t kTileBytes = 128 * 128 * 2;   // one bf16 128x128 tile (two 64-column halves)
constexpr uint32_t kHalfBytes = 128 * 128;       // one half: 128 rows x 128 bytes
constexpr uint32_t OFF_QA = 0;
constexpr uint32_t OFF_QB = kTileBytes;
constexpr uint32_t OFF_K = 2 * kTileBytes;
constexpr uint32_t OFF_V = OFF_K + kKStages * kTileBytes;
constexpr uint32_t OFF_BAR = OFF_V + kVStages * kTileBytes;
enum {
  B_Q = 0,
  B_KFULL = 1,
  B_KEMPTY = B_KFULL + kKStages,
  B_VFULL = B_KEMPTY + kKStages,
  B_VEMPTY = B_VFULL + kVStages,
  B_SFULL = B_VEMPTY + kVStages,   // [2]: S_X landed
  B_PFULL = B_SFULL + 2,           // [2]: P_X written (128 arrivals)
  B_DONE = B_PFULL + 2,            // [2]: last P_X V landed
  B_DRAIN = B_DONE + 2,
  B_COUNT = B_DRAIN + 1
};
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + 8 * B_COUNT;
constexpr uint32_t OFF_ABORT = OFF_TMEMPTR + 4;
constexpr uint32_t kSmemBytes = OFF_ABORT + 4 + 1024;   // + slack to align the base to 1024
static_assert(kSmemBytes <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.f;

struct TcArgs {
  int n, nb, words, group, h_q, n_pairs;
  float scale_log2;
  int dense;
  const int32_t* route;
  const uint32_t* vs_mask;
  const uint32_t* pe_mask;
  __nv_bfloat16* out;
  int32_t* status;
};

__device__ __forceinline__ uint32_t bar_addr(uint32_t base, int i) { return base + OFF_BAR + 8u * i; }

__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int32_t* status,
                                          int where) {
  const bool ok = dev::mbar_wait(bar, parity, abort_flag, status, where);
  return __all_sync(0xffffffffu, ok);
}

// The two query tiles' schedules (same head, tiles IA and IB = IA - 1).
struct Sched {
  int IA, IB, route;
  bool dense;
  const uint32_t *vmask, *smask, *peA, *peB;
  __device__ int kindA(int t) const { return dev::tile_kind(route, vmask, smask, peA, dense, IA, t); }
  __device__ int kindB(int t) const {
    return (IB >= 0 && t <= IB) ? dev::tile_kind(route, vmask, smask, peB, dense, IB, t) : (int)dev::kSkip;
  }
  // next tile >= t needed by A or B; returns false at the end
  __device__ bool next(int& t, int& ka, int& kb) const {
    for (; t <= IA; ++t) {
      ka = kindA(t);
      kb = kindB(t);
      if (ka != dev::kSkip || kb != dev::kSkip) return true;
    }
    return false;
  }
};

// Kept columns of a row: all (full tile), c <= r (lower) or c > r (upper).
__device__ __forceinline__ void mask_row(float (&s)[128], int kind, int r) {
  if (kind == dev::kLower) {
#pragma unroll
    for (int c = 0; c < 128; ++c) s[c] = c <= r ? s[c] : -INFINITY;
  } else if (kind == dev::kUpper) {
#pragma unroll
    for (int c = 0; c < 128; ++c) s[c] = c > r ? s[c] : -INFINITY;
  }
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
  // KV group by KV group (CTAs that run together share K/V through L2),
  // heaviest pairs first within a group, the group's query heads adjacent
  const int per_group = a.n_pairs * a.group;
  const int g_major = blockIdx.x / per_group;
  const int rem = blockIdx.x - g_major * per_group;
  const int pair = rem / a.group;
  const int h = g_major * a.group + rem % a.group;
  Sched sc;
  sc.IA = (a.nb - 1) - 2 * pair;
  sc.IB = sc.IA - 1;
  sc.dense = a.dense != 0;
  sc.route = sc.dense ? 0 : a.route[h];
  sc.vmask = a.vs_mask + (size_t)h * 2 * a.words;
  sc.smask = sc.vmask + a.words;
  sc.peA = a.pe_mask + ((size_t)h * a.nb + sc.IA) * a.words;
  sc.peB = a.pe_mask + ((size_t)h * a.nb + (sc.IB >= 0 ? sc.IB : 0)) * a.words;
  const int g = h / a.group;
  const bool hasB = sc.IB >= 0;

  if (threadIdx.x == 0) {
    *abort_flag = dev::load_volatile(a.status) != 0 ? 1 : 0;   // an earlier failure: do nothing
    dev::mbar_init(bar_addr(sbase, B_Q), 1);
    for (int s = 0; s < kKStages; ++s) {
      dev::mbar_init(bar_addr(sbase, B_KFULL + s), 1);
      dev::mbar_init(bar_addr(sbase, B_KEMPTY + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      dev::mbar_init(bar_addr(sbase, B_VFULL + s), 1);
      dev::mbar_init(bar_addr(sbase, B_VEMPTY + s), 1);
    }
    for (int x = 0; x < 2; ++x) {
      dev::mbar_init(bar_addr(sbase, B_SFULL + x), 1);
      dev::mbar_init(bar_addr(sbase, B_PFULL + x), 128);
      dev::mbar_init(bar_addr(sbase, B_DONE + x), 1);
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

  if (warp < 4) dev::regs_release<kRegsControl>();
  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      dev::prefetch_tmap(&tm_q);
      dev::prefetch_tmap(&tm_k);
      dev::prefetch_tmap(&tm_v);
      const uint32_t bq = bar_addr(sbase, B_Q);
      dev::mbar_arrive_expect_tx(bq, hasB ? 2 * kTileBytes : kTileBytes);
      dev::tma_load_3d(sbase + OFF_QA, &tm_q, bq, 0, sc.IA * 128, h);
      dev::tma_load_3d(sbase + OFF_QA + kHalfBytes, &tm_q, bq, 64, sc.IA * 128, h);
      if (hasB) {
        dev::tma_load_3d(sbase + OFF_QB, &tm_q, bq, 0, sc.IB * 128, h);
        dev::tma_load_3d(sbase + OFF_QB + kHalfBytes, &tm_q, bq, 64, sc.IB * 128, h);
      }
      int u = 0, t = 0, ka = 0, kb = 0, prev_t = -1;
      int issued_k = 0, issued_v = 0;
      bool ok = true, more = true;
      while (ok && (more || prev_t >= 0)) {
        more = more && sc.next(t, ka, kb);
        if (more) {   // K of tile u
          const int s = u % kKStages;
          if (!dev::mbar_wait(bar_addr(sbase, B_KEMPTY + s), ((u / kKStages) & 1) ^ 1, abort_flag, a.status, 1)) {
            ok = false;
            break;
          }
          const uint32_t bk = bar_addr(sbase, B_KFULL + s);
          dev::mbar_arrive_expect_tx(bk, kTileBytes);
          dev::tma_load_3d(sbase + OFF_K + s * kTileBytes, &tm_k, bk, 0, t * 128, g);
          dev::tma_load_3d(sbase + OFF_K + s * kTileBytes + kHalfBytes, &tm_k, bk, 64, t * 128, g);
          ++issued_k;
        }
        if (prev_t >= 0) {   // V of tile u-1
          const int uv = u - 1, s = uv % kVStages;
          if (!dev::mbar_wait(bar_addr(sbase, B_VEMPTY + s), ((uv / kVStages) & 1) ^ 1, abort_flag, a.status, 2)) {
            ok = false;
            break;
          }
          const uint32_t bv = bar_addr(sbase, B_VFULL + s);
          dev::mbar_arrive_expect_tx(bv, kTileBytes);
          dev::tma_load_3d(sbase + OFF_V + s * kTileBytes, &tm_v, bv, 0, prev_t * 128, g);
          dev::tma_load_3d(sbase + OFF_V + s * kTileBytes + kHalfBytes, &tm_v, bv, 64, prev_t * 128, g);
          ++issued_v;
        }
        prev_t = more ? t : -1;
        if (more) {
          ++t;
          ++u;
        }
      }
      if (!ok) {
        // error path: let the copies already issued land before the CTA exits
        dev::mbar_drain(bq, 0);
        for (int s = 0; s < kKStages && s < issued_k; ++s) {
          const int last = issued_k - 1 - ((issued_k - 1 - s) % kKStages);
          dev::mbar_drain(bar_addr(sbase, B_KFULL + s), (last / kKStages) & 1);
        }
        for (int s = 0; s < kVStages && s < issued_v; ++s) {
          const int last = issued_v - 1 - ((issued_v - 1 - s) % kVStages);
          dev::mbar_drain(bar_addr(sbase, B_VFULL + s), (last / kVStages) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // The whole warp walks the schedule and waits (the descriptors stay
    // warp-uniform); one elected lane issues every tcgen05.mma and commit.
    const uint32_t idesc_qk = dev::umma_idesc_bf16(128, 128, false);
    const uint32_t idesc_pv = dev::umma_idesc_bf16(128, 128, true);
    // descriptors of the first K stage and V stage; stages and Q_B are
    // whole tiles further (kTileBytes / 16 in the start-address field)
    const uint64_t QD0 = dev::smem_desc_sw128(sbase + OFF_QA, 16, 1024);
    const uint64_t KD0 = dev::smem_desc_sw128(sbase + OFF_K, 16, 1024);
    const uint64_t VD0 = dev::smem_desc_sw128(sbase + OFF_V, kHalfBytes, 1024);
    int kx0 = 0, kx1 = 0;   // P.V issued per tile
    auto qk = [&](int x, int u) {
      dev::umma_ss8_w(tmem + (uint32_t)x * 128u, QD0 + (uint64_t)(x * (kTileBytes >> 4)),
                      KD0 + (uint64_t)((u % kKStages) * (kTileBytes >> 4)), idesc_qk, 0u);
      dev::umma_commit_w(bar_addr(sbase, B_SFULL + x));
    };
    auto pv = [&](int x, int u) -> bool {
      const int kx = x == 0 ? kx0 : kx1;
      if (!warp_wait(bar_addr(sbase, B_PFULL + x), kx & 1, abort_flag, a.status, 4 + x)) return false;
      dev::tc_fence_after();
      dev::umma_ts8_w(tmem + 256u + (uint32_t)x * 128u, tmem + (uint32_t)x * 128u,
                      VD0 + (uint64_t)((u % kVStages) * (kTileBytes >> 4)), idesc_pv, kx > 0 ? 1u : 0u);
      if (x == 0) ++kx0; else ++kx1;
      return true;
    };
    bool ok = warp_wait(bar_addr(sbase, B_Q), 0, abort_flag, a.status, 3);
    int t = 0, ka = 0, kb = 0;
    bool have = ok && sc.next(t, ka, kb);
    if (have) {
      ok = warp_wait(bar_addr(sbase, B_KFULL + 0), 0, abort_flag, a.status, 6);
      dev::tc_fence_after();
      if (ok && ka != dev::kSkip) qk(0, 0);
    }
    int u = 0;
    while (ok && have) {
      if (kb != dev::kSkip) qk(1, u);
      dev::umma_commit_w(bar_addr(sbase, B_KEMPTY + u % kKStages));
      // find the tile after u while the tensor pipe computes S_B(u) and the
      // softmax of A works on P_A(u)
      int t2 = t + 1, ka2 = 0, kb2 = 0;
      const bool have2 = sc.next(t2, ka2, kb2);
      if (!warp_wait(bar_addr(sbase, B_VFULL + u % kVStages), (u / kVStages) & 1, abort_flag, a.status, 7)) {
        ok = false;
        break;
      }
      dev::tc_fence_after();
      if (ka != dev::kSkip && !pv(0, u)) {
        ok = false;
        break;
      }
      if (have2) {
        if (!warp_wait(bar_addr(sbase, B_KFULL + (u + 1) % kKStages), ((u + 1) / kKStages) & 1, abort_flag,
                       a.status, 8)) {
          ok = false;
          break;
        }
        dev::tc_fence_after();
        if (ka2 != dev::kSkip) qk(0, u + 1);
      }
      if (kb != dev::kSkip && !pv(1, u)) {
        ok = false;
        break;
      }
      dev::umma_commit_w(bar_addr(sbase, B_VEMPTY + u % kVStages));
      t = t2;
      ka = ka2;
      kb = kb2;
      have = have2;
      ++u;
    }
    if (ok) {
      dev::umma_commit_w(bar_addr(sbase, B_DONE + 0));
      dev::umma_commit_w(bar_addr(sbase, B_DONE + 1));
    }
    // every MMA issued must complete before TMEM is released
    dev::umma_commit_w(bar_addr(sbase, B_DRAIN));
    dev::mbar_drain(bar_addr(sbase, B_DRAIN), 0);
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax warps
    dev::regs_acquire<kRegsSoftmax>();
    const int x = (warp - 4) >> 2;                // 0: tile A, 1: tile B
    const int quarter = warp & 3;                 // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;            // query row inside the tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_col = tmem + lane_base + (uint32_t)x * 128;
    const uint32_t o_col = tmem + lane_base + 256u + (uint32_t)x * 128;
    const int I = x == 0 ? sc.IA : sc.IB;
    if (I >= 0) {
      const float sl2 = a.scale_log2;
      float m_ref = -INFINITY, l = 0.f;
      int k = 0;
      bool ok = true;
      for (int t = 0; t <= I; ++t) {
        const int kind = x == 0 ? sc.kindA(t) : sc.kindB(t);
        if (kind == dev::kSkip) continue;
        if (!warp_wait(bar_addr(sbase, B_SFULL + x), k & 1, abort_flag, a.status, 10 + x)) {
          ok = false;
          break;
        }
        dev::tc_fence_after();
        float s[128];
        dev::tmem_ld128(s_col, s);
        dev::tmem_wait_ld();
        mask_row(s, kind, r);
        float mx[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
        for (int c = 4; c < 128; c += 8) {
          mx[0] = dev::max3(mx[0], s[c], s[c + 1]);
          mx[1] = dev::max3(mx[1], s[c + 2], s[c + 3]);
          mx[2] = dev::max3(mx[2], s[c + 4], s[c + 5]);
          mx[3] = dev::max3(mx[3], s[c + 6], s[c + 7]);
        }
        const float tmax = fmaxf(dev::max3(mx[0], mx[1], mx[2]), mx[3]) * sl2;
        const bool need = tmax > m_ref + kRescaleLog2;
        const float factor = need ? dev::ex2(m_ref - tmax) : 1.f;   // 0 when m_ref = -inf
        if (k > 0 && __any_sync(0xffffffffu, need)) {
          // O holds P V of every earlier tile (it completed before S landed)
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t v[32];
            dev::tmem_ld32(o_col + c0, v);
            dev::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * factor);
            dev::tmem_st32(o_col + c0, v);
          }
        }
        if (need) {
          l *= factor;
          m_ref = tmax;
        }
        const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
        // P = 2^(s*scale - m); chunk c0 of P (bf16 pairs) goes to S columns
        // [c0/2, c0/2 + 16), already consumed. Arguments and row sums use
        // packed f32x2 arithmetic, exponentials MUFU. Masked entries (-inf)
        // give exactly 0.
        const uint64_t scale2 = dev::f2_pack(sl2, sl2), negm2 = dev::f2_pack(neg_m, neg_m);
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int c = c0 + 2 * j;
            const uint64_t x2 = dev::f2_fma(dev::f2_pack(s[c], s[c + 1]), scale2, negm2);
            float x0, x1;
            dev::f2_unpack(x2, x0, x1);
            const float p0 = dev::ex2(x0), p1 = dev::ex2(x1);
            acc[j & 3] = dev::f2_add(acc[j & 3], dev::f2_pack(p0, p1));
            pk[j] = dev::pack_bf16x2(p0, p1);
          }
          dev::tmem_st16(s_col + (c0 >> 1), pk);
        }
        float sum[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) dev::f2_unpack(acc[j], sum[2 * j], sum[2 * j + 1]);
        dev::tmem_wait_st();
        dev::tc_fence_before();
        dev::mbar_arrive(bar_addr(sbase, B_PFULL + x));
        l += ((sum[0] + sum[1]) + (sum[2] + sum[3])) + ((sum[4] + sum[5]) + (sum[6] + sum[7]));
        ++k;
      }
      // epilogue: O / l -> bf16 row of the output
      if (ok && k > 0) ok = warp_wait(bar_addr(sbase, B_DONE + x), 0, abort_flag, a.status, 12 + x);
      if (ok && k > 0) {
        dev::tc_fence_after();
        const float inv = 1.f / l;
        __nv_bfloat16* orow = a.out + ((size_t)h * a.n + (size_t)I * 128 + r) * kHeadDim;
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t v[32];
          dev::tmem_ld32(o_col + c0, v);
          dev::tmem_wait_ld();
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            w[j] = dev::pack_bf16x2(__uint_as_float(v[2 * j]) * inv, __uint_as_float(v[2 * j + 1]) * inv);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(orow + c0 + 8 * j) =
                make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        }
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
  if (!make_bf16_map(&mq, q, s.n, s.h_q, 128) || !make_bf16_map(&mk, k, s.n, s.h_kv, 128) ||
      !make_bf16_map(&mv, v, s.n, s.h_kv, 128))
    return cudaErrorInvalidValue;
  TcArgs a;
  a.n = s.n;
  a.nb = s.nb;
  a.words = s.words;
  a.group = s.group;
  a.h_q = s.h_q;
  a.n_pairs = (s.nb + 1) / 2;
  a.scale_log2 = s.scale_log2;
  a.dense = dense ? 1 : 0;
  a.route = route;
  a.vs_mask = vs_mask;
  a.pe_mask = pe_mask;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.status = status;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  attn_tc_kernel<<<a.n_pairs * s.h_q, kThreads, kSmemBytes, st>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace crisp
