// Internal declarations shared by the CRISP CUDA sources (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "crisp.h"

namespace crisp {

constexpr int kBlock = 128;       // B: keys per block, queries per tile
constexpr int kHeadDim = 128;     // d
constexpr int kProxyRows = 64;    // |Q-hat|
constexpr int kChunkTiles = 8;    // key tiles per proxy chunk (one (m, l) pair per chunk)

// Device status word layout (int32 x 8 at the start of the workspace).
enum StatusSlot { kStatusCode = 0, kStatusInfo = 1, kStatusInfo2 = 2 };

// Byte offsets of every region of the workspace (all 256-byte aligned).
struct WsLayout {
  size_t status;      // int32[8]
  size_t part_lo;     // f32 [h_q][last_q][N_b]  proxy partial: keys c <= r of the tile
  size_t part_hi;     // f32 [h_q][last_q][N_b]  proxy partial: keys c >  r of the tile
  size_t chunk_ml;    // f32x2 [h_q][last_q][n_chunks] (log2-domain max, sum) per chunk
  size_t chunk_w;     // f32 [h_q][last_q][n_chunks] weight of each chunk's partials
  size_t tile_a;      // f32 [h_q][N_b]  sum over rows of weighted part_lo
  size_t tile_b;      // f32 [h_q][N_b]  sum over rows of weighted part_hi
  size_t qhi, qlo;    // bf16 [h_q][N_b][d]          pooled Q * scale_log2, hi and lo parts
  size_t khi, klo;    // bf16 [h_kv][nt*128][d]      pooled K, hi and lo parts (rows past N_b zero)
  size_t row_stat;    // f32x2 [h_q][N_b]            pooled-map row (maximum, 1 / (sum * N_b)), log2 domain
  size_t tile_kr;     // u32x2 [h_q][nt][nt][4]      (min, max) key of each 32-row quarter of a 128x128 map tile
  size_t tie_cnt;     // u32 [h_q][N_b][nt]          entries equal to the cut per (row, tile), then before each tile
  size_t tie_row;     // u32 [h_q][N_b]              entries equal to the cut per row, then offsets
  size_t hist;        // per head: PeHist
  size_t pe_state;    // per head: PeState
  size_t kv_pe;       // int32 [h_kv]: 1 if any query head of the group routes PE
  // internal index (used by crisp_prefill / crisp_route)
  size_t route, c_struct, p_v, p_s, mu, vs_mask, v_idx, s_idx, nv, ns, pe_mask, pe_count, pe_cut;
  size_t total;
};

struct Shape {
  int n, h_q, h_kv, d, group, nb, words, n_chunks, last_q;
  int nt;                // 128-block tiles of the pooled map per side: ceil(N_b / 128)
  bool fp32;
  float sm_scale;     // natural-log domain scale
  float scale_log2;   // sm_scale * log2(e)
  float tau, alpha, gamma;
  int force_route;
};

WsLayout ws_layout(const Shape& s);

// Validate a cfg and derive its Shape (the checks every entry point runs).
crisp_status shape_from_cfg(const crisp_cfg* c, Shape* s);

// Device pointers for one index set.
struct IndexPtrs {
  int32_t* route;
  float* c_struct;
  float* p_v;
  float* p_s;
  float* mu;
  uint32_t* vs_mask;
  int32_t* v_idx;
  int32_t* s_idx;
  int32_t* nv;
  int32_t* ns;
  uint32_t* pe_mask;
  int64_t* pe_count;
  float* pe_cut;
};

// Query heads of one call (after batch folding).
constexpr int kMaxHeads = 1024;

// Per-head histogram for the PE gamma cut: three radix levels of the fp32 bit pattern.
constexpr int kHistL0 = 4096;   // bits 31..20
constexpr int kHistL1 = 4096;   // bits 19..8
constexpr int kHistL2 = 256;    // bits 7..0
// Mass is kept in fixed point, units of 2^-62 (every entry of the normalised
// map is at most 1/4, the total is 1): integer sums are exact in any order,
// so the cut does not depend on the order of the atomics.
constexpr double kMassUnit = 1.0 / 4611686018427387904.0;   // 2^-62
struct PeHist {
  unsigned long long count[kHistL0];
  unsigned long long mass[kHistL0];
};
struct PeState {
  double s_above;       // mass strictly above the current key prefix
  double total;         // total mass (level 0)
  uint32_t prefix;      // key bits fixed so far
  uint32_t level;       // next level to histogram
  uint32_t cut_key;     // final cut value (fp32 bits)
  uint32_t all;         // 1: keep every causal block
  unsigned long long n_ties;   // entries equal to the cut value
  unsigned long long t_keep;   // ties to keep (by ascending flat index)
  unsigned long long pad[2];
};

// ---- launchers (each enqueues on `st`; return cudaGetLastError()) ----
cudaError_t launch_proxy_simt(const void* q, const void* k, const Shape& s, char* ws, const WsLayout& L,
                              cudaStream_t st);
cudaError_t launch_proxy_tc(const void* q, const void* k, const Shape& s, char* ws, const WsLayout& L,
                            cudaStream_t st);
cudaError_t launch_finalize(const Shape& s, char* ws, const WsLayout& L, const IndexPtrs& ix, cudaStream_t st);
cudaError_t launch_vs_select(const Shape& s, char* ws, const WsLayout& L, const IndexPtrs& ix, cudaStream_t st);
cudaError_t launch_pe(const void* q, const void* k, const Shape& s, char* ws, const WsLayout& L,
                      const IndexPtrs& ix, cudaStream_t st);
cudaError_t launch_attn_simt(const void* q, const void* k, const void* v, void* out, const Shape& s,
                             const int32_t* route, const uint32_t* vs_mask, const uint32_t* pe_mask, bool dense,
                             int32_t* status, cudaStream_t st);
cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, void* out, const Shape& s,
                           const int32_t* route, const uint32_t* vs_mask, const uint32_t* pe_mask, bool dense,
                           int32_t* status, cudaStream_t st);

}  // namespace crisp
