// C ABI of the CRISP sparse-prefill library: argument validation, workspace
// layout and the order of kernel launches. Nothing here synchronises with the
// device except crisp_device_status.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "crisp.h"
#include "internal.h"

namespace crisp {

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

WsLayout ws_layout(const Shape& s) {
  WsLayout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t hq = s.h_q, hkv = s.h_kv, nb = s.nb, rows = (size_t)s.h_q * s.last_q;
  L.status = take(256);
  L.part_lo = take(rows * nb * 4);
  L.part_hi = take(rows * nb * 4);
  L.chunk_ml = take(rows * s.n_chunks * 8);
  L.chunk_w = take(rows * s.n_chunks * 4);
  L.tile_a = take(hq * nb * 4);
  L.tile_b = take(hq * nb * 4);
  const size_t nb_pad = (size_t)s.nt * 128;
  L.qhi = take(hq * nb * kHeadDim * 2);
  L.qlo = take(hq * nb * kHeadDim * 2);
  L.khi = take(hkv * nb_pad * kHeadDim * 2);
  L.klo = take(hkv * nb_pad * kHeadDim * 2);
  L.row_stat = take(hq * nb * 8);
  L.tile_kr = take(hq * (size_t)s.nt * s.nt * 4 * 8);
  L.tie_cnt = take(hq * nb * (size_t)s.nt * 4);
  L.tie_row = take(hq * nb * 4);
  L.hist = take(hq * sizeof(PeHist));
  L.pe_state = take(hq * sizeof(PeState));
  L.kv_pe = take(hkv * 4);
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
  L.pe_mask = take(hq * nb * (size_t)s.words * 4);
  L.pe_count = take(hq * 8);
  L.pe_cut = take(hq * 4);
  L.total = off;
  return L;
}

static IndexPtrs internal_index(char* ws, const WsLayout& L) {
  IndexPtrs p;
  p.route = reinterpret_cast<int32_t*>(ws + L.route);
  p.c_struct = reinterpret_cast<float*>(ws + L.c_struct);
  p.p_v = reinterpret_cast<float*>(ws + L.p_v);
  p.p_s = reinterpret_cast<float*>(ws + L.p_s);
  p.mu = reinterpret_cast<float*>(ws + L.mu);
  p.vs_mask = reinterpret_cast<uint32_t*>(ws + L.vs_mask);
  p.v_idx = reinterpret_cast<int32_t*>(ws + L.v_idx);
  p.s_idx = reinterpret_cast<int32_t*>(ws + L.s_idx);
  p.nv = reinterpret_cast<int32_t*>(ws + L.nv);
  p.ns = reinterpret_cast<int32_t*>(ws + L.ns);
  p.pe_mask = reinterpret_cast<uint32_t*>(ws + L.pe_mask);
  p.pe_count = reinterpret_cast<int64_t*>(ws + L.pe_count);
  p.pe_cut = reinterpret_cast<float*>(ws + L.pe_cut);
  return p;
}

static crisp_status make_shape(const crisp_cfg* c, Shape* s) {
  if (c == nullptr) return CRISP_ERR_INVALID_ARG;
  if (c->reserved != 0) return CRISP_ERR_INVALID_ARG;
  if (c->dtype != CRISP_BF16 && c->dtype != CRISP_FP32) return CRISP_ERR_DTYPE;
  if (c->d != kHeadDim) return CRISP_ERR_SHAPE;
  if (c->n < 512 || c->n % kBlock != 0 || c->n > (1 << 20)) return CRISP_ERR_SHAPE;
  if (c->h_q <= 0 || c->h_kv <= 0 || c->h_q % c->h_kv != 0 || c->h_q / c->h_kv > 16 || c->h_q > kMaxHeads)
    return CRISP_ERR_SHAPE;
  if (c->block != kBlock || c->last_q != kProxyRows || c->w_sink != kBlock || c->w_local != kBlock)
    return CRISP_ERR_UNSUPPORTED;
  if (!isfinite(c->tau_proxy) || !isfinite(c->alpha) || c->alpha < 0.f) return CRISP_ERR_INVALID_ARG;
  if (!(c->gamma > 0.f && c->gamma <= 1.f)) return CRISP_ERR_INVALID_ARG;
  if (!isfinite(c->sm_scale)) return CRISP_ERR_INVALID_ARG;
  if (c->force_route < -1 || c->force_route > 1) return CRISP_ERR_INVALID_ARG;
  s->n = c->n;
  s->h_q = c->h_q;
  s->h_kv = c->h_kv;
  s->d = c->d;
  s->group = c->h_q / c->h_kv;
  s->nb = c->n / kBlock;
  s->words = (s->nb + 31) / 32;
  s->n_chunks = (s->nb + kChunkTiles - 1) / kChunkTiles;
  s->last_q = c->last_q;
  s->nt = (s->nb + 127) / 128;
  s->fp32 = c->dtype == CRISP_FP32;
  s->sm_scale = c->sm_scale > 0.f ? c->sm_scale : 1.f / sqrtf((float)c->d);
  s->scale_log2 = s->sm_scale * 1.4426950408889634f;
  s->tau = c->tau_proxy;
  s->alpha = c->alpha;
  s->gamma = c->gamma;
  s->force_route = c->force_route;
  return CRISP_OK;
}

crisp_status shape_from_cfg(const crisp_cfg* c, Shape* s) { return make_shape(c, s); }

static crisp_status check_tensor(const void* p) {
  if (p == nullptr) return CRISP_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(p) % 16 != 0) return CRISP_ERR_ALIGN;
  return CRISP_OK;
}

static crisp_status check_ws(const crisp_cfg* c, const WsLayout& L) {
  if (c->workspace == nullptr) return CRISP_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(c->workspace) % 256 != 0) return CRISP_ERR_ALIGN;
  if (c->workspace_bytes < L.total) return CRISP_ERR_WORKSPACE;
  return CRISP_OK;
}

static crisp_status check_index(const crisp_index* ix, bool full) {
  if (ix == nullptr) return CRISP_ERR_INVALID_ARG;
  const void* need[] = {ix->route, ix->vs_mask, ix->pe_mask};
  for (const void* p : need)
    if (p == nullptr) return CRISP_ERR_INVALID_ARG;
  if (full) {
    const void* all[] = {ix->c_struct, ix->p_v, ix->p_s, ix->mu, ix->v_idx, ix->s_idx,
                         ix->nv, ix->ns, ix->pe_count, ix->pe_cut};
    for (const void* p : all)
      if (p == nullptr) return CRISP_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(ix->pe_count) % 8 != 0) return CRISP_ERR_ALIGN;
  }
  const void* al[] = {ix->route, ix->vs_mask, ix->pe_mask, ix->c_struct, ix->p_v, ix->p_s, ix->mu,
                      ix->v_idx, ix->s_idx, ix->nv, ix->ns, ix->pe_cut};
  for (const void* p : al)
    if (p != nullptr && reinterpret_cast<uintptr_t>(p) % 4 != 0) return CRISP_ERR_ALIGN;
  return CRISP_OK;
}

static IndexPtrs from_abi(const crisp_index* ix) {
  IndexPtrs p;
  p.route = ix->route;
  p.c_struct = ix->c_struct;
  p.p_v = ix->p_v;
  p.p_s = ix->p_s;
  p.mu = ix->mu;
  p.vs_mask = ix->vs_mask;
  p.v_idx = ix->v_idx;
  p.s_idx = ix->s_idx;
  p.nv = ix->nv;
  p.ns = ix->ns;
  p.pe_mask = ix->pe_mask;
  p.pe_count = ix->pe_count;
  p.pe_cut = ix->pe_cut;
  return p;
}

#define CRISP_TRY(expr)                         \
  do {                                          \
    if ((expr) != cudaSuccess) {                \
      (void)cudaGetLastError();                 \
      return CRISP_ERR_CUDA;                    \
    }                                           \
  } while (0)

// Algorithm 2 (proxy map, finalisation, route) and Algorithm 3's selection;
// Algorithm 4 too when `with_pe`. bf16 layers take the tensor-core proxy
// kernel unless `simt` (the diagnostics entry points) asks for the CUDA-core one.
static crisp_status run_index(const void* q, const void* k, const Shape& s, char* ws, const WsLayout& L,
                              const IndexPtrs& ix, bool with_pe, cudaStream_t st, bool simt = false) {
  CRISP_TRY(cudaMemsetAsync(ws + L.kv_pe, 0, (size_t)s.h_kv * 4, st));
  if (!s.fp32 && !simt)
    CRISP_TRY(launch_proxy_tc(q, k, s, ws, L, st));
  else
    CRISP_TRY(launch_proxy_simt(q, k, s, ws, L, st));
  CRISP_TRY(launch_finalize(s, ws, L, ix, st));
  CRISP_TRY(launch_vs_select(s, ws, L, ix, st));
  if (with_pe) CRISP_TRY(launch_pe(q, k, s, ws, L, ix, st));
  return CRISP_OK;
}

static crisp_status run_attention(const void* q, const void* k, const void* v, void* out, const Shape& s,
                                  char* ws, const WsLayout& L, const int32_t* route, const uint32_t* vs_mask,
                                  const uint32_t* pe_mask, bool dense, cudaStream_t st, bool simt = false) {
  int32_t* status = reinterpret_cast<int32_t*>(ws + L.status);
  if (!s.fp32 && !simt)
    CRISP_TRY(launch_attn_tc(q, k, v, out, s, route, vs_mask, pe_mask, dense, status, st));
  else
    CRISP_TRY(launch_attn_simt(q, k, v, out, s, route, vs_mask, pe_mask, dense, status, st));
  return CRISP_OK;
}

// Validate a call that reads q, k (and v, out when given) and uses the workspace.
static crisp_status prepare(const crisp_cfg* cfg, const void* q, const void* k, const void* v, const void* out,
                            bool need_vo, Shape* s, WsLayout* L) {
  crisp_status r = make_shape(cfg, s);
  if (r != CRISP_OK) return r;
  if ((r = check_tensor(q)) != CRISP_OK) return r;
  if ((r = check_tensor(k)) != CRISP_OK) return r;
  if (need_vo) {
    if ((r = check_tensor(v)) != CRISP_OK) return r;
    if ((r = check_tensor(out)) != CRISP_OK) return r;
  }
  *L = ws_layout(*s);
  return check_ws(cfg, *L);
}

// Algorithm 1 on one layer; `clear` resets the device status word first.
static crisp_status prefill_impl(const void* q, const void* k, const void* v, void* out, const crisp_cfg* cfg,
                                 cudaStream_t st, bool clear) {
  Shape s;
  WsLayout L;
  crisp_status r = prepare(cfg, q, k, v, out, true, &s, &L);
  if (r != CRISP_OK) return r;
  char* ws = static_cast<char*>(cfg->workspace);
  if (clear) CRISP_TRY(cudaMemsetAsync(ws + L.status, 0, 32, st));
  IndexPtrs ix = internal_index(ws, L);
  r = run_index(q, k, s, ws, L, ix, true, st);
  if (r != CRISP_OK) return r;
  return run_attention(q, k, v, out, s, ws, L, ix.route, ix.vs_mask, ix.pe_mask, false, st);
}

// One sequence's cfg -> the cfg of `batch` sequences laid out head after head.
static crisp_status fold_batch(const crisp_cfg* cfg, int32_t batch, crisp_cfg* folded) {
  if (cfg == nullptr || batch < 1) return CRISP_ERR_INVALID_ARG;
  const long long hq = (long long)cfg->h_q * batch, hkv = (long long)cfg->h_kv * batch;
  if (hq > INT32_MAX || hkv > INT32_MAX) return CRISP_ERR_INVALID_ARG;
  *folded = *cfg;
  folded->h_q = (int32_t)hq;
  folded->h_kv = (int32_t)hkv;
  return CRISP_OK;
}

// Device staging of crisp_prefill_host: one group's scratch workspace first
// (so the status word sits at offset 0, where crisp_device_status reads it),
// then two slots of one KV group's Q, K, V and out.
struct HostPlan {
  crisp_cfg group_cfg;       // one KV group: h_q / h_kv query heads, one K/V head
  size_t q_bytes, kv_bytes;  // per group
  size_t slot_bytes;         // Q + K + V + out of one group, 256-byte aligned pieces
  size_t slot_off, total;
};

static crisp_status host_plan(const crisp_cfg* cfg, HostPlan* p) {
  Shape s;
  crisp_status r = make_shape(cfg, &s);
  if (r != CRISP_OK) return r;
  p->group_cfg = *cfg;
  p->group_cfg.h_q = s.group;
  p->group_cfg.h_kv = 1;
  p->group_cfg.workspace = nullptr;
  p->group_cfg.workspace_bytes = 0;
  Shape gs;
  if ((r = make_shape(&p->group_cfg, &gs)) != CRISP_OK) return r;
  const size_t elem = s.fp32 ? 4 : 2;
  p->q_bytes = (size_t)s.group * s.n * s.d * elem;
  p->kv_bytes = (size_t)s.n * s.d * elem;
  p->slot_bytes = 2 * align256(p->q_bytes) + 2 * align256(p->kv_bytes);
  p->slot_off = align256(ws_layout(gs).total);
  p->total = p->slot_off + 2 * p->slot_bytes;
  return CRISP_OK;
}

}  // namespace crisp

using namespace crisp;

extern "C" {

crisp_status crisp_cfg_init(crisp_cfg* cfg, int32_t n, int32_t h_q, int32_t h_kv, int32_t d, int32_t dtype) {
  if (cfg == nullptr) return CRISP_ERR_INVALID_ARG;
  memset(cfg, 0, sizeof(*cfg));
  cfg->n = n;
  cfg->h_q = h_q;
  cfg->h_kv = h_kv;
  cfg->d = d;
  cfg->dtype = dtype;
  cfg->block = kBlock;
  cfg->last_q = kProxyRows;
  cfg->w_sink = kBlock;
  cfg->w_local = kBlock;
  cfg->tau_proxy = 0.10f;
  cfg->alpha = 1.0f;
  cfg->gamma = 0.95f;
  cfg->sm_scale = 0.f;
  cfg->force_route = CRISP_ROUTE_AUTO;
  return CRISP_OK;
}

crisp_status crisp_workspace_size(const crisp_cfg* cfg, size_t* bytes) {
  Shape s;
  crisp_status r = make_shape(cfg, &s);
  if (r != CRISP_OK) return r;
  if (bytes == nullptr) return CRISP_ERR_INVALID_ARG;
  *bytes = ws_layout(s).total;
  return CRISP_OK;
}

crisp_status crisp_index_dims(const crisp_cfg* cfg, int32_t* n_blocks, int32_t* words) {
  Shape s;
  crisp_status r = make_shape(cfg, &s);
  if (r != CRISP_OK) return r;
  if (n_blocks == nullptr || words == nullptr) return CRISP_ERR_INVALID_ARG;
  *n_blocks = s.nb;
  *words = s.words;
  return CRISP_OK;
}

crisp_status crisp_route(const void* q, const void* k, const crisp_cfg* cfg, int32_t* route, float* c_struct,
                         void* stream) {
  Shape s;
  WsLayout L;
  crisp_status r = prepare(cfg, q, k, nullptr, nullptr, false, &s, &L);
  if (r != CRISP_OK) return r;
  if (route == nullptr || c_struct == nullptr) return CRISP_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(cfg->workspace);
  CRISP_TRY(cudaMemsetAsync(ws + L.status, 0, 32, st));
  IndexPtrs ix = internal_index(ws, L);
  r = run_index(q, k, s, ws, L, ix, false, st);
  if (r != CRISP_OK) return r;
  CRISP_TRY(cudaMemcpyAsync(route, ix.route, (size_t)s.h_q * 4, cudaMemcpyDeviceToDevice, st));
  CRISP_TRY(cudaMemcpyAsync(c_struct, ix.c_struct, (size_t)s.h_q * 4, cudaMemcpyDeviceToDevice, st));
  return CRISP_OK;
}

crisp_status crisp_select(const void* q, const void* k, const crisp_cfg* cfg, const crisp_index* index,
                          void* stream) {
  Shape s;
  WsLayout L;
  crisp_status r = prepare(cfg, q, k, nullptr, nullptr, false, &s, &L);
  if (r != CRISP_OK) return r;
  if ((r = check_index(index, true)) != CRISP_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(cfg->workspace);
  CRISP_TRY(cudaMemsetAsync(ws + L.status, 0, 32, st));
  return run_index(q, k, s, ws, L, from_abi(index), true, st);
}

crisp_status crisp_attend(const void* q, const void* k, const void* v, void* out, const crisp_cfg* cfg,
                          const crisp_index* index, void* stream) {
  Shape s;
  WsLayout L;
  crisp_status r = prepare(cfg, q, k, v, out, true, &s, &L);
  if (r != CRISP_OK) return r;
  if ((r = check_index(index, false)) != CRISP_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(cfg->workspace);
  CRISP_TRY(cudaMemsetAsync(ws + L.status, 0, 32, st));
  return run_attention(q, k, v, out, s, ws, L, index->route, index->vs_mask, index->pe_mask, false, st);
}

crisp_status crisp_prefill(const void* q, const void* k, const void* v, void* out, const crisp_cfg* cfg,
                           void* stream) {
  return prefill_impl(q, k, v, out, cfg, static_cast<cudaStream_t>(stream), true);
}

crisp_status crisp_workspace_size_batch(const crisp_cfg* cfg, int32_t batch, size_t* bytes) {
  crisp_cfg f;
  crisp_status r = fold_batch(cfg, batch, &f);
  if (r != CRISP_OK) return r;
  return crisp_workspace_size(&f, bytes);
}

crisp_status crisp_prefill_batch(const void* q, const void* k, const void* v, void* out, const crisp_cfg* cfg,
                                 int32_t batch, void* stream) {
  crisp_cfg f;
  crisp_status r = fold_batch(cfg, batch, &f);
  if (r != CRISP_OK) return r;
  return prefill_impl(q, k, v, out, &f, static_cast<cudaStream_t>(stream), true);
}

crisp_status crisp_workspace_size_host(const crisp_cfg* cfg, size_t* bytes) {
  HostPlan p;
  crisp_status r = host_plan(cfg, &p);
  if (r != CRISP_OK) return r;
  if (bytes == nullptr) return CRISP_ERR_INVALID_ARG;
  *bytes = p.total;
  return CRISP_OK;
}

crisp_status crisp_prefill_host(const void* q, const void* k, const void* v, void* out, const crisp_cfg* cfg,
                                void* stream, void* copy_stream) {
  HostPlan p;
  crisp_status r = host_plan(cfg, &p);
  if (r != CRISP_OK) return r;
  const void* hp[] = {q, k, v, out};
  for (const void* x : hp)
    if ((r = check_tensor(x)) != CRISP_OK) return r;
  if (cfg->workspace == nullptr) return CRISP_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(cfg->workspace) % 256 != 0) return CRISP_ERR_ALIGN;
  if (cfg->workspace_bytes < p.total) return CRISP_ERR_WORKSPACE;
  if (copy_stream == stream) return CRISP_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream), cs = static_cast<cudaStream_t>(copy_stream);
  char* ws = static_cast<char*>(cfg->workspace);
  crisp_cfg gc = p.group_cfg;
  gc.workspace = ws;
  gc.workspace_bytes = p.slot_off;
  const int n_groups = cfg->h_kv;
  char* slot_q[2];
  char* slot_k[2];
  char* slot_v[2];
  char* slot_o[2];
  for (int b = 0; b < 2; ++b) {
    char* base = ws + p.slot_off + b * p.slot_bytes;
    slot_q[b] = base;
    slot_k[b] = base + align256(p.q_bytes);
    slot_v[b] = slot_k[b] + align256(p.kv_bytes);
    slot_o[b] = slot_v[b] + align256(p.kv_bytes);
  }
  // events: group copied in, group computed; one more for the last copy out
  const int n_ev = 2 * n_groups + 1;
  std::vector<cudaEvent_t> ev(n_ev);
  for (int i = 0; i < n_ev; ++i) {
    if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(ev[j]);
      return CRISP_ERR_CUDA;
    }
  }
  cudaEvent_t* ev_in = ev.data();
  cudaEvent_t* ev_done = ev.data() + n_groups;
  cudaEvent_t ev_last = ev[2 * n_groups];
  auto h2d = [&](int g) -> cudaError_t {
    const int b = g & 1;
    cudaError_t e;
    if ((e = cudaMemcpyAsync(slot_q[b], static_cast<const char*>(q) + g * p.q_bytes, p.q_bytes,
                             cudaMemcpyHostToDevice, cs)) != cudaSuccess)
      return e;
    if ((e = cudaMemcpyAsync(slot_k[b], static_cast<const char*>(k) + g * p.kv_bytes, p.kv_bytes,
                             cudaMemcpyHostToDevice, cs)) != cudaSuccess)
      return e;
    if ((e = cudaMemcpyAsync(slot_v[b], static_cast<const char*>(v) + g * p.kv_bytes, p.kv_bytes,
                             cudaMemcpyHostToDevice, cs)) != cudaSuccess)
      return e;
    return cudaEventRecord(ev_in[g], cs);
  };
  auto d2h = [&](int g) -> cudaError_t {
    cudaError_t e;
    if ((e = cudaStreamWaitEvent(cs, ev_done[g], 0)) != cudaSuccess) return e;
    return cudaMemcpyAsync(static_cast<char*>(out) + g * p.q_bytes, slot_o[g & 1], p.q_bytes,
                           cudaMemcpyDeviceToHost, cs);
  };
  // the copy stream must not start before work the caller queued on `stream`
  // (e.g. producing the host buffers' consumers) is ordered: start both
  // streams from the same point
  cudaError_t e = cudaEventRecord(ev_last, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, ev_last, 0);
  for (int g = 0; g < n_groups && e == cudaSuccess && r == CRISP_OK; ++g) {
    // copy stream: group g in (its slot was emptied by group g-2's copy out)
    if (g >= 2 && (e = d2h(g - 2)) != cudaSuccess) break;
    if (g < 2 && (e = h2d(g)) != cudaSuccess) break;
    if (g >= 2 && (e = h2d(g)) != cudaSuccess) break;
    // compute stream: group g once it is in
    if ((e = cudaStreamWaitEvent(st, ev_in[g], 0)) != cudaSuccess) break;
    const int b = g & 1;
    r = prefill_impl(slot_q[b], slot_k[b], slot_v[b], slot_o[b], &gc, st, g == 0);
    if (r == CRISP_OK) e = cudaEventRecord(ev_done[g], st);
  }
  // the last two groups' outputs, then `stream` waits for the copy stream
  for (int g = std::max(0, n_groups - 2); g < n_groups && e == cudaSuccess && r == CRISP_OK; ++g) e = d2h(g);
  if (e == cudaSuccess && r == CRISP_OK) e = cudaEventRecord(ev_last, cs);
  if (e == cudaSuccess && r == CRISP_OK) e = cudaStreamWaitEvent(st, ev_last, 0);
  for (int i = 0; i < n_ev; ++i) cudaEventDestroy(ev[i]);
  if (r != CRISP_OK) return r;
  return e == cudaSuccess ? CRISP_OK : CRISP_ERR_CUDA;
}

crisp_status crisp_prefill_varlen(const void* const* q, const void* const* k, const void* const* v,
                                  void* const* out, const int32_t* n, int32_t count, const crisp_cfg* cfg,
                                  void* stream) {
  if (cfg == nullptr || q == nullptr || k == nullptr || v == nullptr || out == nullptr || n == nullptr || count < 1)
    return CRISP_ERR_INVALID_ARG;
  // every sequence is checked before anything is launched
  for (int32_t i = 0; i < count; ++i) {
    crisp_cfg c = *cfg;
    c.n = n[i];
    Shape s;
    WsLayout L;
    crisp_status r = prepare(&c, q[i], k[i], v[i], out[i], true, &s, &L);
    if (r != CRISP_OK) return r;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  for (int32_t i = 0; i < count; ++i) {
    crisp_cfg c = *cfg;
    c.n = n[i];
    // the status word is cleared by the first sequence only, so a device-side
    // failure of any sequence stays visible (later kernels see it and stop)
    crisp_status r = prefill_impl(q[i], k[i], v[i], out[i], &c, st, i == 0);
    if (r != CRISP_OK) return r;
  }
  return CRISP_OK;
}

crisp_status crisp_dense_attention(const void* q, const void* k, const void* v, void* out, const crisp_cfg* cfg,
                                   void* stream) {
  Shape s;
  WsLayout L;
  crisp_status r = prepare(cfg, q, k, v, out, true, &s, &L);
  if (r != CRISP_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(cfg->workspace);
  CRISP_TRY(cudaMemsetAsync(ws + L.status, 0, 32, st));
  return run_attention(q, k, v, out, s, ws, L, nullptr, nullptr, nullptr, true, st);
}

crisp_status crisp_diag_select_simt(const void* q, const void* k, const crisp_cfg* cfg, const crisp_index* index,
                                    void* stream) {
  Shape s;
  WsLayout L;
  crisp_status r = prepare(cfg, q, k, nullptr, nullptr, false, &s, &L);
  if (r != CRISP_OK) return r;
  if ((r = check_index(index, true)) != CRISP_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(cfg->workspace);
  CRISP_TRY(cudaMemsetAsync(ws + L.status, 0, 32, st));
  return run_index(q, k, s, ws, L, from_abi(index), true, st, true);
}

crisp_status crisp_diag_attend_simt(const void* q, const void* k, const void* v, void* out, const crisp_cfg* cfg,
                                    const crisp_index* index, int32_t dense, void* stream) {
  Shape s;
  WsLayout L;
  crisp_status r = prepare(cfg, q, k, v, out, true, &s, &L);
  if (r != CRISP_OK) return r;
  if (!dense && (r = check_index(index, false)) != CRISP_OK) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(cfg->workspace);
  CRISP_TRY(cudaMemsetAsync(ws + L.status, 0, 32, st));
  if (dense) return run_attention(q, k, v, out, s, ws, L, nullptr, nullptr, nullptr, true, st, true);
  return run_attention(q, k, v, out, s, ws, L, index->route, index->vs_mask, index->pe_mask, false, st, true);
}

crisp_status crisp_device_status(const crisp_cfg* cfg, void* stream, int32_t* device_status) {
  Shape s;
  crisp_status r = make_shape(cfg, &s);
  if (r != CRISP_OK) return r;
  if (device_status == nullptr) return CRISP_ERR_INVALID_ARG;
  // only the status word (the first 32 bytes of every workspace layout) is read
  if (cfg->workspace == nullptr) return CRISP_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(cfg->workspace) % 256 != 0) return CRISP_ERR_ALIGN;
  if (cfg->workspace_bytes < 256) return CRISP_ERR_WORKSPACE;
  const WsLayout L = ws_layout(s);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(cfg->workspace);
  int32_t word[2] = {0, 0};
  CRISP_TRY(cudaStreamSynchronize(st));
  CRISP_TRY(cudaMemcpy(word, ws + L.status, sizeof(word), cudaMemcpyDeviceToHost));
  CRISP_TRY(cudaMemset(ws + L.status, 0, 32));
  *device_status = word[0];
  return CRISP_OK;
}

const char* crisp_status_string(crisp_status status) {
  switch (status) {
    case CRISP_OK: return "ok";
    case CRISP_ERR_INVALID_ARG: return "invalid argument";
    case CRISP_ERR_SHAPE: return "unsupported shape";
    case CRISP_ERR_DTYPE: return "unsupported element type";
    case CRISP_ERR_ALIGN: return "misaligned pointer";
    case CRISP_ERR_WORKSPACE: return "workspace missing or too small";
    case CRISP_ERR_UNSUPPORTED: return "unsupported parameter value";
    case CRISP_ERR_CUDA: return "CUDA runtime error";
    case CRISP_ERR_CAPACITY: return "device buffer capacity exceeded";
    case CRISP_ERR_TIMEOUT: return "device wait timed out";
    case CRISP_ERR_NONFINITE: return "non-finite proxy statistic";
    case CRISP_ERR_TOO_LARGE: return "layer too large for the static scratch array";
  }
  return "unknown status";
}

int32_t crisp_version(void) { return 100; }

}  // extern "C"
