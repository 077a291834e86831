/*
 * crisp.h -- C ABI of the CRISP sparse-prefill attention library (B200, sm_100a).
 *
 * CRISP ("Cliff-awaRe Input-adaptive Sparse Prefilling with
 * Structural-Mass-Motivated Routing") prefills one attention layer in three
 * stages per query head (CRISP paper summary page, Methodology and
 * "Algorithm Overview", Algorithms 1-4):
 *
 *   1. proxy map A-hat: the last |Q-hat| = 64 queries scored against every
 *      key, causal softmax taken after the scores (Algorithm 2);
 *   2. route: C_struct = mean post-softmax mass on S_anchor (first w_sink
 *      keys plus the w_local-key recency window), Eq. (2); the head goes to
 *      Vertical-Slash (VS) if C_struct >= tau_proxy, else to pooled
 *      estimation (PE);
 *   3. selection: VS keeps column blocks and diagonal (offset) blocks whose
 *      mass p_j exceeds alpha * mu, the sink-aware noise floor of Eq. (3)-(4),
 *      always keeping the first and last block (Algorithm 3); PE pools Q and
 *      K per block, scores the block map by softmax and keeps the smallest
 *      gamma-cumulative set of blocks (Algorithm 4). Then exact causal
 *      attention over exactly the selected keys (Algorithm 1).
 *
 * Tensors (all device memory, batch 1, head-major, contiguous, row-major):
 *   q, out : [h_q ][n][d]      k, v : [h_kv][n][d]
 * element type bf16 or fp32 (cfg.dtype); out has the same type as q.
 * Query head h reads KV head h / (h_q / h_kv) (grouped-query attention).
 * Blocks: B = cfg.block = 128 keys; N_b = n / B; W = ceil(N_b / 32).
 *
 * Conventions
 * - Every entry point validates its arguments before it launches anything;
 *   a failed validation returns an error and leaves memory untouched.
 * - No entry point synchronises with the host, allocates memory or keeps
 *   global mutable state (one exception, crisp_route_noalloc, is described
 *   at its declaration). All scratch lives in the caller's workspace
 *   (cfg.workspace, >= crisp_workspace_size bytes of device memory, 256-byte
 *   aligned). Calls that share a workspace must be ordered (same stream).
 * - `stream` is a cudaStream_t passed as a plain pointer (NULL = legacy
 *   default stream). All work is enqueued on it.
 * - Conditions found on the device (a bounded wait that ran out, a
 *   non-finite proxy statistic) never trap: they set the workspace status
 *   word, which crisp_device_status reads. Each entry point clears the
 *   status word when it starts, so it reports on the most recent call.
 * - Host-side launch failures return CRISP_ERR_CUDA.
 */
#ifndef CRISP_H
#define CRISP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CRISP_OK = 0,
  CRISP_ERR_INVALID_ARG = 1,   /* null pointer, non-finite or out-of-range knob */
  CRISP_ERR_SHAPE = 2,         /* n, h_q, h_kv, d outside what this build supports */
  CRISP_ERR_DTYPE = 3,         /* unknown element type */
  CRISP_ERR_ALIGN = 4,         /* a tensor or workspace pointer not 16/256-byte aligned */
  CRISP_ERR_WORKSPACE = 5,     /* workspace missing or smaller than crisp_workspace_size */
  CRISP_ERR_UNSUPPORTED = 6,   /* a knob value the kernels do not implement */
  CRISP_ERR_CUDA = 7,          /* a CUDA runtime call or launch failed */
  CRISP_ERR_CAPACITY = 8,      /* device-side: an internal buffer would overflow */
  CRISP_ERR_TIMEOUT = 9,       /* device-side: a bounded wait ran out */
  CRISP_ERR_NONFINITE = 10,    /* device-side: a proxy statistic was NaN or infinite */
  CRISP_ERR_TOO_LARGE = 11     /* crisp_route_noalloc: the layer needs more scratch than its static array */
} crisp_status;

typedef enum { CRISP_BF16 = 0, CRISP_FP32 = 1 } crisp_dtype;

typedef enum { CRISP_ROUTE_AUTO = -1, CRISP_ROUTE_VS = 0, CRISP_ROUTE_PE = 1 } crisp_route_t;

/* Layer shape and the method's knobs. Defaults are set by crisp_cfg_init. */
typedef struct {
  int32_t n;            /* sequence length; this build: multiple of 128, 512 <= n <= 1048576 */
  int32_t h_q;          /* query heads */
  int32_t h_kv;         /* key/value heads; h_q % h_kv == 0, h_q / h_kv <= 16 */
  int32_t d;            /* head dimension; this build: 128 */
  int32_t dtype;        /* crisp_dtype */
  int32_t block;        /* B, block size of the partition (summary page, Eq. (3) text): 128 */
  int32_t last_q;       /* |Q-hat|, proxy query rows (Algorithm 2): 64 */
  int32_t w_sink;       /* sink window of S_anchor (Eq. (2) text): 128 */
  int32_t w_local;      /* recency window of S_anchor (Eq. (2) text): 128 */
  float tau_proxy;      /* route threshold of C_struct; the pages give no value: default 0.10 */
  float alpha;          /* Eq. (4) multiplier on the noise floor; default 1.0; >= 0 */
  float gamma;          /* PE cumulative coverage (Algorithm 4); default 0.95; in (0, 1] */
  float sm_scale;       /* softmax scale; <= 0 means 1/sqrt(d) */
  int32_t force_route;  /* crisp_route_t: -1 route by C_struct, 0 force VS, 1 force PE */
  int32_t reserved;     /* must be 0 */
  void* workspace;      /* device scratch owned by the caller */
  size_t workspace_bytes;
} crisp_cfg;

/* Selection outputs; every pointer is a caller-owned device buffer.
 * Bit b of a mask lives in word b / 32, bit position b % 32. */
typedef struct {
  int32_t* route;       /* [h_q]           0 = VS, 1 = PE */
  float* c_struct;      /* [h_q]           Eq. (2) */
  float* p_v;           /* [h_q][N_b]      column-block masses (sum over each block of the column means) */
  float* p_s;           /* [h_q][N_b]      offset-block masses (diagonal i - j in [bB, bB+B)) */
  float* mu;            /* [h_q][2]        noise floors (mu_v, mu_s), Eq. (3) */
  uint32_t* vs_mask;    /* [h_q][2][W]     selected column blocks, then selected offset blocks */
  int32_t* v_idx;       /* [h_q][N_b]      selected column blocks, ascending, first nv[h] valid */
  int32_t* s_idx;       /* [h_q][N_b]      selected offset blocks, ascending, first ns[h] valid */
  int32_t* nv;          /* [h_q] */
  int32_t* ns;          /* [h_q] */
  uint32_t* pe_mask;    /* [h_q][N_b][W]   PE block mask, row = query block; valid where route == PE */
  int64_t* pe_count;    /* [h_q]           selected causal blocks of the PE mask (0 for VS heads) */
  float* pe_cut;        /* [h_q]           normalised value of the last block kept by the gamma cut
                                           (0 when every block is kept or the head is VS) */
} crisp_index;

/* Fill *cfg with the defaults above for the given shape (workspace NULL). */
crisp_status crisp_cfg_init(crisp_cfg* cfg, int32_t n, int32_t h_q, int32_t h_kv, int32_t d, int32_t dtype);

/* Bytes of workspace the calls below need for cfg's shape. */
crisp_status crisp_workspace_size(const crisp_cfg* cfg, size_t* bytes);

/* Number of 32-bit words W per mask row, and N_b, for cfg's shape. */
crisp_status crisp_index_dims(const crisp_cfg* cfg, int32_t* n_blocks, int32_t* words);

/* Algorithm 2 (PatSearch): proxy map, C_struct (Eq. (2)) and the route of
 * every query head. Writes route[h_q] and c_struct[h_q] (device). */
crisp_status crisp_route(const void* q, const void* k, const crisp_cfg* cfg,
                         int32_t* route, float* c_struct, void* stream);

/* Algorithms 2-4: route and the selected index sets of every head. */
crisp_status crisp_select(const void* q, const void* k, const crisp_cfg* cfg,
                          const crisp_index* index, void* stream);

/* Algorithm 1's last step: causal attention over the keys the given index
 * selects (index->route, vs_mask and pe_mask are read, nothing else). */
crisp_status crisp_attend(const void* q, const void* k, const void* v, void* out,
                          const crisp_cfg* cfg, const crisp_index* index, void* stream);

/* Algorithm 1: route, select and sparse attention for the whole layer. */
crisp_status crisp_prefill(const void* q, const void* k, const void* v, void* out,
                           const crisp_cfg* cfg, void* stream);

/* Algorithm 1 for `batch` independent sequences of one length (no
 * counterpart in the paper, which treats one prompt at a time). q and out
 * are [batch][h_q][n][d], k and v [batch][h_kv][n][d], contiguous; cfg
 * describes ONE sequence. Every stage works per head and the sequences are
 * laid out head after head, so the call is crisp_prefill on the folded shape
 * (batch*h_q query heads, batch*h_kv key/value heads; query head b*h_q + j
 * reads key/value head b*h_kv + j / (h_q/h_kv), i.e. its own sequence's).
 * cfg->workspace must hold crisp_workspace_size_batch(cfg, batch) bytes.
 * batch < 1: CRISP_ERR_INVALID_ARG; a folded shape outside the limits of a
 * single call (h_q * batch <= 1024): CRISP_ERR_SHAPE. */
crisp_status crisp_prefill_batch(const void* q, const void* k, const void* v, void* out,
                                 const crisp_cfg* cfg, int32_t batch, void* stream);

/* Workspace bytes crisp_prefill_batch needs for `batch` sequences of cfg's shape. */
crisp_status crisp_workspace_size_batch(const crisp_cfg* cfg, int32_t batch, size_t* bytes);

/* Algorithm 1 for `count` sequences of different lengths (no counterpart in
 * the paper). Sequence i has its own tensors q[i], out[i] ([h_q][n[i]][d])
 * and k[i], v[i] ([h_kv][n[i]][d]); q, k, v, out and n are HOST arrays of
 * `count` entries (device pointers inside q..out). Each length obeys the
 * rules of cfg->n; cfg->n itself is ignored. The sequences run one after
 * another on `stream` and share cfg's workspace, which must hold
 * crisp_workspace_size for the longest one. Arguments are checked for every
 * sequence before anything is launched; on an error nothing runs. */
crisp_status crisp_prefill_varlen(const void* const* q, const void* const* k, const void* const* v,
                                  void* const* out, const int32_t* n, int32_t count,
                                  const crisp_cfg* cfg, void* stream);

/* Algorithm 1 on a layer held in HOST memory (no counterpart in the paper).
 * q and out are host [h_q][n][d], k and v host [h_kv][n][d]; they should be
 * page-locked (cudaHostAlloc / cudaHostRegister) or the copies do not
 * overlap. The layer runs one KV group at a time (its h_q/h_kv query heads
 * and one K/V head, the same arithmetic as crisp_prefill on the whole layer):
 * while group g is computed on `stream`, group g+1 is copied in and group
 * g-1's output copied out on `copy_stream` (a different stream), with
 * events ordering the two. cfg describes the whole layer; cfg->workspace
 * must hold crisp_workspace_size_host(cfg) bytes (one group's scratch, whose
 * status word crisp_device_status reads as usual, then device copies of two
 * groups' Q, K, V and out). The call returns once
 * everything is enqueued; when `stream` completes, out holds the result, so
 * the host buffers must stay valid until then. copy_stream == stream:
 * CRISP_ERR_INVALID_ARG. */
crisp_status crisp_prefill_host(const void* q, const void* k, const void* v, void* out,
                                const crisp_cfg* cfg, void* stream, void* copy_stream);

/* Workspace bytes crisp_prefill_host needs for cfg's layer. */
crisp_status crisp_workspace_size_host(const crisp_cfg* cfg, size_t* bytes);

/* Exact dense causal attention with the same kernels (the speed reference). */
crisp_status crisp_dense_attention(const void* q, const void* k, const void* v, void* out,
                                   const crisp_cfg* cfg, void* stream);

/* Synchronise `stream`, then read (and clear) the workspace status word.
 * *device_status receives a crisp_status code (CRISP_OK if none). */
crisp_status crisp_device_status(const crisp_cfg* cfg, void* stream, int32_t* device_status);

/* Short English description of a status code (static storage). */
const char* crisp_status_string(crisp_status status);

/* crisp_route without caller memory. The paper has no counterpart; this is
 * for callers that cannot give the library device memory at all: a plugin
 * hook whose enqueue call hands over no workspace pointer, or a serving loop
 * that forbids device allocation once it is running. It computes exactly what
 * crisp_route computes (same kernels, same outputs), but its scratch is a
 * static 32 MiB device array inside the library (CRISP_NOALLOC_SCRATCH_BYTES),
 * which every GPU that loads the library holds until the process exits.
 * - cfg->workspace and cfg->workspace_bytes are ignored; q, k, route and
 *   c_struct are the caller's device buffers as for crisp_route.
 * - Layers needing more scratch than the array holds (about
 *   h_q * n / 128 * 640 bytes; e.g. 32 query heads up to n = 131072) are
 *   rejected with CRISP_ERR_TOO_LARGE before anything is launched.
 * - The array's device address is looked up on the first call on each
 *   device, with that device current; make that first call before any stream
 *   capture on the device. A failed lookup is not cached (the next call tries
 *   again). The address belongs to the device's primary context: after
 *   cudaDeviceReset the process must not call this entry point again.
 * - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * - All calls share the one array and leave their contents in it (each call
 *   clears what must start at zero): calls that can overlap on the GPU
 *   (different streams, or several host threads) race and must be
 *   serialised by the caller.
 * - Device-side failures are reported in the outputs, since there is no
 *   caller workspace for crisp_device_status to read: if a bounded wait ran
 *   out or a proxy statistic was NaN or infinite (for example a NaN in the
 *   last 64 query rows), every route[h] is -1 and every c_struct[h] NaN once
 *   the stream completes. */
#define CRISP_NOALLOC_SCRATCH_BYTES (32u << 20)
crisp_status crisp_route_noalloc(const void* q, const void* k, const crisp_cfg* cfg,
                                 int32_t* route, float* c_struct, void* stream);

/* Diagnostics: evaluate, on the device, the exp2 approximations the kernels
 * use on the FMA pipe (degree-3 and degree-5 minimax polynomials after an
 * integer/fraction split) next to CUDA's exp2f, for n float32 inputs x
 * (device pointers; poly3, poly5 and ref receive n values each). */
crisp_status crisp_exp2_selftest(const float* x, float* poly3, float* poly5, float* ref, int32_t n, void* stream);

/* Diagnostics: run the bounded mbarrier wait every kernel uses against a
 * barrier nothing arrives on, giving up after limit_cycles SM clocks
 * (1000 <= limit_cycles <= 4e9). status points to 8 int32 of device memory
 * laid out like the workspace status word (zeroed by the caller); after the
 * stream completes it holds CRISP_ERR_TIMEOUT and the wait site 99. Checks
 * that a wait which runs out ends the kernel with a status, not a hang. */
crisp_status crisp_wait_selftest(int64_t limit_cycles, int32_t* status, void* stream);

/* Diagnostics: crisp_select and crisp_attend with the proxy map and the
 * attention on the CUDA-core kernels that fp32 layers use, for bf16 layers
 * too, so that a test can hold the tensor-core kernels against a second
 * implementation on the same inputs. Arguments as for crisp_select and
 * crisp_attend; dense != 0 attends over every causal key (as
 * crisp_dense_attention; index may then be NULL). Not a production path. */
crisp_status crisp_diag_select_simt(const void* q, const void* k, const crisp_cfg* cfg,
                                    const crisp_index* index, void* stream);
crisp_status crisp_diag_attend_simt(const void* q, const void* k, const void* v, void* out,
                                    const crisp_cfg* cfg, const crisp_index* index, int32_t dense,
                                    void* stream);

/* Library version as major*10000 + minor*100 + patch. */
int32_t crisp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CRISP_H */
