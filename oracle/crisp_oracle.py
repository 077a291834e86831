"""CPU oracle for CRISP sparse prefill attention -- TEST INFRASTRUCTURE ONLY.

Plain, slow, float64 restatement of what the method computes. Only the tests,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may import it.
It shares no code with the CUDA library and never reads anything the CUDA
path produced.

Sources (web pages on CRISP, "Cliff-awaRe Input-adaptive Sparse Prefilling
with Structural-Mass-Motivated Routing"):

* [S]  the paper summary page (picx.dev): Methodology -- Eq. (2) C_struct,
       S_anchor, routing rule; "Sink-Aware Thresholding" -- block partition,
       Eq. (3) noise floor, Eq. (4) selection rule, alpha = 1.0 default;
       "Algorithm Overview" -- Algorithms 1-4.
* [W]  the AI-research-wiki page on CRISP: "What it actually does" (prose on
       the proxy map, C_struct and the noise-floor cut).

Readings taken where the pages leave a step open (each is also listed in the
design notes of the repository):

* Q-hat (the "query subset" of Algorithm 2) is the last ``last_q`` = 64 query
  rows; the proxy map is their causal softmax over all keys.
* S_anchor(i) is the set union {j < w_sink} U {j : 0 <= i - j < w_local}
  (sinks plus a per-query recency window), counted once.
* a_v (column means) and a_s (diagonal means) divide by |Q-hat| with masked
  entries counted as zero, so each sums to one; block pooling is a sum, so a
  block score p_j is a block mass as Eq. (3) treats it.
* For the diagonal direction the retained "first" and "last" blocks are the
  offset blocks N_b - 1 (the diagonal through the sinks) and 0 (the local
  window). N_b <= 2 keeps every block.
* Algorithm 4 pools Q and K by block mean, masks c > r (block-causal), scales
  by sm_scale, normalises the flattened map by its total, sorts descending
  with ties broken by ascending flat index r*N_b + c, and keeps the smallest
  prefix whose float64 cumulative sum reaches gamma (all of it if the sum
  never does, or if gamma >= 1). The diagonal block (r, r) is always kept so
  every query attends to at least one key (our addition).
* Sparse attention is exact softmax attention restricted to the selected
  keys: VS keeps key j <= i when its column block or its diagonal (offset)
  block is selected; PE keeps it when block (i//B, j//B) is selected.

Parity pins: see tests/test_oracle_pins.py (brute force on tiny inputs, closed
forms for uniform logits, a library dense-attention check, hand-built
selection cases and planted-structure invariants). No function here is
"parity unpinned" except the choice of tau_proxy itself, which the pages never
give.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Tuple

import numpy as np

VS, PE = 0, 1


@dataclasses.dataclass(frozen=True)
class OracleCfg:
    block: int = 128          # B, [S] Sink-Aware Thresholding
    last_q: int = 64          # |Q-hat|
    w_sink: int = 128         # [S] Eq. (2) text
    w_local: int = 128        # [S] Eq. (2) text
    tau_proxy: float = 0.10   # not given by the pages (our default)
    alpha: float = 1.0        # [S] Eq. (4): the pages' default multiplier
    gamma: float = 0.95       # PE coverage
    sm_scale: Optional[float] = None   # default 1/sqrt(d)
    force_route: int = -1     # -1 auto, 0 VS, 1 PE

    def scale(self, d: int) -> float:
        return self.sm_scale if self.sm_scale is not None else 1.0 / math.sqrt(d)


def n_blocks(n: int, B: int) -> int:
    return -(-n // B)


# ------------------------------------------------------------------ Algorithm 2

def proxy_rows(n: int, last_q: int) -> np.ndarray:
    """Positions of Q-hat: the last ``last_q`` queries (clipped to n)."""
    return np.arange(max(0, n - last_q), n)


def proxy_map(q_hat: np.ndarray, k: np.ndarray, rows: np.ndarray, sm_scale: float) -> np.ndarray:
    """Representative attention A-hat on the query subset ([S] Algorithm 2).

    Scores sm_scale * q_i . k_j for j <= i, softmax taken after the scores,
    zero for j > i. Returns [len(rows), n] float64.
    """
    s = sm_scale * (q_hat @ k.T)
    j = np.arange(k.shape[0])
    future = j[None, :] > rows[:, None]
    s[future] = -np.inf
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    e[future] = 0.0
    return e / e.sum(axis=1, keepdims=True)


def anchor_mask(rows: np.ndarray, n: int, w_sink: int, w_local: int) -> np.ndarray:
    """S_anchor(i) for each proxy row: sinks (first w_sink keys) union the local
    recency window (the w_local keys ending at i), [S] text under Eq. (2)."""
    j = np.arange(n)[None, :]
    i = rows[:, None]
    return (j < w_sink) | ((i - j >= 0) & (i - j < w_local))


def c_struct(A: np.ndarray, rows: np.ndarray, w_sink: int, w_local: int) -> float:
    """Eq. (2): (1/|Q-hat|) sum_i sum_{j in S_anchor} A-hat[i, j]."""
    mask = anchor_mask(rows, A.shape[1], w_sink, w_local)
    return float((A * mask).sum(axis=1).sum() / A.shape[0])


def route_of(c: float, tau_proxy: float, force_route: int = -1) -> int:
    """[S] Methodology: VS if C_struct >= tau_proxy, PE otherwise."""
    if force_route in (VS, PE):
        return force_route
    return VS if c >= tau_proxy else PE


# ------------------------------------------------------------------ Algorithm 3

def directional_scores(A: np.ndarray, rows: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Column means a_v[j] and diagonal means a_s[o] of A-hat ([S] Algorithm 3).

    a_s[o] averages A-hat[i, i - o] over the proxy rows (offset o = i - j).
    Both divide by |Q-hat|; masked entries count as zero.
    """
    nq, n = A.shape
    a_v = A.sum(axis=0) / nq
    a_s = np.zeros(n)
    for r, i in enumerate(rows):
        # offsets 0..i correspond to keys i..0
        a_s[: i + 1] += A[r, i::-1]
    a_s /= nq
    return a_v, a_s


def block_pool(a: np.ndarray, B: int) -> np.ndarray:
    """Sum of a over consecutive blocks of B positions (last block may be short)."""
    nb = n_blocks(len(a), B)
    pad = np.zeros(nb * B)
    pad[: len(a)] = a
    return pad.reshape(nb, B).sum(axis=1)


def noise_floor(p: np.ndarray, first: int, last: int) -> float:
    """Eq. (3): mu = max(1 - a_first - a_last, 0) / (N_b - 2)."""
    nb = len(p)
    return max(1.0 - p[first] - p[last], 0.0) / (nb - 2)


def threshold_blocks(p: np.ndarray, first: int, last: int, alpha: float) -> Tuple[np.ndarray, float]:
    """Eq. (4): keep block j iff p_j > alpha * mu; first and last always kept."""
    nb = len(p)
    if nb <= 2:
        return np.ones(nb, dtype=bool), 0.0
    mu = noise_floor(p, first, last)
    sel = p > alpha * mu
    sel[first] = True
    sel[last] = True
    return sel, mu


def vs_index(p_v: np.ndarray, p_s: np.ndarray, alpha: float):
    """[S] Algorithm 3 on block-pooled directional scores.

    Vertical: first = column block 0 (sinks), last = column block N_b-1.
    Diagonal: first = offset block N_b-1, last = offset block 0 (local).
    Returns (sel_v, sel_s, mu_v, mu_s).
    """
    nb = len(p_v)
    sel_v, mu_v = threshold_blocks(p_v, 0, nb - 1, alpha)
    sel_s, mu_s = threshold_blocks(p_s, nb - 1, 0, alpha)
    return sel_v, sel_s, mu_v, mu_s


# ------------------------------------------------------------------ Algorithm 4

def block_mean(x: np.ndarray, B: int) -> np.ndarray:
    """Mean of the rows of x over consecutive blocks of B rows (short tail block
    averages only the rows it has). x: [n, d] -> [N_b, d]."""
    n, d = x.shape
    nb = n_blocks(n, B)
    out = np.empty((nb, d))
    for b in range(nb):
        out[b] = x[b * B: min(n, (b + 1) * B)].mean(axis=0)
    return out


def pooled_map(q: np.ndarray, k: np.ndarray, B: int, sm_scale: float) -> np.ndarray:
    """A-bar = Softmax(Q-bar K-bar^T * sm_scale) over c <= r ([S] Algorithm 4).

    Returns [N_b, N_b] with zeros above the diagonal.
    """
    qb, kb = block_mean(q, B), block_mean(k, B)
    s = sm_scale * (qb @ kb.T)
    nb = s.shape[0]
    upper = np.triu(np.ones((nb, nb), dtype=bool), k=1)
    s[upper] = -np.inf
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    e[upper] = 0.0
    return e / e.sum(axis=1, keepdims=True)


@dataclasses.dataclass
class PESelection:
    mask: np.ndarray        # [N_b, N_b] bool, block-causal
    values: np.ndarray      # [N_b, N_b] normalised A-bar (zeros above diagonal)
    k_star: int             # number of entries kept by the gamma cut
    cut_value: float        # value of the K*-th entry in sorted order (0 if all kept)


def gamma_select(abar: np.ndarray, gamma: float) -> PESelection:
    """Flatten the causal entries, normalise by their total, sort descending
    (ties by ascending flat index), keep the shortest prefix whose cumulative
    sum reaches gamma; add the diagonal ([S] Algorithm 4)."""
    nb = abar.shape[0]
    r, c = np.tril_indices(nb)
    vals = abar[r, c]
    total = vals.sum()
    a = vals / total
    flat = r * nb + c
    order = np.lexsort((flat, -a))
    if gamma >= 1.0:
        k_star = len(a)
    else:
        cs = np.cumsum(a[order])
        hit = np.nonzero(cs >= gamma)[0]
        k_star = int(hit[0]) + 1 if len(hit) else len(a)
    keep = order[:k_star]
    mask = np.zeros((nb, nb), dtype=bool)
    mask[r[keep], c[keep]] = True
    mask[np.arange(nb), np.arange(nb)] = True
    values = np.zeros((nb, nb))
    values[r, c] = a
    cut = float(a[order[k_star - 1]]) if k_star < len(a) else 0.0
    return PESelection(mask, values, k_star, cut)


def pe_index(q: np.ndarray, k: np.ndarray, B: int, sm_scale: float, gamma: float) -> PESelection:
    return gamma_select(pooled_map(q, k, B, sm_scale), gamma)


# ------------------------------------------------------------------ Algorithm 1 (attention)

def vs_key_mask(rows: np.ndarray, n: int, sel_v: np.ndarray, sel_s: np.ndarray, B: int) -> np.ndarray:
    """Keys of each query under VS: j <= i with column block or offset block selected."""
    j = np.arange(n)[None, :]
    i = rows[:, None]
    off = i - j
    causal = off >= 0
    return causal & (sel_v[j // B] | sel_s[np.where(causal, off, 0) // B])


def pe_key_mask(rows: np.ndarray, n: int, mask: np.ndarray, B: int) -> np.ndarray:
    """Keys of each query under PE: j <= i with block (i//B, j//B) selected."""
    j = np.arange(n)[None, :]
    i = rows[:, None]
    return (j <= i) & mask[i // B, j // B]


def masked_attention(q_rows: np.ndarray, k: np.ndarray, v: np.ndarray, keymask: np.ndarray,
                     sm_scale: float) -> np.ndarray:
    """o_i = sum_{j in K_i} softmax_j(sm_scale q_i . k_j) v_j (exact, float64)."""
    s = sm_scale * (q_rows @ k.T)
    s[~keymask] = -np.inf
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    e[~keymask] = 0.0
    return (e @ v) / e.sum(axis=1, keepdims=True)


# ------------------------------------------------------------------ per head / per layer

@dataclasses.dataclass
class HeadIndex:
    c_struct: float
    route: int
    p_v: np.ndarray
    p_s: np.ndarray
    sel_v: np.ndarray
    sel_s: np.ndarray
    mu_v: float
    mu_s: float
    pe: Optional[PESelection]


def head_index(q: np.ndarray, k: np.ndarray, cfg: OracleCfg, with_pe: Optional[bool] = None) -> HeadIndex:
    """Algorithms 2-4 for one query head (q: [n, d], k: its KV head's [n, d]).

    ``with_pe``: compute the PE selection (default: only when routed PE).
    """
    n, d = q.shape
    B = cfg.block
    sc = cfg.scale(d)
    rows = proxy_rows(n, cfg.last_q)
    A = proxy_map(q[rows], k, rows, sc)
    c = c_struct(A, rows, cfg.w_sink, cfg.w_local)
    route = route_of(c, cfg.tau_proxy, cfg.force_route)
    a_v, a_s = directional_scores(A, rows)
    p_v, p_s = block_pool(a_v, B), block_pool(a_s, B)
    sel_v, sel_s, mu_v, mu_s = vs_index(p_v, p_s, cfg.alpha)
    pe = None
    if with_pe or (with_pe is None and route == PE):
        pe = pe_index(q, k, B, sc, cfg.gamma)
    return HeadIndex(c, route, p_v, p_s, sel_v, sel_s, mu_v, mu_s, pe)


def head_key_mask(idx: HeadIndex, rows: np.ndarray, n: int, B: int) -> np.ndarray:
    if idx.route == VS:
        return vs_key_mask(rows, n, idx.sel_v, idx.sel_s, B)
    return pe_key_mask(rows, n, idx.pe.mask, B)


def head_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, idx: HeadIndex, rows: np.ndarray,
                   cfg: OracleCfg, chunk: int = 256) -> np.ndarray:
    """Sparse attention output for the given query rows of one head ([S] Algorithm 1)."""
    n, d = q.shape
    out = np.empty((len(rows), v.shape[1]))
    for s0 in range(0, len(rows), chunk):
        rr = rows[s0:s0 + chunk]
        hi = int(rr.max()) + 1
        km = head_key_mask(idx, rr, hi, cfg.block)
        out[s0:s0 + len(rr)] = masked_attention(q[rr], k[:hi], v[:hi], km, cfg.scale(d))
    return out


def dense_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, rows: np.ndarray, sm_scale: float,
                    chunk: int = 256) -> np.ndarray:
    """Exact causal attention for the given rows (the dense reference)."""
    out = np.empty((len(rows), v.shape[1]))
    for s0 in range(0, len(rows), chunk):
        rr = rows[s0:s0 + chunk]
        hi = int(rr.max()) + 1
        km = np.arange(hi)[None, :] <= rr[:, None]
        out[s0:s0 + len(rr)] = masked_attention(q[rr], k[:hi], v[:hi], km, sm_scale)
    return out


def layer_index(get_q, get_k, h_q: int, h_kv: int, cfg: OracleCfg, with_pe=None,
                heads: Optional[List[int]] = None) -> Dict[int, HeadIndex]:
    """head_index for every (or the listed) query head. get_q(h) / get_k(g)
    return float64 [n, d] arrays; query head h reads KV head h // (h_q // h_kv)."""
    G = h_q // h_kv
    out = {}
    for h in (heads if heads is not None else range(h_q)):
        out[h] = head_index(get_q(h), get_k(h // G), cfg, with_pe)
    return out
