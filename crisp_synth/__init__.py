"""Seeded synthetic attention-layer inputs for CRISP sparse prefill.

This module only draws and lays out numbers. It holds none of the method's
arithmetic (no scores, softmax, masses, thresholds or selection), so both the
CPU oracle and the CUDA path may take their inputs from it.

The pages measure on InfiniteBench / RULER / LongBench prompts run through
Llama-3.1-8B and Qwen2.5-7B ("CRISP: Cliff-awaRe Input-adaptive Sparse
Prefilling", summary page, Introduction and Results). Neither the datasets nor
the weights are available, so these generators stand in for them: they take
only the models' head counts and head dimension and plant the structures the
pages name (architectural sinks, vertical columns, slash diagonals; summary
page, Introduction, "Theoretical Basis") into otherwise iid Gaussian heads.

Recipe (all randomness from numpy PCG64 seeded by
``SeedSequence([0, config_id, group_or_head, tensor_id])``):

* Q, K, V ~ N(0, 1) per element, drawn in float32 (float64 for the planted
  components), then rounded to bfloat16 (round-to-nearest-even) for the bf16
  layers. V is always plain N(0, 1).
* GQA: query head h reads KV head ``h // (h_q // h_kv)``. Structure is planted
  per KV group, so every query head of a planted group sees it.
* Planted group g: the head dimension is split in two halves. The first
  half carries only the slash structure; the second carries the Gaussian
  noise and a unit vector u. The noise of K (and of the group's Q heads) is
  projected off u, then every query gets ``+a*u`` with ``a = d**0.25``. A key
  that gets ``+c*a*u`` then gains exactly ``c`` logits (after the 1/sqrt(d)
  scale) against every query of the group.
  - sink: key 0 gets ``sink_logits`` extra logits;
  - verticals: ``n_vert`` distinct keys drawn uniformly in blocks
    1 .. N_b-2 get +4 logits;
  - slashes: the layer's ``n_slash`` offsets are dealt round-robin to the
    layer's planted groups. Every position p gets a seeded random unit code
    c_p in the slash half; query i gets ``s * c_i`` and key j gets
    ``s * sum_t c_{j + o_t}`` with ``s**2 = 4*sqrt(d)``. The score then
    gains exactly +4 logits wherever ``i - j = o_t``, and elsewhere a small
    zero-mean term that is independent from one (i, j) pair to the next, so
    it averages out over a block. Offsets are distinct, uniform in [B, n/2).
    (A rotary-position version of the same idea makes that off-peak term a
    function of i - j alone; with several slashes at d = 128 it then tilts
    whole blocks by more than a planted +4-logit key lifts one.)
* Gaussian groups: plain N(0, 1); ``gauss_q_scale`` multiplies Q (2.0 is a
  softmax temperature of 0.5).
* The sink strength for the bf16 layers is set so the sink carries a fraction
  f of a row's mass against the Gaussian background:
  ``sink_logits = ln(f/(1-f)) + ln(n-1) + 1/2``.
* Mass-cliff background (``cliff_sigma`` > 0): the pages' premise is that
  real attention mass falls off a cliff, a few blocks holding most of it
  (summary page, "Theoretical Basis"), which an iid Gaussian background
  lacks. Every KV group then draws a per-key-block logit offset
  ``beta_b = cliff_sigma * z_b`` (z_b ~ N(0, 1), seeded per group) for the
  blocks 1 .. N_b-2; the sink block and the last block keep beta = 0. It
  is planted like the sink: along u in planted groups, along a seeded unit
  vector w (Q and K noise projected off w, every query ``+a*w``) in the
  other groups, so every key of block b gains exactly beta_b logits against
  every query of the group. Block masses are then log-normal with
  log-standard-deviation cliff_sigma. The sink logits add ``cliff_sigma**2/2``
  (the background's mean mass factor) to keep the sink's share.
"""
from __future__ import annotations

import dataclasses
import math
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, List, Optional, Sequence

import numpy as np

BLOCK = 128

# tensor ids for the seed sequence
_T_Q, _T_K, _T_V, _T_STRUCT, _T_CODES, _T_CLIFF = 0, 1, 2, 3, 4, 5


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    config_id: int
    h_q: int
    h_kv: int
    n: int
    d: int
    dtype: str                      # "fp32" or "bf16"
    planted_groups: tuple           # KV groups with planted VS structure
    n_vert: int
    n_slash: int
    sink_logits: float              # extra logits on key 0 in planted groups
    gauss_q_scale: float = 1.0      # Q multiplier on Gaussian groups
    desc: str = ""
    slash_groups: int = 0           # groups the layer's slashes are dealt over (0: planted count)
    cliff_sigma: float = 0.0        # log-normal block background (0: iid Gaussian background)

    @property
    def n_blocks(self) -> int:
        return -(-self.n // BLOCK)

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv


def sink_logits_for_fraction(f: float, n: int, cliff_sigma: float = 0.0) -> float:
    """Extra sink logits so the sink holds fraction f of a Gaussian row's mass
    (with a log-normal block background of log-sd cliff_sigma when given)."""
    return math.log(f / (1.0 - f)) + math.log(n - 1) + 0.5 + 0.5 * cliff_sigma ** 2


def _llama(name, cid, n, n_vert, n_slash, desc, cliff_sigma=0.0):
    return LayerConfig(name, cid, 32, 8, n, 128, "bf16", tuple(range(6)), n_vert, n_slash,
                       sink_logits_for_fraction(0.5, n, cliff_sigma), 1.0, desc, cliff_sigma=cliff_sigma)


CONFIGS: Dict[str, LayerConfig] = {
    "A": LayerConfig("A", 0, 1, 1, 4096, 128, "fp32", (0,), 8, 4, 4.0, 1.0,
                     "1 head, n=4096, d=128, fp32, planted sink + 8 verticals + 4 slashes"),
    "B": _llama("B", 1, 32768, 16, 8, "Llama-3.1-8B-shaped 32Q/8KV, n=32768, bf16"),
    "C": _llama("C", 2, 131072, 64, 16, "Llama-3.1-8B-shaped 32Q/8KV, n=131072, bf16"),
    "D": LayerConfig("D", 3, 28, 4, 131072, 128, "bf16", (0, 1), 64, 8,
                     sink_logits_for_fraction(0.9, 131072), 2.0,
                     "Qwen2.5-7B-shaped 28Q/4KV, n=131072, bf16, half VS (sink 90%), half T=0.5"),
    "E": _llama("E", 4, 524288, 128, 32, "Llama-3.1-8B-shaped 32Q/8KV, n=524288, bf16"),
    # mass-cliff background (log-normal block masses, log-sd 2) on the shapes of C and E
    "C_cliff": _llama("C_cliff", 5, 131072, 64, 16,
                      "Llama-3.1-8B-shaped 32Q/8KV, n=131072, bf16, log-normal block background (sigma 2)",
                      cliff_sigma=2.0),
    "E_cliff": _llama("E_cliff", 6, 524288, 128, 32,
                      "Llama-3.1-8B-shaped 32Q/8KV, n=524288, bf16, log-normal block background (sigma 2)",
                      cliff_sigma=2.0),
}


def scaled(base: str, *, n: Optional[int] = None, h_q: Optional[int] = None,
           h_kv: Optional[int] = None, planted_groups: Optional[Sequence[int]] = None,
           n_vert: Optional[int] = None, n_slash: Optional[int] = None,
           dtype: Optional[str] = None, config_id: Optional[int] = None) -> LayerConfig:
    """A smaller layer with the same recipe as ``base`` (for fast parity cases)."""
    c = CONFIGS[base]
    n2 = n if n is not None else c.n
    h_q2 = h_q if h_q is not None else c.h_q
    h_kv2 = h_kv if h_kv is not None else c.h_kv
    if planted_groups is not None:
        pg = tuple(planted_groups)
    else:
        frac = len(c.planted_groups) / c.h_kv
        npl = int(round(h_kv2 * frac))
        npl = max(1, min(npl, h_kv2 - 1)) if h_kv2 >= 2 else 1
        pg = tuple(range(npl))
    sink = c.sink_logits
    if c.dtype == "bf16":
        f = 0.9 if base == "D" else 0.5
        sink = sink_logits_for_fraction(f, n2, c.cliff_sigma)
    nb = -(-n2 // BLOCK)
    # keep the density of verticals per block of the full-size layer
    nv = n_vert if n_vert is not None else min(max(1, round(c.n_vert * n2 / c.n)), max(nb - 2, 0))
    ns = n_slash if n_slash is not None else c.n_slash
    return dataclasses.replace(
        c, name=f"{base}[n={n2},h={h_q2}/{h_kv2}]", n=n2, h_q=h_q2, h_kv=h_kv2,
        planted_groups=pg, n_vert=nv, n_slash=ns, sink_logits=sink,
        dtype=dtype or c.dtype, slash_groups=len(c.planted_groups),
        config_id=config_id if config_id is not None else 100 + c.config_id)


# --------------------------------------------------------------------------- helpers

def _rng(cfg: LayerConfig, unit: int, tensor: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([0, cfg.config_id, unit, tensor])))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest-even) and return the 16-bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bit patterns to float32."""
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class GroupStructure:
    group: int
    u: np.ndarray                # [d] unit
    verticals: np.ndarray        # sorted key positions
    slash_offsets: np.ndarray    # sorted offsets


def slash_dims(d: int) -> int:
    """Leading head dimensions reserved for the slash structure in planted groups."""
    return d // 2


def slash_count(cfg: LayerConfig, g: int) -> int:
    """Slash offsets of planted group g: the layer's count dealt round-robin."""
    pg = list(cfg.planted_groups)
    if g not in pg:
        return 0
    k = pg.index(g)
    ng = cfg.slash_groups or len(pg)
    return cfg.n_slash // ng + (1 if k < cfg.n_slash % ng else 0)


def group_structure(cfg: LayerConfig, g: int) -> GroupStructure:
    """Seeded planted positions and directions of KV group g."""
    r = _rng(cfg, g, _T_STRUCT)
    d = cfg.d
    ds = slash_dims(d)
    u = np.zeros(d)
    u[ds:] = r.standard_normal(d - ds)
    u /= np.linalg.norm(u)
    nb = cfg.n_blocks
    lo, hi = BLOCK, max(BLOCK, (nb - 1) * BLOCK)
    nvert = min(cfg.n_vert, hi - lo)
    verts = np.sort(r.choice(np.arange(lo, hi), size=nvert, replace=False)) if nvert > 0 else np.zeros(0, np.int64)
    shi = max(BLOCK + 1, cfg.n // 2)
    nsl = min(slash_count(cfg, g), shi - BLOCK)
    offs = np.sort(r.choice(np.arange(BLOCK, shi), size=nsl, replace=False)) if nsl > 0 else np.zeros(0, np.int64)
    return GroupStructure(g, u, verts.astype(np.int64), offs.astype(np.int64))


def position_codes(cfg: LayerConfig, g: int, count: int) -> np.ndarray:
    """Seeded unit codes c_p (float32, [count, d/2]) of planted group g."""
    r = _rng(cfg, g, _T_CODES)
    c = r.standard_normal((count, slash_dims(cfg.d)), dtype=np.float32)
    c /= np.linalg.norm(c, axis=1, keepdims=True)
    return c


def cliff_offsets(cfg: LayerConfig, g: int):
    """Seeded (w, beta) of KV group g's mass-cliff background: w a unit
    direction (used by groups without planted structure), beta [N_b] the
    per-key-block logit offsets (zero for the first and last block)."""
    r = _rng(cfg, g, _T_CLIFF)
    w = r.standard_normal(cfg.d)
    w /= np.linalg.norm(w)
    nb = cfg.n_blocks
    beta = cfg.cliff_sigma * r.standard_normal(nb)
    beta[0] = 0.0
    beta[nb - 1] = 0.0
    return w, beta


def _key_offsets(cfg: LayerConfig, beta: np.ndarray) -> np.ndarray:
    """Per-key logit offset: beta of the key's block."""
    return np.repeat(beta, BLOCK)[: cfg.n]


def _project_off(x: np.ndarray, u: np.ndarray) -> None:
    x -= np.outer(x @ u, u).astype(x.dtype)


def _gen_k(cfg: LayerConfig, g: int, st: Optional[GroupStructure]) -> np.ndarray:
    n, d = cfg.n, cfg.d
    k = _rng(cfg, g, _T_K).standard_normal((n, d), dtype=np.float32)
    a = d ** 0.25
    if st is None:
        if cfg.cliff_sigma > 0:
            w, beta = cliff_offsets(cfg, g)
            w32 = w.astype(np.float32)
            _project_off(k, w32)
            k += (a * _key_offsets(cfg, beta))[:, None].astype(np.float32) * w32[None, :]
        return k
    k[:, : slash_dims(d)] = 0.0
    _project_off(k, st.u.astype(np.float32))
    # sink: +sink_logits against every query of the group
    k[0] += (cfg.sink_logits * math.sqrt(d) / a * st.u).astype(np.float32)
    k[st.verticals] += (4.0 * a * st.u).astype(np.float32)
    if cfg.cliff_sigma > 0:
        _, beta = cliff_offsets(cfg, g)
        k += (a * _key_offsets(cfg, beta))[:, None].astype(np.float32) * st.u.astype(np.float32)[None, :]
    if len(st.slash_offsets):
        s = np.float32(math.sqrt(4.0 * math.sqrt(d)))
        codes = position_codes(cfg, st.group, n + int(st.slash_offsets.max()))
        ds = slash_dims(d)
        for o in st.slash_offsets:
            k[:, :ds] += s * codes[o:o + n]
    return k


def _gen_q(cfg: LayerConfig, h: int, st: Optional[GroupStructure]) -> np.ndarray:
    n, d = cfg.n, cfg.d
    q = _rng(cfg, 1000 + h, _T_Q).standard_normal((n, d), dtype=np.float32)
    if st is None:
        if cfg.cliff_sigma > 0:
            w, _ = cliff_offsets(cfg, h // cfg.group)
            w32 = w.astype(np.float32)
            _project_off(q, w32)
            q += (d ** 0.25 * w32)[None, :]
        if cfg.gauss_q_scale != 1.0:
            q *= np.float32(cfg.gauss_q_scale)
        return q
    a = d ** 0.25
    q[:, : slash_dims(d)] = 0.0
    _project_off(q, st.u.astype(np.float32))
    q += (a * st.u).astype(np.float32)[None, :]
    if len(st.slash_offsets):
        s = np.float32(math.sqrt(4.0 * math.sqrt(d)))
        q[:, : slash_dims(d)] += s * position_codes(cfg, st.group, n)
    return q


def _gen_v(cfg: LayerConfig, g: int) -> np.ndarray:
    return _rng(cfg, g, _T_V).standard_normal((cfg.n, cfg.d), dtype=np.float32)


@dataclasses.dataclass
class Layer:
    """One synthetic attention layer, head-major: q [h_q, n, d], k/v [h_kv, n, d].

    For bf16 layers the arrays hold bfloat16 bit patterns (uint16); for fp32
    layers they hold float32.
    """
    cfg: LayerConfig
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    structure: Dict[int, GroupStructure]

    def as_f64(self, which: str, head: int) -> np.ndarray:
        a = getattr(self, which)[head]
        if self.cfg.dtype == "bf16":
            return bf16_bits_to_f32(a).astype(np.float64)
        return a.astype(np.float64)

    def rows_f64(self, which: str, head: int, rows) -> np.ndarray:
        a = getattr(self, which)[head][rows]
        if self.cfg.dtype == "bf16":
            return bf16_bits_to_f32(a).astype(np.float64)
        return a.astype(np.float64)

    @property
    def planted_q_heads(self) -> List[int]:
        G = self.cfg.group
        return [h for h in range(self.cfg.h_q) if h // G in self.cfg.planted_groups]

    @property
    def gaussian_q_heads(self) -> List[int]:
        G = self.cfg.group
        return [h for h in range(self.cfg.h_q) if h // G not in self.cfg.planted_groups]


def generate(cfg: LayerConfig, threads: int = 8, with_v: bool = True) -> Layer:
    """Draw the whole layer. Deterministic for a given config."""
    h_q, h_kv, n, d = cfg.h_q, cfg.h_kv, cfg.n, cfg.d
    bf16 = cfg.dtype == "bf16"
    st = {g: group_structure(cfg, g) for g in cfg.planted_groups}
    dt = np.uint16 if bf16 else np.float32
    q = np.empty((h_q, n, d), dtype=dt)
    k = np.empty((h_kv, n, d), dtype=dt)
    v = np.empty((h_kv, n, d), dtype=dt) if with_v else np.zeros((h_kv, 0, d), dtype=dt)
    G = cfg.group

    def store(dst, i, x):
        dst[i] = f32_to_bf16_bits(x) if bf16 else x

    jobs = []
    for g in range(h_kv):
        jobs.append(lambda g=g: store(k, g, _gen_k(cfg, g, st.get(g))))
        if with_v:
            jobs.append(lambda g=g: store(v, g, _gen_v(cfg, g)))
    for h in range(h_q):
        jobs.append(lambda h=h: store(q, h, _gen_q(cfg, h, st.get(h // G))))
    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        for f in [ex.submit(j) for j in jobs]:
            f.result()
    return Layer(cfg, q, k, v, st)


def generate_slice(cfg: LayerConfig, g_lo: int, g_hi: int, threads: int = 8, with_v: bool = True):
    """KV groups [g_lo, g_hi) of the layer and their query heads, exactly as
    the same rows of ``generate(cfg)``: (q [(g_hi-g_lo)*G, n, d], k, v
    [g_hi-g_lo, n, d]) in the layer's storage type. Every tensor is drawn from
    its own seed, so a rank can draw only its shard."""
    if not 0 <= g_lo < g_hi <= cfg.h_kv:
        raise ValueError("bad group range")
    n, d, G = cfg.n, cfg.d, cfg.group
    bf16 = cfg.dtype == "bf16"
    st = {g: group_structure(cfg, g) for g in cfg.planted_groups if g_lo <= g < g_hi}
    dt = np.uint16 if bf16 else np.float32
    ng = g_hi - g_lo
    q = np.empty((ng * G, n, d), dtype=dt)
    k = np.empty((ng, n, d), dtype=dt)
    v = np.empty((ng, n, d), dtype=dt) if with_v else np.zeros((ng, 0, d), dtype=dt)

    def store(dst, i, x):
        dst[i] = f32_to_bf16_bits(x) if bf16 else x

    jobs = []
    for g in range(g_lo, g_hi):
        jobs.append(lambda g=g: store(k, g - g_lo, _gen_k(cfg, g, st.get(g))))
        if with_v:
            jobs.append(lambda g=g: store(v, g - g_lo, _gen_v(cfg, g)))
        for h in range(g * G, (g + 1) * G):
            jobs.append(lambda h=h, g=g: store(q, h - g_lo * G, _gen_q(cfg, h, st.get(g))))
    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        for f in [ex.submit(j) for j in jobs]:
            f.result()
    return q, k, v


def to_torch(layer: Layer):
    """(q, k, v) as CPU torch tensors of the layer's dtype (views, no copy)."""
    import torch
    if layer.cfg.dtype == "bf16":
        return tuple(torch.from_numpy(a).view(torch.bfloat16) for a in (layer.q, layer.k, layer.v))
    return tuple(torch.from_numpy(a) for a in (layer.q, layer.k, layer.v))
