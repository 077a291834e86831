"""Pins for the CPU oracle, independent of the oracle's own code.

Each test checks the oracle against something the pages or mathematics fix:
brute-force enumeration on tiny inputs (scalar loops, not the oracle's
vectorised formulation), closed forms for uniform logits, a library routine
(torch's CPU scaled_dot_product_attention in float64) for the all-selected
case, hand-computed selections on exact binary fractions, and planted
structure. Source: CRISP summary page, Methodology -- Eq. (2), Eq. (3),
Eq. (4) and Algorithms 1-4.
"""
import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import crisp_oracle as O
import crisp_synth as S


# ---------------------------------------------------------------- brute force helpers

def brute_proxy(q, k, rows, scale):
    """A-hat as a dict {(i, j): prob} by scalar loops (math.exp)."""
    A = {}
    for i in rows:
        logits = [scale * sum(float(q[i, t]) * float(k[j, t]) for t in range(q.shape[1]))
                  for j in range(i + 1)]
        m = max(logits)
        w = [math.exp(x - m) for x in logits]
        z = sum(w)
        for j in range(i + 1):
            A[(i, j)] = w[j] / z
    return A


def brute_masses(A, rows, n, B, w_sink, w_local):
    nb = -(-n // B)
    nq = len(rows)
    p_v = [0.0] * nb
    p_s = [0.0] * nb
    c = 0.0
    for (i, j), a in A.items():
        p_v[j // B] += a / nq
        p_s[(i - j) // B] += a / nq
        if j < w_sink or 0 <= i - j < w_local:
            c += a / nq
    return np.array(p_v), np.array(p_s), c


SMALL = O.OracleCfg(block=16, last_q=16, w_sink=16, w_local=16, tau_proxy=0.1, alpha=1.0, gamma=0.9)


@pytest.mark.parametrize("n,d,seed", [(200, 8, 1), (160, 16, 2), (64, 4, 3)])
def test_proxy_masses_and_cstruct_vs_brute_force(n, d, seed):
    r = np.random.default_rng(seed)
    q = r.standard_normal((n, d)) * 1.5
    k = r.standard_normal((n, d))
    k[3] += 4.0 * q[-16:].mean(axis=0)     # some structure so masses are uneven
    cfg = SMALL
    idx = O.head_index(q, k, cfg)
    rows = list(range(n - cfg.last_q, n))
    A = brute_proxy(q, k, rows, 1.0 / math.sqrt(d))
    p_v, p_s, c = brute_masses(A, rows, n, cfg.block, cfg.w_sink, cfg.w_local)
    np.testing.assert_allclose(idx.p_v, p_v, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(idx.p_s, p_s, rtol=1e-12, atol=1e-14)
    assert abs(idx.c_struct - c) < 1e-12
    # invariants: each direction is a distribution, C_struct in [0, 1]
    assert abs(idx.p_v.sum() - 1) < 1e-12 and abs(idx.p_s.sum() - 1) < 1e-12
    assert 0.0 <= idx.c_struct <= 1.0


def test_proxy_map_rows_are_causal_softmax():
    r = np.random.default_rng(5)
    n, d = 96, 8
    q, k = r.standard_normal((n, d)), r.standard_normal((n, d))
    rows = O.proxy_rows(n, 16)
    A = O.proxy_map(q[rows], k, rows, 0.3)
    Ab = brute_proxy(q, k, list(rows), 0.3)
    for a, i in enumerate(rows):
        for j in range(n):
            want = Ab.get((i, j), 0.0)
            assert abs(A[a, j] - want) < 1e-13


# ---------------------------------------------------------------- closed forms (uniform logits)

def _uniform_closed_forms(n, B, last_q, w_sink, w_local):
    rows = range(n - last_q, n)
    nb = -(-n // B)
    p_v = [Fraction(0)] * nb
    p_s = [Fraction(0)] * nb
    c = Fraction(0)
    for i in rows:
        w = Fraction(1, (i + 1) * last_q)     # A-hat[i, j] = 1/(i+1) for j <= i
        for b in range(nb):
            lo, hi = b * B, min(n, (b + 1) * B) - 1
            p_v[b] += w * max(0, min(hi, i) - lo + 1)        # keys of block b that are <= i
            p_s[b] += w * max(0, min(hi, i) - lo + 1)        # offsets of block b that are <= i
        anchor = set(range(min(w_sink, i + 1))) | set(range(max(0, i - w_local + 1), i + 1))
        c += w * len(anchor)
    return p_v, p_s, c


@pytest.mark.parametrize("n,B,last_q,ws,wl", [(1024, 128, 64, 128, 128), (200, 16, 16, 16, 16),
                                              (300, 64, 64, 64, 128), (96, 32, 64, 64, 64)])
def test_uniform_logits_closed_form(n, B, last_q, ws, wl):
    d = 8
    q = np.zeros((n, d))
    k = np.random.default_rng(0).standard_normal((n, d))
    cfg = O.OracleCfg(block=B, last_q=last_q, w_sink=ws, w_local=wl)
    idx = O.head_index(q, k, cfg)
    p_v, p_s, c = _uniform_closed_forms(n, B, last_q, ws, wl)
    np.testing.assert_allclose(idx.p_v, [float(x) for x in p_v], rtol=1e-12)
    np.testing.assert_allclose(idx.p_s, [float(x) for x in p_s], rtol=1e-12)
    assert abs(idx.c_struct - float(c)) < 1e-12


def test_uniform_logits_sit_exactly_on_the_noise_floor():
    """Uniform rows: every middle block has p_j = mu (exact arithmetic), so the
    strict '>' of Eq. (4) keeps none of them; alpha just below 1 keeps all."""
    n, B = 1024, 128
    q = np.zeros((n, 8))
    k = np.random.default_rng(1).standard_normal((n, 8))
    p_v, _, _ = _uniform_closed_forms(n, B, 64, 128, 128)
    nb = len(p_v)
    mu = (1 - p_v[0] - p_v[-1]) / (nb - 2)
    assert all(p_v[b] == mu for b in range(1, nb - 1))          # exact rational identity
    base = O.head_index(q, k, O.OracleCfg())
    assert np.allclose(base.p_v[1:-1], base.mu_v, rtol=1e-12)
    hi = O.head_index(q, k, O.OracleCfg(alpha=1 + 1e-9))
    lo = O.head_index(q, k, O.OracleCfg(alpha=1 - 1e-9))
    assert hi.sel_v.tolist() == [True] + [False] * (nb - 2) + [True]
    assert lo.sel_v.all()
    # route closed form: C = mean_i 256/(i+1) ~ 0.258 at n=1024 -> VS at tau=0.1 ...
    assert hi.route == O.VS and abs(hi.c_struct - 0.258) < 1e-3
    # ... and ~0.0627 at n=4096 -> PE
    q4 = np.zeros((4096, 8))
    k4 = np.random.default_rng(2).standard_normal((4096, 8))
    u4 = O.head_index(q4, k4, O.OracleCfg(), with_pe=False)
    assert u4.route == O.PE and abs(u4.c_struct - 0.0627) < 1e-3


# ---------------------------------------------------------------- selection on exact fractions

def test_threshold_blocks_hand_values():
    p = np.array([0.5, 0.0625, 0.125, 0.0625, 0.25])
    sel, mu = O.threshold_blocks(p, 0, 4, 1.0)
    assert mu == 0.25 / 3
    assert sel.tolist() == [True, False, True, False, True]


def test_threshold_blocks_strict_inequality_and_alpha():
    p = np.array([0.25, 0.125, 0.125, 0.125, 0.125, 0.25])   # mu = 0.125 exactly
    sel, mu = O.threshold_blocks(p, 0, 5, 1.0)
    assert mu == 0.125 and sel.tolist() == [True, False, False, False, False, True]
    sel, _ = O.threshold_blocks(p, 0, 5, 0.5)
    assert sel.all()
    sel, _ = O.threshold_blocks(p, 0, 5, 1e9)
    assert sel.tolist() == [True, False, False, False, False, True]


def test_noise_floor_clamps_at_zero_and_small_nb():
    p = np.array([0.7, 0.0, 0.1, 0.4])   # 1 - 0.7 - 0.4 < 0 -> mu = 0
    sel, mu = O.threshold_blocks(p, 0, 3, 1.0)
    assert mu == 0.0 and sel.tolist() == [True, False, True, True]
    sel, _ = O.threshold_blocks(np.array([0.3, 0.7]), 0, 1, 1.0)
    assert sel.all()


def test_vs_index_diagonal_direction_uses_offset_blocks_ends():
    # diagonal direction: retained ends are offset block N_b-1 and offset block 0
    p_v = np.array([0.5, 0.1, 0.1, 0.3])
    p_s = np.array([0.6, 0.05, 0.3, 0.05])   # mu_s = (1 - 0.6 - 0.05)/2 = 0.175
    sel_v, sel_s, mu_v, mu_s = O.vs_index(p_v, p_s, 1.0)
    assert abs(mu_s - 0.175) < 1e-15
    assert sel_s.tolist() == [True, False, True, True]
    assert abs(mu_v - 0.1) < 1e-15
    assert sel_v.tolist() == [True, False, False, True]


def test_all_mass_on_sink_routes_vs_and_keeps_only_retained_blocks():
    n, d = 1024, 16
    r = np.random.default_rng(3)
    q = np.tile(r.standard_normal(d), (n, 1))
    k = 0.01 * r.standard_normal((n, d))
    k[0] = 4000.0 * q[0] / np.dot(q[0], q[0])      # sink logit ~ 1000 above the rest
    idx = O.head_index(q, k, O.OracleCfg())
    assert idx.c_struct == pytest.approx(1.0, abs=1e-12)
    assert idx.route == O.VS
    assert idx.mu_v == 0.0
    nb = n // 128
    assert idx.sel_v.tolist() == [True] + [False] * (nb - 2) + [True]


# ---------------------------------------------------------------- PE (Algorithm 4)

def brute_pe(q, k, B, scale, gamma):
    n, d = q.shape
    nb = -(-n // B)
    def bmean(x, b):
        rows = range(b * B, min(n, (b + 1) * B))
        return [sum(float(x[i, t]) for i in rows) / len(rows) for t in range(d)]
    qb = [bmean(q, b) for b in range(nb)]
    kb = [bmean(k, b) for b in range(nb)]
    entries = []
    for r_ in range(nb):
        lg = [scale * sum(qb[r_][t] * kb[c][t] for t in range(d)) for c in range(r_ + 1)]
        m = max(lg)
        w = [math.exp(x - m) for x in lg]
        z = sum(w)
        for c in range(r_ + 1):
            entries.append((w[c] / z, r_ * nb + c))
    tot = sum(v for v, _ in entries)
    entries = [(v / tot, f) for v, f in entries]
    entries.sort(key=lambda t: (-t[0], t[1]))
    keep, acc = [], 0.0
    for v, f in entries:
        keep.append(f)
        acc += v
        if gamma < 1.0 and acc >= gamma:
            break
    mask = np.zeros((nb, nb), dtype=bool)
    for f in keep:
        mask[f // nb, f % nb] = True
    for r_ in range(nb):
        mask[r_, r_] = True
    return mask


@pytest.mark.parametrize("n,B,gamma,seed", [(96, 16, 0.9, 0), (100, 16, 0.5, 1), (64, 8, 0.95, 2), (48, 16, 1.0, 3)])
def test_pe_index_vs_brute_force(n, B, gamma, seed):
    r = np.random.default_rng(seed)
    d = 6
    q, k = 3 * r.standard_normal((n, d)), 3 * r.standard_normal((n, d))
    sel = O.pe_index(q, k, B, 1 / math.sqrt(d), gamma)
    assert (sel.mask == brute_pe(q, k, B, 1 / math.sqrt(d), gamma)).all()


def test_gamma_select_hand_built_ties_and_diagonal():
    abar = np.array([[1.0, 0, 0], [0.75, 0.25, 0], [0.5, 0.25, 0.25]])
    # normalised: 1/3, 1/4, 1/12 | 1/6, 1/12, 1/12 ; ties at 1/12 broken by flat index 4 < 7 < 8
    s = O.gamma_select(abar, 0.8)
    assert s.k_star == 4
    assert s.mask.tolist() == [[True, False, False], [True, True, False], [True, False, True]]
    s = O.gamma_select(abar, 0.7)
    assert s.k_star == 3
    assert s.mask.tolist() == [[True, False, False], [True, True, False], [True, False, True]]
    s = O.gamma_select(abar, 1.0)
    assert s.mask[np.tril_indices(3)].all()


def test_pooled_map_is_block_causal_row_softmax():
    r = np.random.default_rng(9)
    q, k = r.standard_normal((70, 4)), r.standard_normal((70, 4))
    A = O.pooled_map(q, k, 16, 0.5)
    assert A.shape == (5, 5)
    assert np.allclose(A.sum(axis=1), 1.0) and (np.triu(A, 1) == 0).all()
    # short tail block averages its 6 rows only
    assert np.allclose(O.block_mean(q, 16)[4], q[64:].mean(axis=0))


# ---------------------------------------------------------------- attention (Algorithm 1)

def brute_attention(q, k, v, i, keys, scale):
    lg = [scale * sum(float(q[i, t]) * float(k[j, t]) for t in range(q.shape[1])) for j in keys]
    m = max(lg)
    w = [math.exp(x - m) for x in lg]
    z = sum(w)
    return np.array([sum(w[a] * float(v[j, t]) for a, j in enumerate(keys)) / z for t in range(v.shape[1])])


def test_vs_sparse_attention_vs_brute_force():
    r = np.random.default_rng(11)
    n, d, B = 48, 4, 8
    q, k, v = r.standard_normal((n, d)), r.standard_normal((n, d)), r.standard_normal((n, d))
    nb = n // B
    sel_v = np.array([True, False, True, False, False, True])
    sel_s = np.array([True, False, False, True, False, False])
    idx = O.HeadIndex(0.5, O.VS, None, None, sel_v, sel_s, 0, 0, None)
    rows = np.arange(n)
    cfg = O.OracleCfg(block=B)
    out = O.head_attention(q, k, v, idx, rows, cfg)
    for i in range(n):
        keys = [j for j in range(i + 1) if sel_v[j // B] or sel_s[(i - j) // B]]
        np.testing.assert_allclose(out[i], brute_attention(q, k, v, i, keys, 0.5), rtol=1e-12, atol=1e-13)
    assert nb == 6


def test_pe_sparse_attention_vs_brute_force():
    r = np.random.default_rng(12)
    n, d, B = 40, 4, 8
    q, k, v = r.standard_normal((n, d)), r.standard_normal((n, d)), r.standard_normal((n, d))
    nb = n // B
    mask = np.tril(r.random((nb, nb)) < 0.5)
    mask[np.arange(nb), np.arange(nb)] = True
    pe = O.PESelection(mask, None, 0, 0.0)
    idx = O.HeadIndex(0.0, O.PE, None, None, None, None, 0, 0, pe)
    cfg = O.OracleCfg(block=B)
    out = O.head_attention(q, k, v, idx, np.arange(n), cfg)
    for i in range(n):
        keys = [j for j in range(i + 1) if mask[i // B, j // B]]
        np.testing.assert_allclose(out[i], brute_attention(q, k, v, i, keys, 0.5), rtol=1e-12, atol=1e-13)


def test_all_selected_equals_library_dense_causal_attention():
    import torch
    r = np.random.default_rng(13)
    n, d = 384, 32
    q, k, v = r.standard_normal((n, d)), r.standard_normal((n, d)), r.standard_normal((n, d))
    nb = n // 128
    vs = O.HeadIndex(0.0, O.VS, None, None, np.ones(nb, bool), np.zeros(nb, bool), 0, 0, None)
    pe = O.HeadIndex(0.0, O.PE, None, None, None, None, 0, 0,
                     O.PESelection(np.tril(np.ones((nb, nb), bool)), None, 0, 0.0))
    cfg = O.OracleCfg()
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None], torch.from_numpy(v)[None, None],
        is_causal=True)[0, 0].numpy()
    for idx in (vs, pe):
        out = O.head_attention(q, k, v, idx, np.arange(n), cfg)
        np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(O.dense_attention(q, k, v, np.arange(n), 1 / math.sqrt(d)), ref, rtol=1e-10, atol=1e-12)
    # alpha -> 0+: VS selection keeps every block with positive mass (all of them here)
    idx = O.head_index(q, k, O.OracleCfg(alpha=1e-300, force_route=O.VS))
    assert idx.sel_v.all() and idx.sel_s.all()


def test_gamma_one_keeps_every_causal_block():
    r = np.random.default_rng(14)
    q, k = r.standard_normal((512, 16)), r.standard_normal((512, 16))
    s = O.pe_index(q, k, 64, 0.25, 1.0)
    assert s.mask[np.tril_indices(8)].all() and not np.triu(s.mask, 1).any()


# ---------------------------------------------------------------- planted structure (synthetic layers)

def _f64(layer, which, h):
    return layer.as_f64(which, h)


def test_planted_structure_is_selected_and_gaussian_heads_route_pe():
    cfg = S.scaled("B", n=4096, h_q=8, h_kv=2)
    layer = S.generate(cfg, with_v=False)
    st = layer.structure[0]
    oc = O.OracleCfg()
    for h in range(cfg.h_q):
        idx = O.head_index(_f64(layer, "q", h), _f64(layer, "k", h // cfg.group), oc, with_pe=False)
        if h // cfg.group in cfg.planted_groups:
            assert idx.route == O.VS, (h, idx.c_struct)
            assert idx.c_struct > 0.4
            for j in st.verticals:
                assert idx.sel_v[j // 128], (h, j)
            for o in st.slash_offsets:
                assert idx.sel_s[o // 128], (h, o)
            assert idx.sel_v[0]
        else:
            assert idx.route == O.PE, (h, idx.c_struct)
            assert idx.c_struct < 0.1


def test_config_a_planted_selection_under_forced_vs():
    cfg = S.CONFIGS["A"]
    layer = S.generate(cfg, with_v=False)
    st = layer.structure[0]
    idx = O.head_index(_f64(layer, "q", 0), _f64(layer, "k", 0), O.OracleCfg(force_route=O.VS))
    assert idx.route == O.VS
    for j in st.verticals:
        assert idx.sel_v[j // 128]
    for o in st.slash_offsets:
        assert idx.sel_s[o // 128]
    auto = O.head_index(_f64(layer, "q", 0), _f64(layer, "k", 0), O.OracleCfg(), with_pe=False)
    assert 0.0 < auto.c_struct < 0.2
