"""Comparison rules between the CUDA path and the CPU oracle.

* Routes: bit-exact, except a head whose C_struct lies within 1e-3 relative
  of tau_proxy, which is reported as a flip.
* VS masks: bit-exact, except a block whose oracle mass lies within 1e-3
  relative of alpha*mu (a flip).
* PE masks: bit-exact, except an entry whose oracle value lies within 1e-3
  relative of the oracle's cut value, or whose place in the oracle's sorted
  order has a cumulative mass (of the entries before it) within 1e-3
  relative of gamma: Algorithm 4's threshold is gamma on that cumulative sum,
  so an entry sitting on it (for instance when whole rows' mass adds up to
  gamma exactly) is decided by rounding either way (a flip).
* Outputs on the same indices: two normalisations of the max error, each
  within 2e-2 (bf16) or 1e-4 (fp32):
  - per head: max |o - o_ref| / max |o_ref| over the head's checked rows;
  - per row: max over rows of max_c |o - o_ref| / max_c |o_ref| (a row with a
    small output is measured against its own size, not the head's largest).
* Flip counts are reported per head and kind, and bounded: at most 1% of a
  head's VS blocks (2 N_b) or of its causal PE blocks.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List

import numpy as np

REL_FLIP = 1e-3
FLIP_FRAC_MAX = 0.01
TOL = {"bf16": 2e-2, "fp32": 1e-4}


def unpack_mask(words: np.ndarray, nbits: int) -> np.ndarray:
    """uint32 words (..., W) -> bool (..., nbits); bit b in word b//32, position b%32."""
    w = np.ascontiguousarray(words).astype(np.uint32)
    bits = ((w[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool)
    return bits.reshape(*w.shape[:-1], w.shape[-1] * 32)[..., :nbits]


def pack_mask(bits: np.ndarray) -> np.ndarray:
    """bool (..., nbits) -> uint32 words (..., ceil(nbits/32))."""
    nb = bits.shape[-1]
    W = (nb + 31) // 32
    pad = np.zeros(bits.shape[:-1] + (W * 32,), dtype=np.uint64)
    pad[..., :nb] = bits
    pad = pad.reshape(*bits.shape[:-1], W, 32)
    words = (pad << np.arange(32, dtype=np.uint64)).sum(axis=-1)
    return words.astype(np.uint32)


@dataclasses.dataclass
class Report:
    route_flips: List[int] = dataclasses.field(default_factory=list)
    vs_flips: Dict[int, int] = dataclasses.field(default_factory=dict)
    pe_flips: Dict[int, int] = dataclasses.field(default_factory=dict)
    failures: List[str] = dataclasses.field(default_factory=list)

    def heads_with_flips(self):
        return set(self.route_flips) | {h for h, c in self.vs_flips.items() if c} | {
            h for h, c in self.pe_flips.items() if c}

    def assert_ok(self):
        assert not self.failures, "\n".join(self.failures[:20])

    def summary(self) -> str:
        vs = sum(self.vs_flips.values())
        pe = sum(self.pe_flips.values())
        worst_vs = max(self.vs_flips.items(), key=lambda kv: kv[1], default=(None, 0))
        worst_pe = max(self.pe_flips.items(), key=lambda kv: kv[1], default=(None, 0))
        return (f"flips: route {len(self.route_flips)} heads {self.route_flips}; VS blocks {vs} "
                f"(max {worst_vs[1]} on head {worst_vs[0]}); PE blocks {pe} (max {worst_pe[1]} on head {worst_pe[0]})")

    def assert_flips_bounded(self, nb: int, frac: float = FLIP_FRAC_MAX):
        """Each head's flips stay a small fraction of its candidates."""
        for h, c in self.vs_flips.items():
            assert c <= frac * 2 * nb, f"head {h}: {c} VS flips of {2 * nb} blocks"
        for h, c in self.pe_flips.items():
            assert c <= frac * nb * (nb + 1) / 2, f"head {h}: {c} PE flips of {nb * (nb + 1) // 2} blocks"


def compare_route(h, c_gpu, route_gpu, idx, tau, rep: Report):
    if route_gpu != idx.route:
        if abs(idx.c_struct - tau) <= REL_FLIP * abs(tau):
            rep.route_flips.append(h)
        else:
            rep.failures.append(f"head {h}: route gpu={route_gpu} oracle={idx.route} C={idx.c_struct:.6g}")
    if not abs(c_gpu - idx.c_struct) <= 1e-4 + 1e-4 * abs(idx.c_struct):
        rep.failures.append(f"head {h}: C_struct gpu={c_gpu:.7g} oracle={idx.c_struct:.7g}")


def compare_vs(h, sel_v_gpu, sel_s_gpu, idx, alpha, rep: Report):
    nb = len(idx.p_v)
    flips = 0
    for name, gpu, ref, p, mu in (("v", sel_v_gpu, idx.sel_v, idx.p_v, idx.mu_v),
                                  ("s", sel_s_gpu, idx.sel_s, idx.p_s, idx.mu_s)):
        bad = np.nonzero(gpu[:nb] != ref)[0]
        thr = alpha * mu
        for b in bad:
            if abs(p[b] - thr) <= REL_FLIP * abs(thr):
                flips += 1
            else:
                rep.failures.append(f"head {h}: VS {name}-block {b} gpu={gpu[b]} oracle={ref[b]} "
                                    f"p={p[b]:.6g} thr={thr:.6g}")
    rep.vs_flips[h] = flips


def _mass_before(pe, nb):
    """Cumulative mass of the entries ranked before each causal entry in the
    oracle's order (value descending, flat index ascending), as [nb, nb]."""
    r, c = np.tril_indices(nb)
    a = pe.values[r, c]
    order = np.lexsort((r * nb + c, -a))
    before = np.empty(len(a))
    before[order] = np.concatenate(([0.0], np.cumsum(a[order])[:-1]))
    out = np.zeros((nb, nb))
    out[r, c] = before
    return out


def compare_pe(h, mask_gpu, idx, rep: Report, gamma: float = None):
    pe = idx.pe
    nb = pe.mask.shape[0]
    gpu = mask_gpu[:nb, :nb]
    bad = np.argwhere(gpu != pe.mask)
    flips = 0
    cut = pe.cut_value
    before = None
    for r, c in bad:
        if c > r:
            rep.failures.append(f"head {h}: PE mask set above the diagonal at ({r},{c})")
            continue
        v = pe.values[r, c]
        if cut > 0 and abs(v - cut) <= REL_FLIP * cut:
            flips += 1
            continue
        if gamma is not None and gamma < 1.0:
            if before is None:
                before = _mass_before(pe, nb)
            if abs(before[r, c] - gamma) <= REL_FLIP * gamma:
                flips += 1
                continue
        rep.failures.append(f"head {h}: PE block ({r},{c}) gpu={gpu[r, c]} oracle={pe.mask[r, c]} "
                            f"value={v:.6g} cut={cut:.6g}")
    rep.pe_flips[h] = flips


def output_error(o_gpu: np.ndarray, o_ref: np.ndarray) -> float:
    """max |o - o_ref| / max |o_ref| over the whole array (one head's rows)."""
    return float(np.max(np.abs(o_gpu - o_ref)) / max(np.max(np.abs(o_ref)), 1e-30))


def row_error(o_gpu: np.ndarray, o_ref: np.ndarray) -> float:
    """max over rows of max_c |o - o_ref| / max_c |o_ref| (rows: [rows, d])."""
    num = np.max(np.abs(o_gpu - o_ref), axis=-1)
    den = np.maximum(np.max(np.abs(o_ref), axis=-1), 1e-30)
    return float(np.max(num / den))
