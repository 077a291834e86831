"""Host-side helpers of bench.py (no GPU): the computed-tile count that the
attention roofline divides by, and the roofline bookkeeping."""
import importlib.util
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
bench = importlib.util.module_from_spec(spec)
spec.loader.exec_module(bench)

B = 128


def pack(bits):
    w = np.zeros((len(bits) + 31) // 32, np.uint32)
    for i, b in enumerate(bits):
        if b:
            w[i // 32] |= np.uint32(1 << (i % 32))
    return w


def brute_tiles(route, sel_v, sel_s, pe, nb):
    """Tiles (I, t), t <= I, holding at least one selected causal (i, j): element by element."""
    n = nb * B
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    total = 0
    for h in range(len(route)):
        if route[h] == 1:
            keep = pe[h][i // B, j // B] | (i // B == j // B)
        else:
            keep = sel_v[h][j // B] | sel_s[h][np.clip(i - j, 0, n - 1) // B] | (i // B == j // B)
        keep &= j <= i
        tiles = keep.reshape(nb, B, nb, B).any(axis=(1, 3))
        total += int(tiles.sum())
    return total


def test_kept_tiles_matches_element_level_enumeration():
    rng = np.random.default_rng(7)
    nb = 6
    route = np.array([0, 0, 1, 1])
    sel_v = rng.random((4, nb)) < 0.3
    sel_s = rng.random((4, nb)) < 0.3
    pe = rng.random((4, nb, nb)) < 0.3
    vs_mask = np.stack([np.stack([pack(sel_v[h]), pack(sel_s[h])]) for h in range(4)])
    pe_mask = np.stack([np.stack([pack(pe[h][r]) for r in range(nb)]) for h in range(4)])
    assert bench.kept_tiles(route, vs_mask, pe_mask, nb) == brute_tiles(route, sel_v, sel_s, pe, nb)


def test_mufu_roofline_and_traffic_bookkeeping():
    r = bench.mufu_roofline(16 * 148 * 1000 * 1e6 * 1e-3, 1.0, {"sm_mhz": 1000.0}, 148)
    assert abs(r["frac"] - 1.0) < 1e-9 and r["clock_mhz"] == 1000.0
    assert bench.mufu_roofline(1e9, 1.0, {"sm_mhz": None, "sm_max_mhz": None}, 148) is None
    # traffic is reported only for the kernel source and workload it was measured on
    key = next(iter(bench.MEASURED_TRAFFIC))
    e = bench.MEASURED_TRAFFIC[key]
    assert bench.load_traffic(key[0], e["source_hash"], key[1], key[2], key[3]) == e["bytes_per_launch"]
    assert bench.load_traffic(key[0], "0" * 16, key[1], key[2], key[3]) is None
    assert bench.load_traffic(key[0], e["source_hash"], "C", key[2], key[3]) is None
