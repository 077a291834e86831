"""Host-side comparison rules used by the GPU parity tests (no GPU needed)."""
import numpy as np

import parity as P
from oracle import crisp_oracle as O


def test_mask_pack_roundtrip():
    r = np.random.default_rng(0)
    for nb in (1, 31, 32, 33, 100, 4096):
        bits = r.random((3, nb)) < 0.4
        words = P.pack_mask(bits)
        assert words.shape == (3, (nb + 31) // 32)
        assert (P.unpack_mask(words, nb) == bits).all()
    w = P.pack_mask(np.array([True, False, True] + [False] * 29 + [True]))
    assert w.tolist() == [5, 1]


def _idx(route=O.VS, c=0.5):
    p = np.array([0.4, 0.05, 0.2, 0.05, 0.3])
    sel, mu = O.threshold_blocks(p, 0, 4, 1.0)
    return O.HeadIndex(c, route, p, p.copy(), sel, sel.copy(), mu, mu, None)


def test_route_flip_only_near_tau():
    rep = P.Report()
    P.compare_route(0, 0.5, O.PE, _idx(c=0.5), 0.1, rep)
    assert rep.failures
    rep = P.Report()
    P.compare_route(0, 0.10001, O.PE, _idx(c=0.10001), 0.1, rep)
    assert rep.route_flips == [0] and not rep.failures


def test_vs_mismatch_far_from_threshold_fails_near_is_flip():
    idx = _idx()
    gpu = idx.sel_v.copy()
    gpu[1] = True                     # p=0.05 vs thr=0.1: far -> failure
    rep = P.Report()
    P.compare_vs(0, gpu, idx.sel_s, idx, 1.0, rep)
    assert rep.failures
    idx.p_v[1] = idx.mu_v * (1 + 1e-4)  # now within 1e-3 of the threshold -> flip
    idx.sel_v[1] = True
    gpu2 = idx.sel_v.copy()
    gpu2[1] = False
    rep = P.Report()
    P.compare_vs(0, gpu2, idx.sel_s, idx, 1.0, rep)
    assert not rep.failures and rep.vs_flips[0] == 1


def test_row_error_measures_each_row_against_its_own_size():
    ref = np.array([[10.0, -10.0, 1.0], [0.01, 0.02, -0.01]])
    gpu = ref.copy()
    gpu[1, 1] += 0.001                 # 0.001 off a row whose largest entry is 0.02
    assert abs(P.output_error(gpu, ref) - 0.001 / 10.0) < 1e-12
    assert abs(P.row_error(gpu, ref) - 0.001 / 0.02) < 1e-12
    assert P.row_error(ref, ref) == 0.0


def test_flip_bound_is_per_head_and_per_kind():
    rep = P.Report()
    rep.vs_flips = {0: 1, 1: 0}
    rep.pe_flips = {2: 3}
    rep.assert_flips_bounded(nb=64)    # 1 of 128 VS blocks, 3 of 2080 PE blocks
    assert "VS blocks 1" in rep.summary() and "PE blocks 3" in rep.summary()
    rep.vs_flips[1] = 2                # 2 of 128 VS blocks: above 1%
    try:
        rep.assert_flips_bounded(nb=64)
    except AssertionError:
        pass
    else:
        raise AssertionError("2 of 128 VS flips exceeds 1%")


def test_pe_block_on_the_gamma_threshold_is_a_flip():
    # a 3x3 causal map already normalised: sorted 0.4 (0,0), 0.2 (2,0), 0.15 (2,1),
    # 0.1 (1,0), 0.1 (1,1), 0.05 (2,2); gamma = 0.6 is reached by the first two,
    # so (2,1) sits on the threshold (mass before it = gamma) while (1,0) does not
    vals = np.array([[0.4, 0.0, 0.0], [0.1, 0.1, 0.0], [0.2, 0.15, 0.05]])
    sel = O.gamma_select(vals, 0.6)
    assert sel.k_star == 2
    idx = O.HeadIndex(0.0, O.PE, None, None, None, None, 0.0, 0.0, sel)
    gpu = sel.mask.copy()
    gpu[2, 1] = True                  # value 0.15, 25% from the cut 0.2
    rep = P.Report()
    P.compare_pe(0, gpu, idx, rep)    # by value alone: a failure
    assert rep.failures
    rep = P.Report()
    P.compare_pe(0, gpu, idx, rep, 0.6)
    assert not rep.failures and rep.pe_flips[0] == 1
    gpu2 = sel.mask.copy()
    gpu2[1, 0] = True                 # mass before it is 0.75: far from gamma
    rep = P.Report()
    P.compare_pe(0, gpu2, idx, rep, 0.6)
    assert rep.failures
