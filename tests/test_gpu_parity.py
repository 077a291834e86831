"""CUDA path vs the CPU oracle, through the C ABI, on seeded synthetic layers.

Routes and index sets must match bit for bit except documented flips
(tests/parity.py), whose counts are printed and, at full size, bounded;
outputs on the same indices within 2e-2 (bf16) or 1e-4 (fp32) max relative
error, per head and per row. Small layers are checked on every row; the
full-size layers on sampled query rows of every head.

"The same indices" is reached in the direction that keeps the oracle free of
anything the CUDA path produced: crisp_attend is run on the ORACLE's route
and masks for every head, so the attention kernel is checked on all heads,
flipped or not; the whole-path crisp_prefill output (the GPU's own indices)
is checked on the heads whose indices match the oracle's exactly.
"""
import numpy as np
import pytest

import crisp_synth as S
from oracle import crisp_oracle as O
import parity as P

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import long_context_prefill_last_b200 as crisp  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def built():
    from long_context_prefill_last_b200 import build
    build.build()
    crisp.lib()


def f32(x):
    return float(np.float32(x))


def oracle_cfg(cfg: crisp.Config) -> O.OracleCfg:
    # the knobs exactly as the device sees them (float32)
    return O.OracleCfg(tau_proxy=f32(cfg.tau_proxy), alpha=f32(cfg.alpha), gamma=f32(cfg.gamma),
                       force_route=cfg.force_route)


def device_layer(layer):
    return tuple(t.cuda() for t in S.to_torch(layer))


def make_cfg(layer, **kw):
    c = layer.cfg
    cfg = crisp.Config(n=c.n, h_q=c.h_q, h_kv=c.h_kv, d=c.d, dtype=crisp.FP32 if c.dtype == "fp32" else crisp.BF16,
                       **kw)
    cfg.allocate_workspace()
    return cfg


def gpu_select(q, k, cfg):
    ix = crisp.IndexBuffers(cfg)
    crisp.select(q, k, cfg, ix)
    crisp.raise_on_device_status(cfg, where="select")
    nb = cfg.n_blocks
    host = {f: getattr(ix, f).cpu().numpy() for f in ("route", "c_struct", "p_v", "p_s", "mu", "nv", "ns",
                                                       "pe_count", "pe_cut", "v_idx", "s_idx")}
    host["sel_v"] = P.unpack_mask(ix.vs_mask[:, 0].cpu().numpy().view(np.uint32), nb)
    host["sel_s"] = P.unpack_mask(ix.vs_mask[:, 1].cpu().numpy().view(np.uint32), nb)
    host["pe"] = P.unpack_mask(ix.pe_mask.cpu().numpy().view(np.uint32), nb)
    return host, ix


def oracle_heads(layer, ocfg, heads=None):
    G = layer.cfg.group
    kcache = {}

    def getk(g):
        if g not in kcache:
            kcache.clear()
            kcache[g] = layer.as_f64("k", g)
        return kcache[g]

    out = {}
    for h in (heads if heads is not None else range(layer.cfg.h_q)):
        out[h] = O.head_index(layer.as_f64("q", h), getk(h // G), ocfg)
    return out


def check_index(host, oidx, cfg, rep):
    for h, idx in oidx.items():
        P.compare_route(h, float(host["c_struct"][h]), int(host["route"][h]), idx, f32(cfg.tau_proxy), rep)
        P.compare_vs(h, host["sel_v"][h], host["sel_s"][h], idx, f32(cfg.alpha), rep)
        # the compacted lists agree with the masks
        nv, ns = int(host["nv"][h]), int(host["ns"][h])
        assert (host["v_idx"][h][:nv] == np.nonzero(host["sel_v"][h])[0]).all()
        assert (host["s_idx"][h][:ns] == np.nonzero(host["sel_s"][h])[0]).all()
        if idx.route == O.PE and int(host["route"][h]) == O.PE:
            P.compare_pe(h, host["pe"][h], idx, rep, f32(cfg.gamma))
            assert int(host["pe_count"][h]) == int(host["pe"][h][np.tril_indices(cfg.n_blocks)].sum())
        # the block masses themselves (float32 device sums vs float64)
        np.testing.assert_allclose(host["p_v"][h], idx.p_v, rtol=2e-3, atol=2e-6)
        np.testing.assert_allclose(host["p_s"][h], idx.p_s, rtol=2e-3, atol=2e-6)


def sample_rows(n, nb, full):
    if full:
        return np.arange(n)
    tiles = sorted({0, 1, nb // 3, nb // 2, nb - 2, nb - 1})
    rows = []
    for t in tiles:
        rows += [t * 128, t * 128 + 37, t * 128 + 64, t * 128 + 127]
    return np.array(sorted(set(r for r in rows if r < n)))


def check_outputs(layer, out, oidx, ocfg, rows, skip_heads=(), tol=None, head_offset=0):
    """Compare out[head_offset + h] with the oracle's attention on oidx[h] for
    every head not skipped; returns (heads checked, worst head error, worst row error)."""
    tol = tol if tol is not None else P.TOL[layer.cfg.dtype]
    G = layer.cfg.group
    o = out.float().cpu().numpy()
    worst, worst_row, checked = 0.0, 0.0, 0
    for h, idx in oidx.items():
        if h in skip_heads:
            continue
        q, k, v = layer.as_f64("q", h), layer.as_f64("k", h // G), layer.as_f64("v", h // G)
        ref = O.head_attention(q, k, v, idx, rows, ocfg)
        err = P.output_error(o[head_offset + h][rows], ref)
        rerr = P.row_error(o[head_offset + h][rows], ref)
        worst, worst_row = max(worst, err), max(worst_row, rerr)
        checked += 1
        assert err <= tol, f"head {h}: output error {err:.3g} > {tol}"
        assert rerr <= tol, f"head {h}: per-row output error {rerr:.3g} > {tol}"
    return checked, worst, worst_row


def oracle_index_buffers(oidx, cfg):
    """Device index buffers holding the ORACLE's route and masks (inputs for crisp_attend)."""
    ix = crisp.IndexBuffers(cfg)
    nb = cfg.n_blocks
    h_q = cfg.h_q
    route = np.zeros(h_q, np.int32)
    vs = np.zeros((h_q, 2, cfg.words), np.uint32)
    pe = np.zeros((h_q, nb, cfg.words), np.uint32)
    for h, idx in oidx.items():
        route[h] = idx.route
        vs[h, 0] = P.pack_mask(idx.sel_v)
        vs[h, 1] = P.pack_mask(idx.sel_s)
        if idx.pe is not None:
            pe[h] = P.pack_mask(idx.pe.mask)
    ix.route.copy_(torch.from_numpy(route))
    ix.vs_mask.copy_(torch.from_numpy(vs.view(np.int32)))
    ix.pe_mask.copy_(torch.from_numpy(pe.view(np.int32)))
    return ix


# ----------------------------------------------------------------------------- small layers

SMALL = {
    "A-auto": (lambda: S.CONFIGS["A"], {}),
    "A-forceVS": (lambda: S.CONFIGS["A"], {"force_route": 0}),
    "B-4k": (lambda: S.scaled("B", n=4096, h_q=8, h_kv=2), {}),
    "D-2k": (lambda: S.scaled("D", n=2048, h_q=14, h_kv=2), {}),
    "B-512-min": (lambda: S.scaled("B", n=512, h_q=4, h_kv=1, planted_groups=[0]), {}),
    "B-4224-33blocks": (lambda: S.scaled("B", n=4224, h_q=4, h_kv=2), {}),
    "B-4k-alpha1.5": (lambda: S.scaled("B", n=4096, h_q=8, h_kv=2), {"alpha": 1.5}),
    "B-4k-alpha1.25-gamma0.97": (lambda: S.scaled("B", n=4096, h_q=8, h_kv=2), {"alpha": 1.25, "gamma": 0.97}),
    "D-2k-alpha1.5-gamma0.97": (lambda: S.scaled("D", n=2048, h_q=14, h_kv=2), {"alpha": 1.5, "gamma": 0.97}),
    "B-4k-alpha0": (lambda: S.scaled("B", n=4096, h_q=8, h_kv=2), {"alpha": 0.0}),
    "B-4k-gamma1": (lambda: S.scaled("B", n=4096, h_q=8, h_kv=2), {"gamma": 1.0}),
    "B-4k-gamma0.5": (lambda: S.scaled("B", n=4096, h_q=8, h_kv=2), {"gamma": 0.5}),
    "B-4k-forcePE": (lambda: S.scaled("B", n=4096, h_q=8, h_kv=2), {"force_route": 1}),
    "B-4k-alphaHuge": (lambda: S.scaled("B", n=4096, h_q=8, h_kv=2), {"alpha": 1e30}),
    # the largest KV group the kernels take (16 query heads per K/V head): all VS, all PE
    "B-2k-group16-VS": (lambda: S.scaled("B", n=2048, h_q=16, h_kv=1, planted_groups=[0]), {}),
    "B-2k-group16-PE": (lambda: S.scaled("B", n=2048, h_q=16, h_kv=1, planted_groups=[]), {"force_route": 1}),
    # mass-cliff background (log-normal block masses): sparser VS and PE selections
    "Ccliff-4k": (lambda: S.scaled("C_cliff", n=4096, h_q=8, h_kv=2), {}),
    "Ccliff-16k": (lambda: S.scaled("C_cliff", n=16384, h_q=8, h_kv=2), {}),
    "Ccliff-4k-alpha1.5-gamma0.97": (lambda: S.scaled("C_cliff", n=4096, h_q=8, h_kv=2), {"alpha": 1.5, "gamma": 0.97}),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_layer_parity(name):
    make, knobs = SMALL[name]
    layer = S.generate(make())
    q, k, v = device_layer(layer)
    cfg = make_cfg(layer, **knobs)
    ocfg = oracle_cfg(cfg)
    host, _ = gpu_select(q, k, cfg)
    oidx = oracle_heads(layer, ocfg)
    rep = P.Report()
    check_index(host, oidx, cfg, rep)
    rep.assert_ok()
    print(name, rep.summary())
    # whole path; outputs compared where the indices agree exactly
    out = torch.empty_like(q)
    crisp.prefill(q, k, v, out, cfg)
    crisp.raise_on_device_status(cfg, where="prefill")
    rows = sample_rows(cfg.n, cfg.n_blocks, full=cfg.n <= 4224)
    check_outputs(layer, out, oidx, ocfg, rows, skip_heads=rep.heads_with_flips())
    # attention on the oracle's own indices, every head
    ix = oracle_index_buffers(oidx, cfg)
    out2 = torch.empty_like(q)
    crisp.attend(q, k, v, out2, cfg, ix)
    crisp.raise_on_device_status(cfg, where="attend")
    check_outputs(layer, out2, oidx, ocfg, rows)


@pytest.mark.parametrize("base,n,hq,hkv", [("A", 4096, 1, 1), ("B", 4096, 8, 2), ("D", 2048, 14, 2)])
def test_dense_attention_parity(base, n, hq, hkv):
    c = S.CONFIGS["A"] if base == "A" else S.scaled(base, n=n, h_q=hq, h_kv=hkv)
    layer = S.generate(c)
    q, k, v = device_layer(layer)
    cfg = make_cfg(layer)
    out = torch.empty_like(q)
    crisp.dense_attention(q, k, v, out, cfg)
    crisp.raise_on_device_status(cfg, where="dense")
    o = out.float().cpu().numpy()
    rows = np.arange(n) if n <= 4096 and hq <= 8 else sample_rows(n, n // 128, False)
    tol = P.TOL[c.dtype]
    for h in range(hq):
        g = h // c.group
        ref = O.dense_attention(layer.as_f64("q", h), layer.as_f64("k", g), layer.as_f64("v", g), rows,
                                1 / np.sqrt(128))
        assert P.output_error(o[h][rows], ref) <= tol


def test_tensor_core_and_cuda_core_attention_agree():
    # the CUDA-core attention kernel (the fp32 path) run on a bf16 layer
    # through the diagnostics entry point, against the tensor-core kernel
    layer = S.generate(S.scaled("B", n=4096, h_q=8, h_kv=2))
    q, k, v = device_layer(layer)
    cfg = make_cfg(layer)
    ix = crisp.IndexBuffers(cfg)
    crisp.select(q, k, cfg, ix)
    tc_sparse, tc_dense, simt_sparse, simt_dense = (torch.empty_like(q) for _ in range(4))
    crisp.attend(q, k, v, tc_sparse, cfg, ix)
    crisp.dense_attention(q, k, v, tc_dense, cfg)
    crisp.diag_attend_simt(q, k, v, simt_sparse, cfg, ix)
    crisp.diag_attend_simt(q, k, v, simt_dense, cfg, None, dense=True)
    crisp.raise_on_device_status(cfg)
    for a, b in ((tc_sparse, simt_sparse), (tc_dense, simt_dense)):
        a, b = a.float(), b.float()
        err = (a - b).abs().max().item() / b.abs().max().item()
        assert err < 2e-2


@pytest.mark.parametrize("base,n,hq,hkv", [("B", 4096, 8, 2), ("D", 2048, 14, 2), ("B", 640, 1, 1)])
def test_tensor_core_and_cuda_core_proxy_agree(base, n, hq, hkv):
    layer = S.generate(S.scaled(base, n=n, h_q=hq, h_kv=hkv))
    q, k, _ = device_layer(layer)
    cfg = make_cfg(layer)
    host_tc, _ = gpu_select(q, k, cfg)
    ix = crisp.IndexBuffers(cfg)
    crisp.diag_select_simt(q, k, cfg, ix)
    crisp.raise_on_device_status(cfg, where="diag_select_simt")
    for f in ("p_v", "p_s", "c_struct"):
        np.testing.assert_allclose(host_tc[f], getattr(ix, f).cpu().numpy(), rtol=1e-4, atol=1e-7)


def test_fma_pipe_exp2_against_cuda_exp2f():
    x = torch.cat([torch.linspace(-124.0, 8.0, 1 << 20), torch.tensor([0.0, -0.5, 0.5, -1.0, 7.99, -123.7])]).cuda()
    p3, p5, ref = crisp.exp2_selftest(x)
    torch.cuda.synchronize()
    r = ref.double()
    e3 = ((p3.double() - r).abs() / r).max().item()
    e5 = ((p5.double() - r).abs() / r).max().item()
    # minimax bounds of the fits (7.5e-5 and 2.3e-7) plus exp2f's own error
    assert e3 < 8e-5, e3
    assert e5 < 4e-7, e5


def test_repeat_calls_are_deterministic():
    layer = S.generate(S.scaled("D", n=2048, h_q=14, h_kv=2))
    q, k, v = device_layer(layer)
    cfg = make_cfg(layer)
    o1, o2 = torch.empty_like(q), torch.empty_like(q)
    crisp.prefill(q, k, v, o1, cfg)
    crisp.prefill(q, k, v, o2, cfg)
    crisp.raise_on_device_status(cfg)
    assert torch.equal(o1, o2)


def oracle_check_sequence(layer, out, cfg, head_offset=0):
    """One sequence's output (heads head_offset.. of `out`) against the oracle
    on the oracle's own indices, on every head whose GPU selection (a
    crisp_select call on the same inputs) matches the oracle's with no flip."""
    q, k, _ = device_layer(layer)
    ocfg = oracle_cfg(cfg)
    host, _ = gpu_select(q, k, cfg)
    oidx = oracle_heads(layer, ocfg)
    rep = P.Report()
    check_index(host, oidx, cfg, rep)
    rep.assert_ok()
    rows = sample_rows(cfg.n, cfg.n_blocks, full=cfg.n <= 2048)
    checked, _, _ = check_outputs(layer, out, oidx, ocfg, rows, skip_heads=rep.heads_with_flips(),
                                  head_offset=head_offset)
    assert checked >= cfg.h_q - len(rep.heads_with_flips()) and checked > 0


def test_batch_and_varlen_match_single_calls_and_the_oracle():
    # two sequences of one length as a batch, and three lengths as varlen: each
    # output equals the single-sequence call (every stage works per head), and
    # one sequence of each call is held against the oracle directly
    la = S.generate(S.scaled("B", n=2048, h_q=8, h_kv=2))
    lb = S.generate(S.scaled("C_cliff", n=2048, h_q=8, h_kv=2))
    lc = S.generate(S.scaled("B", n=1024, h_q=8, h_kv=2, config_id=977))
    (qa, ka, va), (qb, kb, vb), (qc, kc, vc) = device_layer(la), device_layer(lb), device_layer(lc)
    singles = []
    for (q, k, v), lay in (((qa, ka, va), la), ((qb, kb, vb), lb), ((qc, kc, vc), lc)):
        cfg = make_cfg(lay)
        o = torch.empty_like(q)
        crisp.prefill(q, k, v, o, cfg)
        crisp.raise_on_device_status(cfg)
        singles.append(o)
    cfgb = crisp.Config(n=2048, h_q=8, h_kv=2)
    cfgb.allocate_workspace(batch=2)
    q, k, v = torch.stack([qa, qb]), torch.stack([ka, kb]), torch.stack([va, vb])
    out = torch.empty_like(q)
    crisp.prefill_batch(q, k, v, out, cfgb)
    crisp.raise_on_device_status(cfgb, where="prefill_batch")
    assert torch.equal(out[0], singles[0]) and torch.equal(out[1], singles[1])
    oracle_check_sequence(lb, out[1], make_cfg(lb))                 # second sequence of the batch
    cfgv = crisp.Config(n=2048, h_q=8, h_kv=2)
    cfgv.allocate_workspace(max_n=2048)
    outs = [torch.empty_like(qc), torch.empty_like(qa), torch.empty_like(qb)]
    crisp.prefill_varlen([qc, qa, qb], [kc, ka, kb], [vc, va, vb], outs, cfgv)
    crisp.raise_on_device_status(cfgv, where="prefill_varlen")
    assert torch.equal(outs[0], singles[2]) and torch.equal(outs[1], singles[0]) and torch.equal(outs[2], singles[1])
    oracle_check_sequence(lc, outs[0], make_cfg(lc))                # the shorter sequence of the varlen call


def test_host_prefill_matches_device_prefill_and_the_oracle():
    # the layer in page-locked host memory, computed KV group by KV group with
    # the copies on a second stream: the same output as the device call, and
    # the oracle's on every head
    layer = S.generate(S.scaled("B", n=4096, h_q=16, h_kv=4))
    qh, kh, vh = (t.pin_memory() for t in S.to_torch(layer))
    q, k, v = qh.cuda(), kh.cuda(), vh.cuda()
    cfg = make_cfg(layer)
    ref = torch.empty_like(q)
    crisp.prefill(q, k, v, ref, cfg)
    crisp.raise_on_device_status(cfg)
    c = layer.cfg
    hcfg = crisp.Config(n=c.n, h_q=c.h_q, h_kv=c.h_kv, d=c.d, dtype=crisp.BF16)
    hcfg.allocate_workspace(host=True)
    out_h = torch.empty(qh.shape, dtype=qh.dtype).pin_memory()
    crisp.prefill_host(qh, kh, vh, out_h, hcfg)
    torch.cuda.current_stream().synchronize()
    crisp.raise_on_device_status(hcfg, where="prefill_host")
    assert torch.equal(out_h, ref.cpu())
    oracle_check_sequence(layer, out_h, cfg)


def test_bounded_wait_runs_out_with_a_status_and_the_context_survives():
    # the wait every kernel uses, on a barrier nothing arrives on, with a
    # limit of about a millisecond: the kernel ends and reports the site
    st = torch.zeros(8, dtype=torch.int32, device="cuda")
    crisp.wait_selftest(2_000_000, st)
    torch.cuda.synchronize()
    assert int(st[0]) == 9 and int(st[1]) == 99          # CRISP_ERR_TIMEOUT at site 99
    layer = S.generate(S.scaled("B", n=1024, h_q=4, h_kv=2))
    q, k, v = device_layer(layer)
    cfg = make_cfg(layer)
    out = torch.empty_like(q)
    crisp.prefill(q, k, v, out, cfg)
    crisp.raise_on_device_status(cfg)
    assert torch.isfinite(out.float()).all()


def test_nonfinite_proxy_statistics_are_reported_not_trapped():
    layer = S.generate(S.scaled("B", n=2048, h_q=4, h_kv=2))
    q, k, v = device_layer(layer)
    cfg = make_cfg(layer)
    bad = q.clone()
    bad[1, -1, :] = float("nan")                          # a proxy row of query head 1
    out = torch.empty_like(q)
    crisp.prefill(bad, k, v, out, cfg)
    assert crisp.device_status(cfg) == 10                  # CRISP_ERR_NONFINITE (and cleared by the read)
    crisp.prefill(q, k, v, out, cfg)                       # the next call runs normally
    crisp.raise_on_device_status(cfg)
    assert torch.isfinite(out.float()).all()


# ----------------------------------------------------------------------------- full-size layers

def full_size_outputs(layer, q, k, v, cfg, ocfg, oidx, rep):
    """Whole-path output on heads without flips, and crisp_attend on the
    oracle's own indices on every head (sampled rows)."""
    nb = cfg.n_blocks
    rows = sample_rows(cfg.n, nb, full=False)
    out = torch.empty_like(q)
    crisp.prefill(q, k, v, out, cfg)
    crisp.raise_on_device_status(cfg, where="prefill")
    flipped = rep.heads_with_flips()
    n1, e1, r1 = check_outputs(layer, out, oidx, ocfg, rows, skip_heads=flipped)
    del out
    ix = oracle_index_buffers(oidx, cfg)
    out2 = torch.empty_like(q)
    crisp.attend(q, k, v, out2, cfg, ix)
    crisp.raise_on_device_status(cfg, where="attend on the oracle's indices")
    n2, e2, r2 = check_outputs(layer, out2, oidx, ocfg, rows)
    assert n2 == cfg.h_q
    print(f"{layer.cfg.name}: {rep.summary()}; prefill checked on {n1}/{cfg.h_q} heads (max err {e1:.3g}, "
          f"row {r1:.3g}); attend on the oracle's indices {n2}/{cfg.h_q} heads (max err {e2:.3g}, row {r2:.3g})")


def test_longest_accepted_sequence():
    # n = 2^20, the largest length the boundary accepts (N_b = 8192, 256 mask
    # words per row): one planted (VS) and one Gaussian (PE) KV group
    layer = S.generate(S.scaled("B", n=1 << 20, h_q=8, h_kv=2), threads=16)
    q, k, v = device_layer(layer)
    cfg = make_cfg(layer)
    ocfg = oracle_cfg(cfg)
    host, _ = gpu_select(q, k, cfg)
    oidx = oracle_heads(layer, ocfg)
    rep = P.Report()
    check_index(host, oidx, cfg, rep)
    rep.assert_ok()
    rep.assert_flips_bounded(cfg.n_blocks)
    assert all(host["route"][h] == O.VS for h in layer.planted_q_heads)
    assert all(host["route"][h] == O.PE for h in layer.gaussian_q_heads)
    full_size_outputs(layer, q, k, v, cfg, ocfg, oidx, rep)


@pytest.mark.parametrize("name", ["B", "C", "D", "E", "E_cliff"])
def test_full_size_layer_parity(name):
    layer = S.generate(S.CONFIGS[name], threads=16)
    q, k, v = device_layer(layer)
    cfg = make_cfg(layer)
    ocfg = oracle_cfg(cfg)
    host, _ = gpu_select(q, k, cfg)
    oidx = oracle_heads(layer, ocfg)
    rep = P.Report()
    check_index(host, oidx, cfg, rep)
    rep.assert_ok()
    rep.assert_flips_bounded(cfg.n_blocks)
    if layer.cfg.cliff_sigma > 0:
        # a cliffed background hides planted keys that sit in light blocks; the
        # sink still routes planted heads VS and the cliff keeps the selections sparse
        for h in layer.planted_q_heads:
            assert host["route"][h] == O.VS
            assert host["sel_v"][h].mean() < 0.5 and host["sel_s"][h].mean() < 0.5
    # planted structure must be selected, Gaussian heads must route PE
    for h in ([] if layer.cfg.cliff_sigma > 0 else layer.planted_q_heads):
        assert host["route"][h] == O.VS
        st = layer.structure[h // layer.cfg.group]
        assert host["sel_v"][h][st.verticals // 128].all()
        assert host["sel_s"][h][st.slash_offsets // 128].all()
    for h in layer.gaussian_q_heads:
        assert host["route"][h] == O.PE
    del host
    full_size_outputs(layer, q, k, v, cfg, ocfg, oidx, rep)
