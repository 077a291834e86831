"""The seeded input generator: determinism, dtype handling and planted geometry."""
import dataclasses
import math

import numpy as np
import torch

import crisp_synth as S


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 7
    x[:4] = [0.0, -0.0, 1e-30, 3.3895314e38]
    bits = S.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (bits == ref).all()
    back = S.bf16_bits_to_f32(bits)
    assert (back == torch.from_numpy(x).to(torch.bfloat16).float().numpy()).all()


def test_generation_is_deterministic_and_shaped():
    cfg = S.scaled("B", n=1024, h_q=4, h_kv=2)
    a, b = S.generate(cfg), S.generate(cfg, threads=1)
    assert a.q.shape == (4, 1024, 128) and a.k.shape == (2, 1024, 128) and a.v.shape == (2, 1024, 128)
    assert a.q.dtype == np.uint16
    for t in ("q", "k", "v"):
        assert (getattr(a, t) == getattr(b, t)).all()
    assert a.planted_q_heads == [0, 1] and a.gaussian_q_heads == [2, 3]


def test_planted_logit_boosts_are_exact_in_float64_before_rounding():
    cfg = S.CONFIGS["A"]
    layer = S.generate(cfg, with_v=False)
    st = layer.structure[0]
    q = layer.q[0].astype(np.float64)
    k = layer.k[0].astype(np.float64)
    d = cfg.d
    u = st.u
    # every query has component a = d**0.25 along u; verticals 4*a; sink sink_logits*sqrt(d)/a
    a = d ** 0.25
    assert np.allclose(q @ u, a, atol=1e-4)
    assert np.allclose(k[st.verticals] @ u, 4 * a, atol=1e-4)
    assert abs(k[0] @ u - cfg.sink_logits * math.sqrt(d) / a) < 1e-4
    # slash peak: the slash halves give s^2 * c_i.c_i = 4*sqrt(d) at offset o_t (+ small cross terms)
    ds = S.slash_dims(d)
    i = cfg.n - 1
    for o in st.slash_offsets:
        val = q[i, :ds] @ k[i - o, :ds] / math.sqrt(d)
        assert 2.0 < val < 6.0


def test_sink_fraction_formula():
    # a sink with these extra logits holds fraction f against n-1 lognormal(0,1) keys
    for f, n in [(0.5, 32768), (0.9, 131072)]:
        dl = S.sink_logits_for_fraction(f, n)
        w_sink = math.exp(dl)
        rest = (n - 1) * math.exp(0.5)
        assert abs(w_sink / (w_sink + rest) - f) < 1e-12


def test_cliff_background_offsets_are_exact_per_block():
    # float32 layer (before any bf16 rounding): every key of block b carries
    # exactly beta_b extra logits along the group's cliff direction
    cfg = dataclasses.replace(S.scaled("C_cliff", n=2048, h_q=4, h_kv=2), dtype="fp32")
    layer = S.generate(cfg, with_v=False)
    d, a = cfg.d, cfg.d ** 0.25
    for g in range(cfg.h_kv):
        w, beta = S.cliff_offsets(cfg, g)
        assert beta[0] == 0.0 and beta[-1] == 0.0
        assert abs(np.std(beta[1:-1]) - cfg.cliff_sigma) < 0.5
        k = layer.k[g].astype(np.float64)
        q = layer.q[g * cfg.group].astype(np.float64)
        direction = layer.structure[g].u if g in layer.structure else w
        # queries: component a along the direction; keys: beta_b * a (sink key 0 aside)
        assert np.allclose(q @ direction, a, atol=1e-4)
        kk = k[1:] @ direction
        expect = a * np.repeat(beta, S.BLOCK)[1:cfg.n]
        if g in layer.structure:
            vert = np.zeros(cfg.n, bool)
            vert[layer.structure[g].verticals] = True
            expect = expect + np.where(vert[1:], 4 * a, 0.0)
        assert np.allclose(kk, expect, atol=1e-3)


def test_cliff_sink_fraction_formula():
    # with log-normal block offsets of log-sd sigma the background's mean mass grows by e^(sigma^2/2)
    f, n, sig = 0.5, 131072, 2.0
    dl = S.sink_logits_for_fraction(f, n, sig)
    w_sink = math.exp(dl)
    rest = (n - 1) * math.exp(0.5) * math.exp(sig * sig / 2)
    assert abs(w_sink / (w_sink + rest) - f) < 1e-12


def test_generate_slice_matches_the_full_layer():
    for base in ("B", "C_cliff"):
        cfg = S.scaled(base, n=1024, h_q=8, h_kv=4)
        full = S.generate(cfg)
        G = cfg.group
        for lo, hi in ((0, 1), (1, 3), (2, 4)):
            q, k, v = S.generate_slice(cfg, lo, hi, threads=2)
            assert (q == full.q[lo * G:hi * G]).all()
            assert (k == full.k[lo:hi]).all() and (v == full.v[lo:hi]).all()
