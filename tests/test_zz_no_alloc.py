"""crisp_route_noalloc: the route stage for callers that cannot give the
library any device memory (for example a plugin hook whose enqueue call has
no workspace argument, or a serving loop that bans allocation once running).

Its scratch is a static device array inside the library, shared by every
call, so two calls in a row must not see each other's leftovers: each call
is compared with crisp_route (which uses a caller workspace) on a different
layer, with the tolerance the parity tests use for C_struct and exact routes.
A device-side failure cannot be read from a caller workspace here (there is
none), so the entry point reports it in its outputs: a NaN in a proxy row
must come back as route -1 and C_struct NaN on every head, and the next call
on good inputs must be normal again. This file is collected last so that, if
it fails, a run that stops at the first failure has already run every other
test.
"""
import numpy as np
import pytest

import crisp_synth as S

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import long_context_prefill_last_b200 as crisp  # noqa: E402


def _route_both(layer_cfg):
    from long_context_prefill_last_b200 import build
    build.build()
    layer = S.generate(layer_cfg, with_v=False)
    q, k, _ = (t.cuda() for t in S.to_torch(layer))
    c = layer.cfg
    cfg = crisp.Config(n=c.n, h_q=c.h_q, h_kv=c.h_kv, dtype=crisp.FP32 if c.dtype == "fp32" else crisp.BF16)
    cfg.allocate_workspace()
    r_ref = torch.empty(c.h_q, dtype=torch.int32, device="cuda")
    c_ref = torch.empty(c.h_q, dtype=torch.float32, device="cuda")
    crisp.route(q, k, cfg, r_ref, c_ref)
    crisp.raise_on_device_status(cfg, where="route")
    cfg_noalloc = crisp.Config(n=c.n, h_q=c.h_q, h_kv=c.h_kv, dtype=cfg.dtype)   # no workspace at all
    r_na = torch.full((c.h_q,), -7, dtype=torch.int32, device="cuda")
    c_na = torch.full((c.h_q,), -7.0, dtype=torch.float32, device="cuda")
    crisp.route_noalloc(q, k, cfg_noalloc, r_na, c_na)
    torch.cuda.synchronize()
    return r_ref.cpu().numpy(), c_ref.cpu().numpy(), r_na.cpu().numpy(), c_na.cpu().numpy()


def test_route_noalloc_matches_route_on_two_calls_in_a_row():
    layers = [S.scaled("B", n=8192, h_q=8, h_kv=2), S.scaled("D", n=4096, h_q=14, h_kv=2)]
    for lc in layers:
        r_ref, c_ref, r_na, c_na = _route_both(lc)
        assert (r_na == r_ref).all(), (lc.name, r_na, r_ref)
        np.testing.assert_allclose(c_na, c_ref, rtol=1e-4, atol=1e-4)
        assert set(np.unique(r_na)) <= {0, 1}


def test_route_noalloc_reports_a_device_failure_in_its_outputs():
    from long_context_prefill_last_b200 import build
    build.build()
    layer = S.generate(S.scaled("B", n=4096, h_q=8, h_kv=2), with_v=False)
    q, k, _ = (t.cuda() for t in S.to_torch(layer))
    cfg = crisp.Config(n=4096, h_q=8, h_kv=2)
    bad = q.clone()
    bad[3, -5, :] = float("nan")                 # one of the 64 proxy rows of query head 3
    r = torch.zeros(8, dtype=torch.int32, device="cuda")
    c = torch.zeros(8, dtype=torch.float32, device="cuda")
    crisp.route_noalloc(bad, k, cfg, r, c)
    torch.cuda.synchronize()
    assert (r.cpu() == -1).all() and torch.isnan(c.cpu()).all()
    crisp.route_noalloc(q, k, cfg, r, c)         # the next call starts clean
    torch.cuda.synchronize()
    assert set(r.cpu().tolist()) <= {0, 1} and torch.isfinite(c.cpu()).all()
