"""Host-side helpers of bench.py (no GPU): the schedule statistics the
attention rooflines divide by, the roofline bookkeeping, the multi-rank
aggregation (2 gloo ranks) and the launcher that starts one rank per GPU."""
import importlib.util
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

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


def brute_keep(route, sel_v, sel_s, pe, nb, h):
    """Selected causal (i, j) of head h, element by element (the oracle's key sets)."""
    n = nb * B
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    if route[h] == 1:
        keep = pe[h][i // B, j // B] | (i // B == j // B)
    else:
        keep = sel_v[h][j // B] | sel_s[h][np.clip(i - j, 0, n - 1) // B] | (i // B == j // B)
    return keep & (j <= i)


def random_index(seed, nb, heads=4):
    rng = np.random.default_rng(seed)
    route = np.array([0, 0, 1, 1][:heads])
    sel_v = rng.random((heads, nb)) < 0.3
    sel_s = rng.random((heads, nb)) < 0.3
    sel_s[:, 0] = True            # offset block 0 is always kept by the VS rule
    pe = rng.random((heads, nb, nb)) < 0.3
    vs_mask = np.stack([np.stack([pack(sel_v[h]), pack(sel_s[h])]) for h in range(heads)])
    pe_mask = np.stack([np.stack([pack(pe[h][r]) for r in range(nb)]) for h in range(heads)])
    return route, sel_v, sel_s, pe, vs_mask, pe_mask


@pytest.mark.parametrize("seed,nb", [(7, 6), (8, 7), (9, 1)])
def test_schedule_stats_match_element_level_enumeration(seed, nb):
    route, sel_v, sel_s, pe, vs_mask, pe_mask = random_index(seed, nb)
    tiles = pairs = union = 0
    for h in range(len(route)):
        keep = brute_keep(route, sel_v, sel_s, pe, nb, h)
        t = keep.reshape(nb, B, nb, B).any(axis=(1, 3))
        tiles += int(t.sum())
        pairs += int(keep.sum())
        for ia in range(nb - 1, -1, -2):          # the CTA pairs (I, I-1)
            u = t[ia].copy()
            if ia >= 1:
                u |= t[ia - 1]
            union += int(u.sum())
    assert bench.schedule_stats(route, vs_mask, pe_mask, nb) == (tiles, pairs, union)


def test_mufu_roofline_and_traffic_bookkeeping(monkeypatch):
    r = bench.mufu_roofline(16 * 148 * 1000 * 1e6 * 1e-3, 1.0, {"sm_mhz": 1000.0}, 148)
    assert abs(r["frac"] - 1.0) < 1e-9 and r["clock_mhz"] == 1000.0
    assert bench.mufu_roofline(1e9, 1.0, {"sm_mhz": None, "sm_max_mhz": None}, 148) is None
    # traffic is reported only for the kernel source and workload it was measured on
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, ("attn_tc_kernel", "E", 1.0, 0.95),
                        {"source_hash": "ab" * 8, "bytes_per_launch": 1e12})
    assert bench.load_traffic("attn_tc_kernel", "ab" * 8, "E", 1.0, 0.95) == 1e12
    assert bench.load_traffic("attn_tc_kernel", "0" * 16, "E", 1.0, 0.95) is None
    assert bench.load_traffic("attn_tc_kernel", "ab" * 8, "C", 1.0, 0.95) is None


def test_clock_lines_parse_median_under_load_and_reasons():
    lines = ["0, 1800, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active",
             "0, 1900, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active",
             "0, 300, 1965, 100.0, 0x0, Not Active, Not Active, Not Active, Not Active"]
    c = bench.parse_clock_lines(lines)
    assert c["sm_mhz"] == 1850 and c["sm_max_mhz"] == 1965 and c["reasons"] == ["sw_power_cap"]


def test_launcher_starts_one_rank_per_gpu(monkeypatch):
    cmd = bench.launch_command(4, ["--gpus", "4", "--steps", "2"], port=29555)
    i = cmd.index("torch.distributed.run")
    assert cmd[:4] == ["timeout", "-k", "60", "3600"]
    assert "--nproc-per-node=4" in cmd and cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[i + 1:].count(os.path.join(ROOT, "bench.py")) == 1 and cmd[-4:] == ["--gpus", "4", "--steps", "2"]
    # without a launcher in the environment, --gpus N > 1 re-runs itself under one
    seen = {}
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench.subprocess, "call", lambda c: seen.setdefault("cmd", c) and 0)
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "2", "--steps", "1"])
    assert "--nproc-per-node=2" in seen["cmd"]


def _fake_measurement(rank):
    # a GPU-free stand-in for one rank's measurements (rank 1 is slower)
    f = 1.0 + rank
    return {"step_ms": [10.0 * f, 12.0 * f], "att_ms": [8.0 * f], "sel_ms": [2.0 * f], "dense_ms": [20.0 * f],
            "e2e_ms": [11.0 * f], "route_ms": [0.5 * f], "tiles": 100 + rank, "pairs": 1000, "union_tiles": 120,
            "causal_tiles": 200, "causal_pairs": 4000, "heads_vs": 3, "heads_pe": 1, "groups_pe": 1,
            "h2d": 64, "d2h": 32,
            "rates": {k: 100.0 / f for k in bench.RATE_KEYS}}


def _agg_worker(rank, world, port, heads_mode, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q.put((rank, bench.aggregate(_fake_measurement(rank), world, heads_mode, dist, None)))
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("heads_mode", [False, True])
def test_two_rank_aggregation_max_times_min_rates(heads_mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_agg_worker, args=(r, 2, port, heads_mode, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    a0, a1 = res[0], res[1]
    assert a0 == a1                                   # every rank holds the same numbers
    assert a0["step"] == 22.0 and a0["dense"] == 40.0 and a0["route"] == 1.0   # the slower rank's times
    assert a0["attn_tflops"] == 50.0                  # the slower rank's rate
    if heads_mode:                                    # one layer split by KV group: work adds up
        assert a0["tiles"] == 201 and a0["causal_pairs"] == 8000 and a0["heads_vs"] == 6
    else:                                             # one layer per rank: one layer's counts
        assert a0["tiles"] == 101 and a0["causal_pairs"] == 4000 and a0["heads_vs"] == 3


def test_result_line_has_every_contract_key():
    """The JSON line bench.py prints, built from made-up measurements without a
    GPU: every key of the contract is present and serialisable."""
    import json
    m = {"clocks": {"sm_mhz": 1700.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 10,
                    "power_w_max": 1000.0},
         "sms": 148, "h_q": 32, "h_kv": 8, "route_bytes": 1233649664, "selection_bytes": 1358954496,
         "nb": 4096, "heads_pe": 8}
    a = {"step": 1800.0, "att": 1798.0, "sel": 1.4, "dense": 2000.0, "e2e": 1830.0, "route": 0.5,
         "step_median": 1801.0, "dense_median": 2001.0, "attn_tflops": 950.0, "useful_tflops": 800.0,
         "dense_tflops": 1100.0, "route_gbs": 2400.0, "pe_gbs": 1500.0, "mufu_frac": 0.5,
         "tiles": 202210861, "pairs": 2836148043072, "union_tiles": 111068154, "causal_tiles": 268500992,
         "causal_pairs": 4398054899712, "heads_vs": 24, "heads_pe": 8, "groups_pe": 2,
         "h2d": 6442450944, "d2h": 4294967296}
    res = bench.result_line("E", a, m, 1, False, 1.0, 0.95, 10, 3)
    json.dumps(res)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in res, key
    assert res["value"] == 1800.0 and res["higher_is_better"] is False
    assert set(res["roofline"]) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}
    assert set(res["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    assert res["selection_roofline"]["map_entries"] == 8 * 4096 * 4097 // 2
    assert res["gpu_launches"] == 10 * ((bench.SELECT_KERNELS + 1) + 1 + (bench.SELECT_KERNELS + 1) * 8)
