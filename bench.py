"""Benchmark: CRISP sparse-prefill attention, ms per layer, and speedup over
the dense causal attention kernel built the same way, on one B200 per rank.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config E|all] [--impl crisp|reference]
                    [--alpha A] [--gamma G] [--sweep] [--shard layers|heads]

One step = one pass of the whole hot path over one synthetic layer: proxy map,
route, VS/PE selection and block-sparse attention (crisp_select then
crisp_attend, with an event between them so the attention kernel is timed
live). Inputs stay resident in HBM; they are far larger than L2 at every
full-size layer, so no flush is needed between steps. Every timed step also
runs, right after the CRISP step and on the same stream, the dense reference
(crisp_dense_attention) and the end-to-end call (crisp_prefill_host from
page-locked host buffers, copies included), so all three are timed over the
same K steps, interleaved, each with its own CUDA events.

With --gpus N > 1 the script starts N ranks itself (torch.distributed.run,
one process per GPU) unless it already runs under a launcher. By default
every rank runs its own layer (weak scaling, no collective on the data path);
the step time is the max over ranks and the reported ms/layer divides it by
N. ``--shard heads`` instead splits one layer across the ranks by KV group
(strong scaling: each rank draws and runs only its groups; the layer's time
is the slowest rank's).

``--config all`` prints one line per configuration (A-E); ``--sweep`` one
line per (alpha, gamma) in {1.0, 1.25, 1.5} x {0.95, 0.97} on one layer.

``--impl reference`` times the CPU oracle (float64, host cores): every step
is a bounded sample of the same workload (the index of one VS and one PE
head and exact attention on a few query rows of each), scaled to ms/layer.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import crisp_synth as S  # noqa: E402

METRIC = "sparse-prefill attention ms/layer & speedup vs in-run dense kernel, 128K–512K"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PAGES_SPEEDUP_512K = 5.30   # the pages' figure on a single H100 (context only)
# kernels of one crisp_select: proxy 1, finalise 2, VS select 1,
# PE 12 (pool, 5 sweeps, 3 bucket searches, tie rows, tie scan, mask fill)
SELECT_KERNELS = 16
SWEEP = [(1.0, 0.95), (1.0, 0.97), (1.25, 0.95), (1.25, 0.97), (1.5, 0.95), (1.5, 0.97)]
ALL_CONFIGS = ["A", "B", "C", "D", "E"]
# FP32 lanes per SM (the CUDA-core attention of fp32 layers is bound by FFMA issue)
FP32_LANES_PER_SM = 128


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        return parse_clock_lines(self.lines)


def parse_clock_lines(lines):
    """Median SM clock under load (power above 250 W), max clock and the
    throttle reasons seen, from nvidia-smi csv lines."""
    sm, smax, reasons, power = [], [], set(), []
    for ln in lines:
        parts = [p.strip() for p in ln.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            smax.append(float(parts[2]))
            power.append(float(parts[3]))
        except ValueError:
            continue
        for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                             parts[5:9]):
            if val.lower().startswith("active"):
                reasons.add(name)
    loaded = [s for s, p in zip(sm, power) if p > 250] or sm
    return {"sm_mhz": statistics.median(loaded) if loaded else None,
            "sm_max_mhz": max(smax) if smax else None,
            "reasons": sorted(reasons), "samples": len(sm),
            "power_w_max": max(power) if power else None}


# ----------------------------------------------------------------------------- schedule statistics

def unpack_bits(words, nb):
    w = np.ascontiguousarray(words).astype(np.uint32)
    bits = ((w[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool)
    return bits.reshape(*w.shape[:-1], w.shape[-1] * 32)[..., :nb]


# (query, key) pairs inside one 128x128 tile of each kind the attention kernel computes
PAIRS_FULL, PAIRS_LOWER, PAIRS_UPPER = 128 * 128, 128 * 129 // 2, 128 * 127 // 2


def schedule_stats(route, vs_mask, pe_mask, nb):
    """Work of the sparse schedule, summed over heads, by the kernel's rule:
    VS keeps key tile t of query tile I whole when column block t is selected,
    the part c <= r when offset block I-t is, the part c > r when offset block
    I-t-1 is; PE keeps tile (I, t) when block (I, t) is; the diagonal tile
    (its causal half) always.

    Returns computed 128x128 tiles, selected (query, key) pairs, and the tiles
    of the union schedules of the query-tile pairs (I, I-1) one CTA computes."""
    tiles = pairs = union = 0
    I = np.arange(nb)[:, None]
    t = np.arange(nb)[None, :]
    causal = t <= I
    below = t < I
    diag = np.arange(nb)
    for h in range(len(route)):
        if route[h] == 1:
            full = unpack_bits(pe_mask[h], nb) & below
            lower = np.zeros_like(full)
            upper = np.zeros_like(full)
        else:
            v = unpack_bits(vs_mask[h, 0], nb)
            s = unpack_bits(vs_mask[h, 1], nb)
            lo = s[np.clip(I - t, 0, nb - 1)] & below
            hi = s[np.clip(I - t - 1, 0, nb - 1)] & (I - t - 1 >= 0)
            vcol = v[t] & below
            full = vcol | (lo & hi)
            lower = ~full & lo
            upper = ~full & hi & ~lo
        kept = full | lower | upper
        kept[diag, diag] = True
        tiles += int(kept.sum())
        pairs += (int(full.sum()) * PAIRS_FULL + int(lower.sum()) * PAIRS_LOWER + int(upper.sum()) * PAIRS_UPPER
                  + nb * PAIRS_LOWER)
        # CTA pairs: query tiles (nb-1, nb-2), (nb-3, nb-4), ...; the union over both rows
        ia = np.arange(nb - 1, -1, -2)
        ib = ia - 1
        u = kept[ia].copy()
        has_b = ib >= 0
        u[has_b] |= kept[ib[has_b]]
        union += int(u.sum())
    return tiles, pairs, union


def kernel_source_hash(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "long_context_prefill_last_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# dram__bytes_read.sum + dram__bytes_write.sum per attention launch, measured
# by ncu on a scaled case of the layer (one KV group, the same n) and scaled by
# the KV groups; valid only for the kernel source it was taken on. Layer E:
# a planted group 12791037952 + 529213440 bytes, a Gaussian group
# 453424689664 + 533230848 bytes; 6 planted and 2 Gaussian groups.
MEASURED_TRAFFIC = {
    ("attn_tc_kernel", "E", 1.0, 0.95): {
        "source_hash": "d8a76d3717b90444",
        "bytes_per_launch": 6 * (12791037952 + 529213440) + 2 * (453424689664 + 533230848),
    },
}


def load_traffic(kernel, src_hash, config, alpha, gamma):
    """DRAM bytes per launch measured on this kernel source and workload, else None."""
    e = MEASURED_TRAFFIC.get((kernel, config, float(alpha), float(gamma)))
    if not e or e["source_hash"] != src_hash:
        return None
    return e["bytes_per_launch"]


def mufu_roofline(exps, ms, clk, sms):
    """Exponentials per second against the MUFU rate (16 per clock per SM) at the sampled SM clock."""
    mhz = clk.get("sm_mhz") or clk.get("sm_max_mhz")
    if not mhz or ms <= 0:
        return None
    peak = 16.0 * sms * mhz * 1e6
    achieved = exps / (ms * 1e-3)
    return {"exps": int(exps), "achieved_per_s": round(achieved / 1e12, 3), "peak_per_s": round(peak / 1e12, 3),
            "unit": "T exp2/s", "frac": round(achieved / peak, 4), "clock_mhz": mhz}


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((i.get("num_threads") or 1) for i in threadpool_info()) if threadpool_info() else 1
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def config_dict(name, alpha, gamma, world=1, heads_mode=False):
    """The workload description shared by both arms."""
    c = S.CONFIGS[name]
    slash_note = ("planted slash offsets dealt round-robin over the planted KV groups "
                  f"({c.n_slash} per layer, about {max(1, c.n_slash // max(1, len(c.planted_groups)))} per planted "
                  "group); verticals per planted group as named")
    return {"workload": f"layer {name}: {c.desc}", "h_q": c.h_q, "h_kv": c.h_kv, "seq_len": c.n,
            "alpha": alpha, "gamma": gamma, "head_dim": c.d, "batch": 1,
            "parallelism": (f"one layer split by KV group over {world} GPUs (no exchange)" if heads_mode
                            else f"independent layer per GPU x{world}"),
            "structure": slash_note,
            "l2": ("inputs far exceed the 126 MB L2 at every full-size layer; no flush between steps" if c.n >= 32768
                   else "small layer: inputs fit in L2 (no flush); timings are launch-bound")}


# ----------------------------------------------------------------------------- CPU oracle baseline

class OracleSampler:
    """The oracle on a bounded sample of a layer, scaled to ms/layer.

    One sample: the proxy/route/selection of one planted (VS) head and one
    Gaussian (PE) head, and exact sparse attention for `rows` random query
    rows of each. Scaled: index time per head x heads of each kind, plus
    attention time per row x rows x heads (the oracle's attention cost per row
    grows with the selected keys; rows are drawn uniformly over the sequence,
    so their mean matches the layer's)."""

    def __init__(self, cfg_name, alpha=1.0, gamma=0.95, threads=8):
        from oracle import crisp_oracle as O
        self.O = O
        c = S.CONFIGS[cfg_name]
        self.c = c
        self.name = cfg_name
        # one KV group of each kind is enough: a 2-group slice of the layer
        small = dataclasses.replace(c, h_q=2 * c.group, h_kv=2, planted_groups=(0,),
                                    slash_groups=len(c.planted_groups) if c.planted_groups else 0)
        if len(c.planted_groups) == c.h_kv:
            small = dataclasses.replace(small, planted_groups=(0, 1))
        self.layer = S.generate(small, threads=threads)
        self.ocfg = O.OracleCfg(alpha=alpha, gamma=gamma)
        G = c.group
        self.heads = {"vs": 0, "pe": G} if c.h_q > 1 else {"vs": 0}
        self.n_vs = len(c.planted_groups) * G
        self.n_pe = c.h_q - self.n_vs
        self.rng = np.random.default_rng(0)
        self.rows_done = {k: 0 for k in self.heads}

    def sample(self, rows=8):
        """One bounded sample; returns (its wall seconds, the ms/layer it extrapolates to)."""
        O, c, G = self.O, self.c, self.c.group
        t_start = time.perf_counter()
        t_index, t_row = {}, {}
        for kind, h in self.heads.items():
            q = self.layer.as_f64("q", h)
            k = self.layer.as_f64("k", h // G)
            v = self.layer.as_f64("v", h // G)
            t0 = time.perf_counter()
            idx = O.head_index(q, k, self.ocfg)
            t_index[kind] = time.perf_counter() - t0
            r = np.sort(self.rng.choice(c.n, size=min(rows, c.n), replace=False))
            t0 = time.perf_counter()
            O.head_attention(q, k, v, idx, r, self.ocfg, chunk=8)
            t_row[kind] = (time.perf_counter() - t0) / len(r)
            self.rows_done[kind] += len(r)
        if "pe" not in t_index:   # a one-head layer
            t_index["pe"], t_row["pe"] = t_index["vs"], t_row["vs"]
        n_vs = self.n_vs if c.h_q > 1 else c.h_q
        n_pe = self.n_pe if c.h_q > 1 else 0
        total_s = (n_vs * (t_index["vs"] + c.n * t_row["vs"]) + n_pe * (t_index["pe"] + c.n * t_row["pe"]))
        return time.perf_counter() - t_start, total_s * 1e3

    def describe(self):
        parts = " + ".join(str(v) for v in self.rows_done.values())
        kinds = "one planted (VS) and one Gaussian (PE) head" if len(self.heads) == 2 else "the layer's one head"
        return (f"{kinds} of layer {self.name}: full proxy/route/selection, exact attention on {parts} random "
                f"query rows; scaled to {self.c.h_q} heads x {self.c.n} rows")


def oracle_ms_per_layer(cfg_name, budget_s=20.0, alpha=1.0, gamma=0.95):
    """The cpu_baseline leg: samples until about budget_s seconds of CPU work."""
    smp = OracleSampler(cfg_name, alpha, gamma)
    est, spent = [], 0.0
    while spent < budget_s or not est:
        dt, ms = smp.sample()
        spent += dt
        est.append(ms)
    return statistics.mean(est), smp.describe(), spent


def run_reference(args, rank, world):
    """The reference arm: the oracle as it stands, on the host cores; each
    step one bounded sample. Under a launcher only rank 0 works."""
    if rank != 0:
        return
    cfg_name = "E" if args.config == "all" else args.config
    smp = OracleSampler(cfg_name, args.alpha, args.gamma)
    for _ in range(args.warmup):
        smp.sample(rows=4)
    walls, est = [], []
    for _ in range(args.steps):
        dt, ms = smp.sample(rows=4)
        walls.append(dt)
        est.append(ms)
    value = statistics.mean(est)
    cores = cpu_cores()
    res = {"metric": METRIC, "value": round(value, 1), "unit": "ms/layer", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup,
           # the wall time of one sample step (the scaled per-layer estimate is `value`)
           "ms_per_step": round(statistics.mean(walls) * 1e3, 1),
           "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "impl": "reference",
           "config": config_dict(cfg_name, args.alpha, args.gamma, world, args.shard == "heads" and world > 1),
           "cpu_baseline": {"value": round(value, 1), "unit": "ms/layer", "cores": cores, "kind": "oracle",
                            "sample": smp.describe() + " (one sample per step)"},
           "e2e": {"value": round(value, 1), "unit": "ms/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


# ----------------------------------------------------------------------------- GPU arm

def load_layer(cfg_name, rank, world, heads_mode):
    """Host tensors (q, k, v) of this rank's layer or slice, and its (h_q, h_kv)."""
    import torch
    from long_context_prefill_last_b200 import shard
    c = S.CONFIGS[cfg_name]
    # the ranks of one node generate their inputs at the same time: share the cores
    local_world = max(1, int(os.environ.get("LOCAL_WORLD_SIZE", "1")))
    threads = max(2, min(32, (os.cpu_count() or 8) // local_world))
    if heads_mode:
        if world > c.h_kv:
            raise SystemExit(f"--shard heads needs at most {c.h_kv} ranks for layer {cfg_name}")
        g_lo, g_hi = shard.kv_group_range(c.h_kv, world, rank)
        arrays = S.generate_slice(c, g_lo, g_hi, threads=threads)
        h_q, h_kv = (g_hi - g_lo) * c.group, g_hi - g_lo
        if c.dtype == "bf16":
            q_h, k_h, v_h = (torch.from_numpy(a).view(torch.bfloat16) for a in arrays)
        else:
            q_h, k_h, v_h = (torch.from_numpy(a) for a in arrays)
    else:
        layer = S.generate(c, threads=threads)
        q_h, k_h, v_h = S.to_torch(layer)
        h_q, h_kv = c.h_q, c.h_kv
    return (q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()), h_q, h_kv


def measure(cfg_name, host, h_q, h_kv, alpha, gamma, steps, warmup, local_rank, barrier):
    """Time K interleaved steps (CRISP step, dense reference, end-to-end) on
    this rank; returns the per-rank measurements."""
    import torch
    import long_context_prefill_last_b200 as crisp

    c = S.CONFIGS[cfg_name]
    dev = torch.device("cuda", local_rank)
    q_h, k_h, v_h = host
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    out = torch.empty_like(q)
    out_dense = torch.empty_like(q)
    out_h = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    dtype = crisp.FP32 if c.dtype == "fp32" else crisp.BF16
    cfg = crisp.Config(n=c.n, h_q=h_q, h_kv=h_kv, d=c.d, dtype=dtype, alpha=alpha, gamma=gamma)
    cfg.allocate_workspace(dev)
    dcfg = crisp.Config(n=c.n, h_q=h_q, h_kv=h_kv, d=c.d, dtype=dtype, alpha=alpha, gamma=gamma)
    dcfg.allocate_workspace(dev)
    hcfg = crisp.Config(n=c.n, h_q=h_q, h_kv=h_kv, d=c.d, dtype=dtype, alpha=alpha, gamma=gamma)
    hcfg.allocate_workspace(dev, host=True)
    ix = crisp.IndexBuffers(cfg, dev)
    stream = torch.cuda.current_stream(dev)
    copy_stream = torch.cuda.Stream(device=dev)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    def one_step(evs=None):
        e = evs or [None] * 7

        def rec(i):
            if e[i] is not None:
                e[i].record(stream)
        rec(0)
        crisp.select(q, k, cfg, ix, stream)
        rec(1)
        crisp.attend(q, k, v, out, cfg, ix, stream)
        rec(2)
        crisp.dense_attention(q, k, v, out_dense, dcfg, stream)
        rec(3)
        rec(4)
        crisp.prefill_host(q_h, k_h, v_h, out_h, hcfg, stream, copy_stream)
        rec(5)

    for _ in range(warmup):
        one_step()
    crisp.raise_on_device_status(cfg, stream, "warm-up")
    crisp.raise_on_device_status(dcfg, stream, "warm-up dense")
    crisp.raise_on_device_status(hcfg, stream, "warm-up e2e")
    route = ix.route.cpu().numpy()
    tiles, pairs, union = schedule_stats(route, ix.vs_mask.cpu().numpy().view(np.uint32),
                                         ix.pe_mask.cpu().numpy().view(np.uint32), cfg.n_blocks)
    nb = cfg.n_blocks

    clocks = ClockSampler(local_rank)
    clocks.start()
    barrier()
    torch.cuda.synchronize(dev)
    evs = [[ev() for _ in range(7)] for _ in range(steps)]
    for e in evs:
        one_step(e)
    torch.cuda.synchronize(dev)
    barrier()
    crisp.raise_on_device_status(cfg, stream, "timed steps")
    crisp.raise_on_device_status(dcfg, stream, "timed dense")
    crisp.raise_on_device_status(hcfg, stream, "timed e2e")
    step_ms = [e[0].elapsed_time(e[2]) for e in evs]
    sel_ms = [e[0].elapsed_time(e[1]) for e in evs]
    att_ms = [e[1].elapsed_time(e[2]) for e in evs]
    dense_ms = [e[2].elapsed_time(e[3]) for e in evs]
    e2e_ms = [e[4].elapsed_time(e[5]) for e in evs]

    # the route pass alone (proxy map + finalisation + route/VS masses)
    r_out = torch.empty(h_q, dtype=torch.int32, device=dev)
    c_out = torch.empty(h_q, dtype=torch.float32, device=dev)
    crisp.route(q, k, cfg, r_out, c_out, stream)
    torch.cuda.synchronize(dev)
    rev = [(ev(), ev()) for _ in range(steps)]
    for a, b in rev:
        a.record(stream)
        crisp.route(q, k, cfg, r_out, c_out, stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    route_ms = [a.elapsed_time(b) for a, b in rev]
    crisp.raise_on_device_status(cfg, stream, "route")
    clk = clocks.stop()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    n_pe = int((route == 1).sum())
    g_pe = len({h // (h_q // h_kv) for h in range(h_q) if route[h] == 1})
    h2d = int(sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h)))
    d2h = int(out_h.numel() * out_h.element_size())
    causal_tiles = h_q * nb * (nb + 1) // 2
    mean = statistics.mean
    att, dense, rt = mean(att_ms), mean(dense_ms), mean(route_ms)
    pe = max(mean(sel_ms) - rt, 1e-6)
    rb = route_bytes(h_q, h_kv, c.n, c.d, nb)
    sb = selection_bytes(n_pe, g_pe, c.n, c.d, nb, cfg.words)
    # this rank's rates (per GPU)
    rates = {"attn_tflops": 4.0 * c.d * 128 * 128 * tiles / (att * 1e-3) / 1e12,
             "useful_tflops": 4.0 * c.d * pairs / (att * 1e-3) / 1e12,
             "dense_tflops": 4.0 * c.d * 128 * 128 * causal_tiles / (dense * 1e-3) / 1e12,
             "route_gbs": rb / (rt * 1e-3) / 1e9, "pe_gbs": sb / (pe * 1e-3) / 1e9,
             "mufu_frac": (mufu_roofline(h_q * 64 * c.n, rt, clk, sms) or {}).get("frac", 0.0)}
    return {"step_ms": step_ms, "sel_ms": sel_ms, "att_ms": att_ms, "dense_ms": dense_ms, "e2e_ms": e2e_ms,
            "route_ms": route_ms, "tiles": tiles, "pairs": pairs, "union_tiles": union,
            "causal_tiles": causal_tiles, "causal_pairs": h_q * c.n * (c.n + 1) // 2,
            "heads_vs": int((route == 0).sum()), "heads_pe": n_pe, "groups_pe": g_pe,
            "h_q": h_q, "h_kv": h_kv, "clocks": clk, "sms": sms, "h2d": h2d, "d2h": d2h,
            "words": cfg.words, "nb": nb, "route_bytes": rb, "selection_bytes": sb, "rates": rates}


def route_bytes(h_q, h_kv, n, d, nb):
    """Algorithmic HBM bytes of the route pass: K read once, the proxy rows of
    Q read once, the per-(row, tile) partials written and read back, and the
    per-chunk statistics."""
    rows = h_q * 64
    return h_kv * n * d * 2 + rows * d * 2 + 2 * rows * nb * 8 + rows * ((nb + 7) // 8) * 24


def selection_bytes(n_pe, g_pe, n, d, nb, words):
    """Algorithmic HBM bytes of the PE pass: the PE heads' Q and their groups'
    K read once (block pooling) and the PE masks written once."""
    return (n_pe + g_pe) * n * d * 2 + n_pe * nb * words * 4


RATE_KEYS = ["attn_tflops", "useful_tflops", "dense_tflops", "route_gbs", "pe_gbs", "mufu_frac"]


def aggregate(m, world, heads_mode, dist=None, device=None):
    """Combine the per-rank measurements: times are the maximum over ranks,
    rates (per GPU) the minimum, i.e. the slowest rank's; with the layer split
    by KV group, work counts add up (otherwise every rank's counts describe
    one whole layer and are equal). Returns the combined numbers, identical
    on every rank."""
    import torch
    mean = statistics.mean
    vals = torch.tensor([mean(m["step_ms"]), mean(m["att_ms"]), mean(m["sel_ms"]), mean(m["dense_ms"]),
                         mean(m["e2e_ms"]), mean(m["route_ms"]), statistics.median(m["step_ms"]),
                         statistics.median(m["dense_ms"])], dtype=torch.float64, device=device)
    rates = torch.tensor([m["rates"][k] for k in RATE_KEYS], dtype=torch.float64, device=device)
    counts = torch.tensor([m["tiles"], m["pairs"], m["union_tiles"], m["causal_tiles"], m["causal_pairs"],
                           m["heads_vs"], m["heads_pe"], m["groups_pe"], m["h2d"], m["d2h"]],
                          dtype=torch.float64, device=device)
    if world > 1 and dist is not None:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
        dist.all_reduce(rates, op=dist.ReduceOp.MIN)
        dist.all_reduce(counts, op=dist.ReduceOp.SUM if heads_mode else dist.ReduceOp.MAX)
    keys_v = ["step", "att", "sel", "dense", "e2e", "route", "step_median", "dense_median"]
    keys_c = ["tiles", "pairs", "union_tiles", "causal_tiles", "causal_pairs", "heads_vs", "heads_pe",
              "groups_pe", "h2d", "d2h"]
    out = dict(zip(keys_v, vals.tolist()))
    out.update(zip(RATE_KEYS, rates.tolist()))
    out.update(zip(keys_c, (int(x) for x in counts.tolist())))
    return out


def result_line(cfg_name, a, m, world, heads_mode, alpha, gamma, steps, warmup):
    """The JSON line of the CRISP arm from the aggregated numbers `a` (and
    rank 0's own measurements `m` for the clocks)."""
    c = S.CONFIGS[cfg_name]
    peaks, peak_src = load_peaks()
    tflops_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    hbm_peak = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    clk = m["clocks"]
    fp32 = c.dtype == "fp32"
    achieved = a["attn_tflops"]
    if fp32:
        mhz = clk.get("sm_max_mhz") or 1965.0
        peak = m["sms"] * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12
        roof = {"kernel": "attn_simt_kernel (block-sparse attention, fp32 CUDA cores)", "bound": "alu",
                "achieved": round(achieved, 3), "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": None,
                "peak_source": f"derived: {m['sms']} SMs x {FP32_LANES_PER_SM} FP32 lanes x 2 flop x {mhz:g} MHz",
                "work": "4*d*128*128 flop per computed 128x128 tile x computed tiles per launch"}
    else:
        src_hash = kernel_source_hash(["attn_tc.cu", "ptx.cuh"])
        traffic = load_traffic("attn_tc_kernel", src_hash, cfg_name, alpha, gamma) if not heads_mode else None
        roof = {"kernel": "attn_tc_kernel (block-sparse attention)", "bound": "tensor",
                "achieved": round(achieved, 2), "peak": tflops_peak, "unit": "TFLOP/s",
                "frac": round(achieved / tflops_peak, 4), "traffic": traffic,
                "peak_source": f"{peak_src} bf16 dense, sustained (kernel runs inside a seconds-long step)",
                "work": "4*d*128*128 flop per computed 128x128 tile x computed tiles per launch"}
    mufu = mufu_roofline(m["h_q"] * 64 * c.n, a["route"], clk, m["sms"])
    if mufu is not None:
        mufu["frac"] = round(a["mufu_frac"], 4)
    pe_ms = max(a["sel"] - a["route"], 1e-6)
    per_layer = 1 if heads_mode else world
    res = {
        "metric": METRIC,
        "value": round(a["step"] / per_layer, 4),
        "unit": "ms/layer",
        "n_gpus": world,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": round(a["step"], 4),
        "higher_is_better": False,
        "scaling": "strong" if heads_mode else "weak",
        "vs_baseline": None,
        "dtype": "f32" if fp32 else "bf16",
        "data": ("synthetic (seeded Gaussian heads with planted sink/vertical/slash structure"
                 + (f", log-normal block background sigma {c.cliff_sigma:g}" if c.cliff_sigma > 0 else "")
                 + "; no datasets or weights)"),
        "config": config_dict(cfg_name, alpha, gamma, world, heads_mode),
        "speedup_vs_dense": round(a["dense"] / a["step"], 4),
        "speedup_vs_dense_median": round(a["dense_median"] / a["step_median"], 4),
        "dense_ms_per_layer": round(a["dense"] / per_layer, 4),
        "timing": f"{steps} interleaved steps: CRISP step, dense attention, end-to-end call; means (medians also given)",
        "stages_ms": {"proxy_route_select": round(a["sel"], 4), "sparse_attention": round(a["att"], 4),
                      "crisp_step_median": round(a["step_median"], 4), "dense_median": round(a["dense_median"], 4)},
        "density": {"computed_tiles": a["tiles"], "causal_tiles": a["causal_tiles"],
                    "fraction": round(a["tiles"] / a["causal_tiles"], 4),
                    "useful_pairs": a["pairs"], "causal_pairs": a["causal_pairs"],
                    "useful_pair_fraction": round(a["pairs"] / a["causal_pairs"], 4),
                    "cta_union_tiles": a["union_tiles"],
                    "heads_vs": a["heads_vs"], "heads_pe": a["heads_pe"]},
        "effective_tflops": {
            "dense_equivalent": round(4.0 * c.d * a["causal_pairs"] / (a["step"] / per_layer * 1e-3) / 1e12, 2),
            "useful_pairs": round(a["useful_tflops"], 2),
            "computed_tiles": round(achieved, 2),
            "note": "dense-equivalent = 4*d*causal pairs / CRISP step time; useful = 4*d*selected pairs / "
                    "attention time; computed = 4*d*128*128*computed tiles / attention time"},
        "pages_speedup_context": f"{PAGES_SPEEDUP_512K}x at 512K tokens on one H100 (pages' figure, not comparable)",
        "roofline": roof,
        "dense_tflops": round(a["dense_tflops"], 2),
        "route_roofline": {"stage": "crisp_route (proxy map + finalize + VS masses)", "bound": "hbm",
                           "ms": round(a["route"], 4), "algorithmic_bytes": m["route_bytes"],
                           "achieved": round(a["route_gbs"], 1), "peak": hbm_peak,
                           "unit": "GB/s", "frac": round(a["route_gbs"] / hbm_peak, 4),
                           "mufu": mufu},
        "selection_roofline": {"stage": "PE pooling, pooled map, gamma cut, masks (select minus route)",
                               "bound": "hbm", "ms": round(pe_ms, 4), "algorithmic_bytes": m["selection_bytes"],
                               "achieved": round(a["pe_gbs"], 1), "peak": hbm_peak, "unit": "GB/s",
                               "frac": round(a["pe_gbs"] / hbm_peak, 4),
                               "work": "PE heads' Q and their groups' K read once, PE masks written once",
                               "map_entries": a["heads_pe"] * m["nb"] * (m["nb"] + 1) // 2,
                               "map_note": "pooled-map entries evaluated per pass (statistics, level 0; later "
                                           "passes recompute only the tiles the prefix or the cut crosses): "
                                           "compute the byte count does not include"},
        "e2e": {"value": round(a["e2e"] / per_layer, 4), "unit": "ms/layer", "h2d_bytes_per_step": a["h2d"],
                "d2h_bytes_per_step": a["d2h"],
                "api": "crisp_prefill_host: page-locked host buffers, copies overlapped with the kernels per KV group"},
        # per step: crisp_select + crisp_attend, the dense launch, crisp_prefill_host (one select+attend per KV group)
        "gpu_launches": steps * ((SELECT_KERNELS + 1) + 1 + (SELECT_KERNELS + 1) * m["h_kv"]),
        "clocks": {k: clk.get(k) for k in ("sm_mhz", "sm_max_mhz", "reasons", "samples", "power_w_max")},
    }
    return res


def init_dist(world):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    return dist


def run_configs(args, rank, world, local_rank, cfg_names, settings):
    """Measure every (config, alpha, gamma); rank 0 prints one JSON line each."""
    import torch
    torch.cuda.set_device(local_rank)
    dist = init_dist(world)
    heads_mode = args.shard == "heads" and world > 1

    def barrier():
        if dist is not None:
            dist.barrier()

    try:
        for name in cfg_names:
            host, h_q, h_kv = load_layer(name, rank, world, heads_mode)
            for alpha, gamma in settings:
                m = measure(name, host, h_q, h_kv, alpha, gamma, args.steps, args.warmup, local_rank, barrier)
                a = aggregate(m, world, heads_mode, dist, torch.device("cuda", local_rank))
                if rank == 0:
                    res = result_line(name, a, m, world, heads_mode, alpha, gamma, args.steps, args.warmup)
                    if world == 1 and not args.no_cpu_baseline and len(cfg_names) == 1 and len(settings) == 1:
                        ms, sample, _ = oracle_ms_per_layer(name, budget_s=20.0, alpha=alpha, gamma=gamma)
                        res["cpu_baseline"] = {"value": round(ms, 1), "unit": "ms/layer", "cores": cpu_cores(),
                                               "kind": "oracle", "sample": sample}
                    print(json.dumps(res), flush=True)
                torch.cuda.empty_cache()
            del host
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()


def run_stage(args):
    """Time one stage on a (possibly scaled) layer; used for ncu captures."""
    import torch
    import long_context_prefill_last_b200 as crisp
    c = S.CONFIGS[args.config]
    if args.n or args.h_q or args.h_kv or args.planted is not None:
        pg = None if args.planted is None else [int(x) for x in args.planted.split(",") if x.strip()]
        c = S.scaled(args.config, n=args.n, h_q=args.h_q, h_kv=args.h_kv, planted_groups=pg)
    layer = S.generate(c, threads=min(32, os.cpu_count() or 8))
    q, k, v = (t.cuda() for t in S.to_torch(layer))
    out = torch.empty_like(q)
    cfg = crisp.Config(n=c.n, h_q=c.h_q, h_kv=c.h_kv, dtype=crisp.FP32 if c.dtype == "fp32" else crisp.BF16,
                       alpha=args.alpha, gamma=args.gamma)
    cfg.allocate_workspace()
    ix = crisp.IndexBuffers(cfg)
    crisp.select(q, k, cfg, ix)
    route_out = torch.empty(c.h_q, dtype=torch.int32, device="cuda")
    cs_out = torch.empty(c.h_q, dtype=torch.float32, device="cuda")
    fn = {"select": lambda: crisp.select(q, k, cfg, ix),
          "route": lambda: crisp.route(q, k, cfg, route_out, cs_out),
          "attend": lambda: crisp.attend(q, k, v, out, cfg, ix),
          "dense": lambda: crisp.dense_attention(q, k, v, out, cfg),
          "prefill": lambda: crisp.prefill(q, k, v, out, cfg)}[args.only]
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    crisp.raise_on_device_status(cfg, where=args.only)
    ms = a.elapsed_time(b) / max(1, args.steps)
    print(json.dumps({"stage": args.only, "layer": c.name, "n": c.n, "h_q": c.h_q, "h_kv": c.h_kv,
                      "ms": round(ms, 4)}))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def launch_command(n_gpus, argv, port=None):
    """The command that runs this script on n_gpus ranks of this node (one
    process per GPU, rendezvous on 127.0.0.1), bounded by `timeout`."""
    port = port or _free_port()
    return ["timeout", "-k", "60", "3600", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={n_gpus}", "--master-addr", "127.0.0.1", "--master-port", str(port),
            os.path.abspath(__file__), *argv]


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="E", choices=sorted(S.CONFIGS) + ["all"])
    ap.add_argument("--impl", default="crisp", choices=["crisp", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--alpha", type=float, default=1.0, help="Eq. (4) noise-floor multiplier")
    ap.add_argument("--gamma", type=float, default=0.95, help="PE cumulative coverage")
    ap.add_argument("--sweep", action="store_true",
                    help="one line per (alpha, gamma) in {1.0, 1.25, 1.5} x {0.95, 0.97}")
    ap.add_argument("--shard", choices=["layers", "heads"], default="layers",
                    help="with N > 1 GPUs: an independent layer per GPU (weak scaling, default) or one layer "
                         "split by KV group (strong scaling)")
    ap.add_argument("--only", choices=["select", "attend", "dense", "prefill", "route"],
                    help="profiling mode: time one stage alone (no contract line)")
    ap.add_argument("--n", type=int, help="profiling mode: scaled sequence length")
    ap.add_argument("--h-q", type=int, help="profiling mode: scaled query heads")
    ap.add_argument("--h-kv", type=int, help="profiling mode: scaled KV heads")
    ap.add_argument("--planted", help="profiling mode: comma-separated planted KV groups of the scaled layer "
                                      "('' for none: every group Gaussian)")
    return ap.parse_args(argv)


def main(argv=None):
    argv = list(sys.argv[1:] if argv is None else argv)
    args = parse_args(argv)
    if args.only:
        run_stage(args)
        return
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # not under a launcher: start one rank per GPU and wait for them
        cmd = launch_command(args.gpus, argv)
        sys.stdout.flush()
        raise SystemExit(subprocess.call(cmd))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    names = ALL_CONFIGS if args.config == "all" else [args.config]
    settings = SWEEP if args.sweep else [(args.alpha, args.gamma)]
    run_configs(args, rank, world, local_rank, names, settings)


if __name__ == "__main__":
    main()
