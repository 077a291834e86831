"""Benchmark: CRISP sparse-prefill attention, ms per layer, and speedup over
the dense causal attention kernel built the same way, on one B200 per rank.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config E] [--impl crisp|reference]

One step = one pass of the whole hot path over one synthetic layer: proxy map,
route, VS/PE selection and block-sparse attention (crisp_select then
crisp_attend, with an event between them so the attention kernel is timed
live). Inputs stay resident in HBM; they are far larger than L2 at every
full-size layer, so no flush is needed between steps. The dense reference and
the end-to-end number (crisp_prefill through host buffers, copies included)
are timed the same way. With N > 1 (torchrun) every rank runs its own layer
(weak scaling, no collective on the data path); the step time is the max over
ranks and the reported ms/layer divides it by N. ``--shard heads`` instead
splits one layer across the ranks by KV group (strong scaling: each rank draws
and runs only its groups; the layer's time is the slowest rank's).

``--impl reference`` times the CPU oracle (float64, host cores) on a bounded
sample of the same workload and scales it to ms/layer.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
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
KERNELS_PER_STEP = 17       # proxy 1, finalise 2, VS select 1, PE 12, attention 1


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
        sm, smax, reasons, power = [], [], set(), []
        for ln in self.lines:
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


# ----------------------------------------------------------------------------- helpers

def unpack_bits(words, nb):
    w = np.ascontiguousarray(words).astype(np.uint32)
    bits = ((w[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).astype(bool)
    return bits.reshape(*w.shape[:-1], w.shape[-1] * 32)[..., :nb]


def kept_tiles(route, vs_mask, pe_mask, nb):
    """Computed 128x128 tiles of the sparse schedule, summed over heads (the
    kernel's rule: VS keeps tile (I, t) when column block t or offset block
    I-t or I-t-1 is selected; PE when block (I, t) is; the diagonal always)."""
    total = 0
    I = np.arange(nb)[:, None]
    t = np.arange(nb)[None, :]
    causal = t <= I
    for h in range(len(route)):
        if route[h] == 1:
            m = unpack_bits(pe_mask[h], nb) & causal
            m[np.arange(nb), np.arange(nb)] = True
        else:
            v = unpack_bits(vs_mask[h, 0], nb)
            s = unpack_bits(vs_mask[h, 1], nb)
            off = np.clip(I - t, 0, nb - 1)
            off1 = np.clip(I - t - 1, 0, nb - 1)
            m = causal & (v[t] | s[off] | ((I - t - 1 >= 0) & s[off1]))
            m[np.arange(nb), np.arange(nb)] = True
        total += int(m.sum())
    return total


def kernel_source_hash(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "long_context_prefill_last_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# dram__bytes_read.sum + dram__bytes_write.sum of one launch, from the ncu
# capture summarised in profiles/attn_tc_traffic_layerE.md (layer E, default
# alpha and gamma); reported only for the kernel source it was taken on.
MEASURED_TRAFFIC = {
    ("attn_tc_kernel", "E", 1.0, 0.95): {"source_hash": "e805491e5011c54d", "bytes_per_launch": 949.2e9 + 4.32e9},
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


# ----------------------------------------------------------------------------- CPU oracle baseline

def oracle_ms_per_layer(cfg_name: str, budget_s: float = 20.0):
    """Time the oracle on a bounded sample of the layer and scale to ms/layer.

    Sample: the proxy/route/selection of one planted (VS) head and one
    Gaussian (PE) head, and exact sparse attention for sampled query rows of
    those heads. Scaled: index time per head x heads of each kind; attention
    time per row x rows x heads (the oracle's attention cost per row grows
    with the selected keys; rows are drawn evenly over the sequence so their
    mean matches the layer's)."""
    from oracle import crisp_oracle as O
    c = S.CONFIGS[cfg_name]
    # one KV group of each kind is enough: generate a 2-group slice of the layer
    small = S.dataclasses.replace(c, h_q=2 * c.group, h_kv=2, planted_groups=(0,),
                                  slash_groups=len(c.planted_groups) if c.planted_groups else 0)
    if len(c.planted_groups) == c.h_kv:
        small = S.dataclasses.replace(small, planted_groups=(0, 1))
    layer = S.generate(small, threads=8)
    ocfg = O.OracleCfg()
    t_index = {}
    t_rows = {}
    n = c.n
    G = c.group
    t_start = time.perf_counter()
    heads = {"vs": 0, "pe": G}
    rows_done = {"vs": 0, "pe": 0}
    for kind, h in heads.items():
        q = layer.as_f64("q", h)
        k = layer.as_f64("k", h // G)
        v = layer.as_f64("v", h // G)
        t0 = time.perf_counter()
        idx = O.head_index(q, k, ocfg)
        t_index[kind] = time.perf_counter() - t0
        # attention rows, evenly spread, until this head's share of the budget is used
        rng = np.random.default_rng(0)
        t_att = 0.0
        nrows = 0
        while t_att < budget_s / 4 and nrows < n:
            rows = np.sort(rng.choice(n, size=8, replace=False))
            t0 = time.perf_counter()
            O.head_attention(q, k, v, idx, rows, ocfg, chunk=8)
            t_att += time.perf_counter() - t0
            nrows += len(rows)
        t_rows[kind] = t_att / nrows
        rows_done[kind] = nrows
    n_vs = len(c.planted_groups) * G
    n_pe = c.h_q - n_vs
    total_s = n_vs * (t_index["vs"] + n * t_rows["vs"]) + n_pe * (t_index["pe"] + n * t_rows["pe"])
    sample = (f"one planted (VS) and one Gaussian (PE) head of layer {cfg_name}: full proxy/route/selection, "
              f"exact attention on {rows_done['vs']} + {rows_done['pe']} random query rows; "
              f"scaled to {c.h_q} heads x {n} rows")
    return total_s * 1e3, sample, time.perf_counter() - t_start


# ----------------------------------------------------------------------------- GPU arm

def run_crisp(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import long_context_prefill_last_b200 as crisp
    from long_context_prefill_last_b200 import shard

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    c = S.CONFIGS[args.config]
    threads = min(32, os.cpu_count() or 8)
    heads_mode = args.shard == "heads" and world > 1
    if heads_mode:
        # one layer split by KV group: this rank draws and runs only its groups
        if world > c.h_kv:
            raise SystemExit(f"--shard heads needs at most {c.h_kv} ranks for layer {args.config}")
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
    q_h, k_h, v_h = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    out = torch.empty_like(q)
    out_h = torch.empty(q.shape, dtype=q.dtype).pin_memory()
    dtype = crisp.FP32 if c.dtype == "fp32" else crisp.BF16
    cfg = crisp.Config(n=c.n, h_q=h_q, h_kv=h_kv, d=c.d, dtype=dtype, alpha=args.alpha, gamma=args.gamma)
    cfg.allocate_workspace(dev)
    ix = crisp.IndexBuffers(cfg, dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def step(ev_mid=None):
        crisp.select(q, k, cfg, ix, stream)
        if ev_mid is not None:
            ev_mid.record(stream)
        crisp.attend(q, k, v, out, cfg, ix, stream)

    # warm-up (also builds the index used for the tile count)
    for _ in range(args.warmup):
        step()
    crisp.raise_on_device_status(cfg, stream, "warm-up")
    route = ix.route.cpu().numpy()
    tiles = kept_tiles(route, ix.vs_mask.cpu().numpy().view(np.uint32), ix.pe_mask.cpu().numpy().view(np.uint32),
                       cfg.n_blocks)
    causal_tiles = h_q * cfg.n_blocks * (cfg.n_blocks + 1) // 2

    clocks = ClockSampler(local_rank)
    clocks.start()
    # --- timed: the CRISP path
    barrier()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, m, b in evs:
        a.record(stream)
        step(m)
        b.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    step_ms = [a.elapsed_time(b) for a, m, b in evs]
    sel_ms = [a.elapsed_time(m) for a, m, b in evs]
    att_ms = [m.elapsed_time(b) for a, m, b in evs]
    crisp.raise_on_device_status(cfg, stream, "timed steps")

    # --- timed: the route pass alone (proxy map + finalisation + route/VS masses)
    r_out = torch.empty(h_q, dtype=torch.int32, device=dev)
    c_out = torch.empty(h_q, dtype=torch.float32, device=dev)
    crisp.route(q, k, cfg, r_out, c_out, stream)
    torch.cuda.synchronize(dev)
    rev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in rev:
        a.record(stream)
        crisp.route(q, k, cfg, r_out, c_out, stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    route_ms = [a.elapsed_time(b) for a, b in rev]
    crisp.raise_on_device_status(cfg, stream, "route")

    # --- timed: dense reference
    for _ in range(max(1, args.warmup // 2)):
        crisp.dense_attention(q, k, v, out, cfg, stream)
    barrier()
    torch.cuda.synchronize(dev)
    dev_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.dense_steps)]
    for a, b in dev_evs:
        a.record(stream)
        crisp.dense_attention(q, k, v, out, cfg, stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    dense_ms = [a.elapsed_time(b) for a, b in dev_evs]
    crisp.raise_on_device_status(cfg, stream, "dense")

    # --- timed: end to end from page-locked host buffers through
    # crisp_prefill_host (copies of one KV group overlap the kernels of the
    # previous one); the device-resident copy of the layer is freed first
    del q, k, v, out, ix
    cfg.workspace = None
    torch.cuda.empty_cache()
    hcfg = crisp.Config(n=c.n, h_q=h_q, h_kv=h_kv, d=c.d, dtype=dtype, alpha=args.alpha, gamma=args.gamma)
    hcfg.allocate_workspace(dev, host=True)
    copy_stream = torch.cuda.Stream(device=dev)
    crisp.prefill_host(q_h, k_h, v_h, out_h, hcfg, stream, copy_stream)   # warm-up
    e2e_steps = max(1, min(args.steps, 3))
    barrier()
    torch.cuda.synchronize(dev)
    e2e_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(e2e_steps)]
    for a, b in e2e_evs:
        a.record(stream)
        crisp.prefill_host(q_h, k_h, v_h, out_h, hcfg, stream, copy_stream)
        b.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = [a.elapsed_time(b) for a, b in e2e_evs]
    crisp.raise_on_device_status(hcfg, stream, "e2e")
    clk = clocks.stop()

    # per-rank work of this rank's launches
    peaks, peak_src = load_peaks()
    tflops_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    hbm_peak = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    att_l, sel_l, route_l = statistics.mean(att_ms), statistics.mean(sel_ms), statistics.mean(route_ms)
    flops = 4.0 * c.d * 128 * 128 * tiles          # computed-tile work of one attention launch
    # algorithmic HBM bytes of the route pass: K read once, proxy rows of Q,
    # per-(row, tile) partials written and read back, chunk statistics
    nb = cfg.n_blocks
    rows = h_q * 64
    route_bytes = (h_kv * c.n * c.d * 2 + rows * c.d * 2 + 2 * rows * nb * 8
                   + rows * ((nb + 7) // 8) * 24)
    # selection (PE heads): their Q and their groups' K pooled once, the pooled
    # map written once and swept by the softmax (read+write), two histogram
    # passes and the mask pass (reads), plus the PE masks written
    n_pe = int((route == 1).sum())
    g_pe = len({h // c.group for h in range(h_q) if route[h] == 1})
    tri = nb * (nb + 1) // 2
    pe_bytes = (n_pe + g_pe) * c.n * c.d * 2 + n_pe * tri * 4 * 6 + n_pe * nb * cfg.words * 4
    pe_ms = max(sel_l - route_l, 1e-6)
    mufu = mufu_roofline(h_q * cfg.last_q * c.n, route_l, clk, sms)

    # across ranks: times are the maximum; rates the minimum (slowest rank);
    # with the layer split by KV group, tile and head counts add up
    vals = torch.tensor([statistics.mean(step_ms), att_l, sel_l, statistics.mean(dense_ms),
                         statistics.mean(e2e_ms), route_l], dtype=torch.float64, device=dev)
    rates = torch.tensor([flops / (att_l * 1e-3) / 1e12, route_bytes / (route_l * 1e-3) / 1e9,
                          pe_bytes / (pe_ms * 1e-3) / 1e9, (mufu or {}).get("frac", 0.0)],
                         dtype=torch.float64, device=dev)
    counts = torch.tensor([tiles, causal_tiles, int((route == 0).sum()), int((route == 1).sum())],
                          dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(vals, op=dist.ReduceOp.MAX)
        dist.all_reduce(rates, op=dist.ReduceOp.MIN)
        if heads_mode:
            dist.all_reduce(counts, op=dist.ReduceOp.SUM)
    step_m, att_m, sel_m, dense_m, e2e_m, route_m = vals.tolist()
    achieved, route_gbs, pe_gbs, mufu_frac = rates.tolist()
    tiles_all, causal_all, heads_vs, heads_pe = (int(x) for x in counts.tolist())
    if rank != 0:
        return None
    if mufu is not None:
        mufu["frac"] = round(mufu_frac, 4)
    dense_flops = 4.0 * c.d * 128 * 128 * causal_tiles
    h2d = int(q_h.numel() * q_h.element_size() + k_h.numel() * k_h.element_size() + v_h.numel() * v_h.element_size())
    d2h = int(out_h.numel() * out_h.element_size())
    src_hash = kernel_source_hash(["attn_tc.cu", "ptx.cuh"])
    traffic = (load_traffic("attn_tc_kernel", src_hash, args.config, args.alpha, args.gamma)
               if not heads_mode else None)
    # whole-job ms per layer: independent layers per GPU divide by the GPUs;
    # one layer split by KV group takes the slowest rank's time
    per_layer = 1 if heads_mode else world
    res = {
        "metric": METRIC,
        "value": round(step_m / per_layer, 4),
        "unit": "ms/layer",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_m, 4),
        "higher_is_better": False,
        "scaling": "strong" if heads_mode else "weak",
        "vs_baseline": None,
        "dtype": "bf16" if c.dtype == "bf16" else "f32",
        "data": ("synthetic (seeded Gaussian heads with planted sink/vertical/slash structure"
                 + (f", log-normal block background sigma {c.cliff_sigma:g}" if c.cliff_sigma > 0 else "")
                 + "; no datasets or weights)"),
        "config": {"workload": f"layer {args.config}: {c.desc}", "h_q": c.h_q, "h_kv": c.h_kv, "seq_len": c.n,
                   "alpha": args.alpha, "gamma": args.gamma,
                   "head_dim": c.d, "batch": 1,
                   "parallelism": (f"one layer split by KV group over {world} GPUs (no exchange)" if heads_mode
                                   else f"independent layer per GPU x{world}"),
                   "l2": "inputs (>= 6 GiB at 512K) far exceed the 126 MB L2; no flush between steps"},
        "speedup_vs_dense": round(dense_m / step_m, 4),
        "dense_ms_per_layer": round(dense_m, 4),
        "stages_ms": {"proxy_route_select": round(sel_m, 4), "sparse_attention": round(att_m, 4)},
        "density": {"computed_tiles": tiles_all, "causal_tiles": causal_all,
                    "fraction": round(tiles_all / causal_all, 4), "heads_vs": heads_vs, "heads_pe": heads_pe},
        "pages_speedup_context": f"{PAGES_SPEEDUP_512K}x at 512K tokens on one H100 (pages' figure, not comparable)",
        "roofline": {"kernel": "attn_tc_kernel (block-sparse attention)", "bound": "tensor",
                     "achieved": round(achieved, 2), "peak": tflops_peak, "unit": "TFLOP/s",
                     "frac": round(achieved / tflops_peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_src} bf16 dense, sustained (kernel runs inside a seconds-long step)",
                     "work": "4*d*128*128 flop per computed 128x128 tile x computed tiles per launch"},
        "dense_tflops": round(dense_flops / (dense_m * 1e-3) / 1e12, 2),
        "route_roofline": {"stage": "crisp_route (proxy_tc_kernel + finalize + VS masses)", "bound": "hbm",
                           "ms": round(route_m, 4), "algorithmic_bytes": route_bytes,
                           "achieved": round(route_gbs, 1), "peak": hbm_peak,
                           "unit": "GB/s", "frac": round(route_gbs / hbm_peak, 4),
                           # the proxy's exponentials (h_q x 64 x n) against MUFU at 16 per clock per SM
                           # and the median SM clock sampled under load
                           "mufu": mufu},
        "selection_roofline": {"stage": "PE pooling, pooled map, gamma cut, masks (select minus route)",
                               "bound": "hbm", "ms": round(max(sel_m - route_m, 1e-6), 4),
                               "algorithmic_bytes": pe_bytes,
                               "achieved": round(pe_gbs, 1),
                               "peak": hbm_peak, "unit": "GB/s",
                               "frac": round(pe_gbs / hbm_peak, 4)},
        "e2e": {"value": round(e2e_m / per_layer, 4), "unit": "ms/layer", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "api": "crisp_prefill_host: page-locked host buffers, copies overlapped with the kernels per KV group"},
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "clocks": clk,
    }
    return res


def run_stage(args):
    """Time one stage on a (possibly scaled) layer; used for ncu captures."""
    import torch
    import long_context_prefill_last_b200 as crisp
    c = S.CONFIGS[args.config]
    if args.n or args.h_q or args.h_kv:
        c = S.scaled(args.config, n=args.n, h_q=args.h_q, h_kv=args.h_kv)
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
    print(json.dumps({"stage": args.only, "layer": c.name, "ms": round(ms, 4)}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--dense-steps", type=int, default=3)
    ap.add_argument("--config", default="E", choices=sorted(S.CONFIGS))
    ap.add_argument("--impl", default="crisp", choices=["crisp", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--alpha", type=float, default=1.0, help="Eq. (4) noise-floor multiplier")
    ap.add_argument("--gamma", type=float, default=0.95, help="PE cumulative coverage")
    ap.add_argument("--shard", choices=["layers", "heads"], default="layers",
                    help="with N > 1 GPUs: an independent layer per GPU (weak scaling, default) or one layer "
                         "split by KV group (strong scaling)")
    ap.add_argument("--only", choices=["select", "attend", "dense", "prefill", "route"],
                    help="profiling mode: time one stage alone (no contract line)")
    ap.add_argument("--n", type=int, help="profiling mode: scaled sequence length")
    ap.add_argument("--h-q", type=int, help="profiling mode: scaled query heads")
    ap.add_argument("--h-kv", type=int, help="profiling mode: scaled KV heads")
    args = ap.parse_args()
    if args.only:
        run_stage(args)
        return

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        ms, sample, spent = oracle_ms_per_layer(args.config, budget_s=max(8.0, 40.0 / max(1, args.steps)))
        cores = cpu_cores()
        res = {"metric": METRIC, "value": round(ms, 1), "unit": "ms/layer", "n_gpus": args.gpus,
               "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": False,
               "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
               "impl": "reference",
               "config": {"workload": f"layer {args.config}: {S.CONFIGS[args.config].desc}"},
               "cpu_baseline": {"value": round(ms, 1), "unit": "ms/layer", "cores": cores, "kind": "oracle",
                                "sample": sample},
               "e2e": {"value": round(ms, 1), "unit": "ms/layer", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(res))
        return

    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    res = run_crisp(args, rank, world, local_rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            ms, sample, _ = oracle_ms_per_layer(args.config, budget_s=20.0)
            res["cpu_baseline"] = {"value": round(ms, 1), "unit": "ms/layer", "cores": cpu_cores(), "kind": "oracle",
                                   "sample": sample}
        print(json.dumps(res))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
