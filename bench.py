#!/usr/bin/env python
"""Benchmark of the Fourier-approximated KV cache hot path on B200.

One step = one pass of the whole path over one batch of the workload: build the basis
table, fa_compress (sink/recent copy, retained-dim packing and the tcgen05 projection of
K and V) and one fa_decode step (prologue, split-L main kernel, combine). Default
workload: LLaMA-2-7B attention shape, batch 8, 32 MHA heads, L = 32768, S = 32, R = 64,
k = 255, 96 of 128 dims compressed per head (seeded random masks), synthetic caches.

Prints ONE JSON line (rank 0). ``value`` is microseconds per step (lower is better),
timed with CUDA events on the launching stream over exactly --steps steps after
--warmup steps, max over ranks. With --gpus N each rank runs its own batch (weak
scaling, no collective in the data path).

--impl reference times the fp64 CPU oracle on the host cores on a bounded sample of the
same workload (whole (batch, KV head) pairs, scaled to the full step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fa_decode μs/step & HBM GB/s; fa_compress TFLOP/s; % of B200 roofline"
L2_BYTES = 126 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama2_7b_mha_b8_L32768_k255")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload measurements added to the default line")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch")
    ap.add_argument("--no-clock-probe", action="store_true",
                    help="skip the extra clock-sampling loop after a short timed region")
    ap.add_argument("--fft-probe", action="store_true",
                    help="time the cuFFT building blocks of an O(M log M) decode beside fa_decode "
                         "(k = 511 and k = 1023 workloads); a measurement, not a product path")
    ap.add_argument("--sweep", action="store_true",
                    help="time every single-layer workload and the 32-layer LLaMA-3-8B decode "
                         "sweep (one JSON line each) instead of the default bench line")
    ap.add_argument("--sweep-points", default="",
                    help="comma list of BxL points for the 32-layer sweep (default: all 12)")
    return ap.parse_args()


def workload_by_name(name):
    """One of the named single-layer workloads, or one layer of the 32-layer LLaMA-3-8B
    cache as llama3_8b_layer<layer>_b<B>_L<L>[_k<k>] (k is always L / 128 - 1)."""
    import re
    import workloads as wl
    for w in wl.CONFIGS:
        if w.name == name:
            return w
    m = re.fullmatch(r"llama3_8b_layer(\d+)_b(\d+)_L(\d+)(_k\d+)?", name)
    if m:
        return wl.llama3_8b_layer(int(m.group(2)), int(m.group(3)), int(m.group(1)))
    raise SystemExit(f"unknown workload {name}; known: {[w.name for w in wl.CONFIGS]} or "
                     "llama3_8b_layer<layer>_b<B>_L<L>")


# ----------------------------------------------------------------------------- algorithmic work

def work_model(w, plan):
    """Algorithmic bytes / flops per step, from the plan's per-head dim split.

    Two byte counts per half of the path:
    * ``*_bytes``: what this implementation moves by design: C stored in fp32, and
      fa_compress also copies the sink / recent rows into F;
    * ``*_bytes_alg``: the method's minimum (bf16 C; compress reads the middle rows once
      and writes C and E, decode reads F, E and C of K and V plus q and writes out).
    Rooflines are reported against ``*_bytes_alg`` (the smaller, so the harder, figure)."""
    B, Hkv, G, D = w.B, w.Hkv, w.G, 128
    S, R, M, k = plan.S, plan.R, plan.M, w.k
    dcs = [plan.dc[g] for g in range(Hkv)]
    des = [plan.de[g] for g in range(Hkv)]
    kk = k if M > 0 else 0
    # compress: read the middle rows once, write C (fp32) and E, copy the sink/recent rows
    # (K and V)
    c_bytes = 2 * B * sum(2 * M * D + 4 * kk * dc + 2 * M * de + 2 * 2 * (S + R) * D
                          for dc, de in zip(dcs, des))
    c_bytes_alg = 2 * B * sum(2 * M * D + 2 * kk * dc + 2 * M * de for dc, de in zip(dcs, des))
    c_flops = 2 * 2 * B * sum(kk * M * dc for dc in dcs)
    # decode: read F, E (bf16) and C of K and V, the queries, write the outputs
    qo = 2 * 2 * B * w.Hq * D
    d_bytes = 2 * B * sum(2 * (S + R) * D + 2 * M * de + 4 * kk * dc for dc, de in zip(dcs, des)) + qo
    d_bytes_alg = 2 * B * sum(2 * (S + R) * D + 2 * M * de + 2 * kk * dc
                              for dc, de in zip(dcs, des)) + qo
    d_flops = B * G * sum(4 * D * (S + R) + 4 * de * M + 4 * kk * dc + 4 * M * kk
                          for dc, de in zip(dcs, des))
    return dict(compress_bytes=c_bytes, compress_bytes_alg=c_bytes_alg, compress_flops=c_flops,
                decode_bytes=d_bytes, decode_bytes_alg=d_bytes_alg, decode_flops=d_flops)


def decode_path(w, plan):
    """Which split kernel fa_decode runs for this plan (the library's own answer)."""
    import fourier_basis_attention_b200 as fa
    info = fa.fa_decode_describe(plan, 1)
    name = fa.SPLIT_KERNELS[info.split_kernel]
    return name + (f", clusters of {info.cluster}" if info.cluster > 1 else "")


def config_dict(w, world=1):
    """The ``config`` object of the JSON line; both arms print exactly this."""
    import workloads as wl
    mask = wl.dim_mask(w)
    dcs = sorted({int(x) for x in mask.sum(axis=1)})
    return {"workload": w.name, "global_batch": w.B * world, "seq_len": w.L, "Hq": w.Hq,
            "Hkv": w.Hkv, "k": w.k, "S": w.S, "R": w.R,
            "dims_compressed_per_head": dcs[0] if len(dcs) == 1 else dcs,
            "parallelism": f"replica x{world}",
            "l2": ("inputs larger than L2 (K+V %.2f GB per replica)" if 2 * K_bytes(w) > L2_BYTES
                   else "inputs fit in L2 (K+V %.4f GB per replica)") % (2 * K_bytes(w) / 1e9)}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            pk = json.load(fh)
        return pk, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def compress_traffic():
    """Measured DRAM traffic of the compress kernel (profiles/), if taken on this source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rec = json.load(fh)
    src = os.path.join(ROOT, "fourier_basis_attention_b200", "csrc", rec.get("source", ""))
    if not os.path.exists(src):
        return None
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return rec if digest == rec.get("source_sha256_16") else None


def decode_traffic():
    """Measured DRAM traffic of one fa_decode on the bench workload (profiles/), if it was
    taken on the current decode sources."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rec = json.load(fh)
    h = hashlib.sha256()
    for name in rec.get("sources", []):
        src = os.path.join(ROOT, "fourier_basis_attention_b200", "csrc", name)
        if not os.path.exists(src):
            return None
        h.update(open(src, "rb").read())
    return rec.get("bytes_per_step") if h.hexdigest()[:16] == rec.get("sources_sha256_16") else None


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu_index = gpu_index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.out = open("/tmp/fa_clocks_%d.csv" % os.getpid(), "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_index, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return []
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.out.name) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), sm_max=float(parts[2]),
                                     power=float(parts[3]) if parts[3] not in ("[N/A]", "") else 0.0,
                                     hw=parts[5], hw_thermal=parts[6], sw_thermal=parts[7],
                                     sw_power=parts[8]))
                except ValueError:
                    continue
        os.unlink(self.out.name)
        return rows


def summarize_clocks(rows):
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    loaded = [r for r in rows if r["power"] > 200.0] or rows
    reasons = set()
    for r in loaded:
        for key, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                          ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
            if r[key].lower().startswith("active"):
                reasons.add(name)
    return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
            "sm_max_mhz": max(r["sm_max"] for r in rows), "reasons": sorted(reasons),
            "samples": len(loaded)}


# ----------------------------------------------------------------------------- oracle timing

ORACLE_PAIRS = 4  # (batch, KV head) pairs the oracle runs per sampled step


def oracle_step_seconds(w, pairs):
    """One sampled oracle step, scaled to the whole workload, in seconds.

    The same policy serves the GPU arm's ``cpu_baseline`` and ``--impl reference``: the
    oracle's basis cache is cleared, the basis is built once (timed: the GPU step rebuilds
    its table every step too), then len(pairs) whole (batch, KV head) pairs run fp64
    compress of K and V and the decode step; the pair time is scaled to all B * Hkv pairs."""
    from oracle import fourier_oracle as fo
    fo._basis_full.cache_clear()
    S_, R_, M = fo.partition(w.L, w.S, w.R)
    t0 = time.perf_counter()
    if M > 0:
        fo._basis_full(M, w.k, M)
    t_basis = time.perf_counter() - t0
    t0 = time.perf_counter()
    for (Kh, Vh, qh, m) in pairs:
        hk = fo.compress(Kh, m, w.S, w.R, w.k)
        hv = fo.compress(Vh, m, w.S, w.R, w.k)
        fo.decode(qh, hk, hv)
    t_pairs = time.perf_counter() - t0
    return t_basis + t_pairs / len(pairs) * (w.B * w.Hkv)


def oracle_sample_note(w, n_pairs):
    n_units = w.B * w.Hkv
    return (f"{n_pairs} of {n_units} (batch, KV head) pairs per step (fp64 compress of K and V + "
            f"decode), scaled x{n_units / n_pairs:g}, plus one basis build per step (the oracle's "
            f"basis cache cleared before every step)")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((d.get("num_threads", 1) for d in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def host_pairs(w, n_pairs, seed_shift=0):
    """A few (batch, KV head) pairs of the workload drawn on the host (fp64 arrays)."""
    import workloads as wl
    ws = wl.shrink(w, B=1, seed=w.seed + seed_shift)
    K = wl.kv_cache(ws, "K")[0]
    V = wl.kv_cache(ws, "V")[0]
    q = wl.queries(ws)[0]
    mask = wl.dim_mask(w)
    out = []
    for g in range(min(n_pairs, w.Hkv)):
        out.append((K[g].double().numpy(), V[g].double().numpy(),
                    q[g * w.G:(g + 1) * w.G].double().numpy(), mask[g]))
    return out


# ----------------------------------------------------------------------------- ranks

def rank_workload(base, rank):
    """Rank r's replica of the workload: the same shapes with its own seed (weak scaling: each
    rank compresses and decodes its own batch; no data crosses ranks)."""
    import workloads as wl
    return wl.shrink(base, seed=base.seed + 1000 * rank) if rank else base


def max_over_ranks(values, device=None):
    """Element-wise max over all ranks of a list of floats (the slowest rank sets every
    reported time). Every rank must call it, in the same order; one rank: returned as is."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def prints_line(rank):
    """Only rank 0 prints the JSON line."""
    return rank == 0


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if not prints_line(rank):
        return  # the reference arm runs on rank 0 alone
    w = workload_by_name(args.workload)
    if args.batch > 0:
        import workloads as wl
        w = wl.shrink(w, B=args.batch)
    pairs = host_pairs(w, ORACLE_PAIRS)
    for _ in range(args.warmup):
        oracle_step_seconds(w, pairs)
    times = [oracle_step_seconds(w, pairs) for _ in range(args.steps)]
    us = statistics.mean(times) * 1e6
    cores = blas_threads()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    line = {
        "impl": "reference", "metric": METRIC, "value": us, "unit": "us/step",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_dict(w, world),
        "cpu_baseline": {"value": us, "unit": "us/step", "cores": cores, "kind": "oracle",
                         "sample": oracle_sample_note(w, len(pairs))},
        "e2e": {"value": us, "unit": "us/step", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm

def roofline_entry(kind, bytes_, flops, ms, peaks, peak_src, kernel, traffic=None):
    """A roofline object: HBM-bound unless the path's arithmetic intensity is above the
    ridge of the bf16 tensor peak over the HBM peak (compress at large k)."""
    hbm = peaks["hbm_gbs"]
    tc = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    ridge = tc * 1e12 / (hbm * 1e9)
    gbs = bytes_ / (ms * 1e-3) / 1e9
    tfl = flops / (ms * 1e-3) / 1e12
    if kind == "compress" and flops / bytes_ >= ridge:
        roof = {"bound": "tensor", "achieved": tfl, "peak": tc, "unit": "TFLOP/s", "frac": tfl / tc}
    else:
        roof = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm}
    roof.update({"kernel": kernel, "traffic": traffic,
                 "algorithmic_bytes": bytes_,
                 "peak_source": ("measured (MEASURED_PEAKS.json hbm_gbs / bf16_tflops)"
                                 if peak_src == "measured" else
                                 "fallback (6.65 TB/s, 1.59 PFLOP/s: no MEASURED_PEAKS.json)")})
    return roof


def timed_loop(fn, stream, min_s=0.6, max_iter=4000):
    """Average device time (ms) of fn() over a loop of back-to-back calls lasting about
    min_s seconds (long enough for the clock sampler), CUDA events on ``stream``."""
    import torch
    t_one = _time(fn, 3, stream)
    n = int(min(max_iter, max(10, min_s * 1e3 / max(t_one, 1e-3))))
    return _time(fn, n, stream), n


def measure_workload(w, dev, stream, peaks, peak_src, gpu_index):
    """Per-workload figures for the bench line: compress and decode timed in loops of
    about 0.6 s each (decode also as CUDA-graph replays), with the SM clocks sampled during
    each loop."""
    import torch

    import fourier_basis_attention_b200 as fa
    import workloads as wl
    mask = wl.dim_mask(w)
    K = wl.kv_cache(w, "K", device=dev)
    V = wl.kv_cache(w, "V", device=dev)
    q = wl.queries(w, device=dev)
    plan = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
    cache = fa.Cache(plan, device=dev)
    phiT = torch.empty(w.k, plan.phi_ld, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(fa.fa_decode_workspace_size(plan), dtype=torch.uint8, device=dev)
    out = torch.empty(w.B, w.Hq, 128, dtype=torch.bfloat16, device=dev)
    fa.fa_build_basis(plan.P, w.k, phiT, plan.phi_ld, False, stream)
    comp = lambda: fa.fa_compress(plan, K, V, phiT, cache, stream)
    dec = lambda: fa.fa_decode(plan, q, cache, out, ws, 0, stream)
    for f in (comp, dec):
        f(); f(); f()
    sampler = ClockSampler(gpu_index)
    sampler.start()
    time.sleep(0.25)
    t_c, n_c = timed_loop(comp, stream)
    t_d, n_d = timed_loop(dec, stream)
    rows = sampler.stop()
    t_dg = _time_graph(lambda s: fa.fa_decode(plan, q, cache, out, ws, 0, s), max(10, n_d // 4))
    fa.fa_device_status(stream)
    wm = work_model(w, plan)
    rc = roofline_entry("compress", wm["compress_bytes_alg"], wm["compress_flops"], t_c, peaks,
                        peak_src, "fa_compress")
    rd = roofline_entry("decode", wm["decode_bytes_alg"], wm["decode_flops"], t_d, peaks,
                        peak_src, "fa_decode")
    rdg = roofline_entry("decode", wm["decode_bytes_alg"], wm["decode_flops"], t_dg, peaks,
                         peak_src, "fa_decode")
    hbm = peaks["hbm_gbs"]
    tcp = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    res = {
        "shape": {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "S": w.S, "R": w.R, "k": w.k},
        "fa_compress": {"us": t_c * 1e3, "iterations": n_c,
                        "tflops": wm["compress_flops"] / t_c / 1e9,
                        "frac_tensor": wm["compress_flops"] / t_c / 1e9 / tcp,
                        "hbm_gbs": wm["compress_bytes_alg"] / t_c / 1e6,
                        "frac_hbm": wm["compress_bytes_alg"] / t_c / 1e6 / hbm,
                        "bound": rc["bound"], "frac_of_bound": rc["frac"]},
        "fa_decode": {"us": t_d * 1e3, "iterations": n_d, "us_graph_replay": t_dg * 1e3,
                      "path": decode_path(w, plan),
                      "hbm_gbs": wm["decode_bytes_alg"] / t_d / 1e6, "frac_hbm": rd["frac"],
                      "frac_hbm_graph_replay": rdg["frac"],
                      "algorithmic_bytes": wm["decode_bytes_alg"]},
        "clocks": summarize_clocks(rows),
    }
    del K, V, q, cache, phiT, ws, out
    torch.cuda.empty_cache()
    return res


def measure_layers(B, L, dev, stream, peaks, gpu_index, layers=32):
    """One point of the 32-layer LLaMA-3-8B cache: fa_compress of every layer (distinct
    seeded masks) and one decode step over all layers (32 fa_decode calls), each timed in
    loops of about 0.6 s, clocks sampled."""
    import torch

    import fourier_basis_attention_b200 as fa
    import workloads as wl
    w0 = wl.llama3_8b_layer(B, L, 0)
    K = wl.kv_cache(w0, "K", device=dev)
    V = wl.kv_cache(w0, "V", device=dev)
    q = wl.queries(w0, device=dev)
    plans, caches, wms = [], [], []
    phiT = None
    for layer in range(layers):
        wlay = wl.llama3_8b_layer(B, L, layer)
        plan = fa.fa_plan_init(B, 32, 8, L, wlay.S, wlay.R, wlay.k, wl.dim_mask(wlay))
        plans.append(plan)
        caches.append(fa.Cache(plan, device=dev))
        wms.append(work_model(wlay, plan))
        if phiT is None:
            phiT = torch.empty(wlay.k, plan.phi_ld, dtype=torch.bfloat16, device=dev)
            fa.fa_build_basis(plan.P, wlay.k, phiT, plan.phi_ld, False, stream)

    def comp():  # the K / V of every layer are one synthetic draw; the masks differ
        for p, c in zip(plans, caches):
            fa.fa_compress(p, K, V, phiT, c, stream)
    ws = torch.empty(max(fa.fa_decode_workspace_size(p) for p in plans), dtype=torch.uint8,
                     device=dev)
    out = torch.empty(B, 32, 128, dtype=torch.bfloat16, device=dev)

    def dec(s=stream):
        for p, c in zip(plans, caches):
            fa.fa_decode(p, q, c, out, ws, 0, s)
    comp(); dec()
    sampler = ClockSampler(gpu_index)
    sampler.start()
    time.sleep(0.25)
    t_c, n_c = timed_loop(comp, stream)
    t_d, n_d = timed_loop(dec, stream)
    rows = sampler.stop()
    t_dg = _time_graph(dec, max(5, n_d // 4))
    fa.fa_device_status(stream)
    hbm = peaks["hbm_gbs"]
    tcp = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    cfl = sum(m["compress_flops"] for m in wms)
    cby = sum(m["compress_bytes_alg"] for m in wms)
    dby = sum(m["decode_bytes_alg"] for m in wms)
    res = {
        "shape": {"layers": layers, "B": B, "Hq": 32, "Hkv": 8, "L": L, "S": w0.S, "R": w0.R,
                  "k": w0.k},
        "fa_compress": {"us": t_c * 1e3, "iterations": n_c, "tflops": cfl / t_c / 1e9,
                        "frac_tensor": cfl / t_c / 1e9 / tcp, "hbm_gbs": cby / t_c / 1e6,
                        "frac_hbm": cby / t_c / 1e6 / hbm},
        "fa_decode": {"us": t_d * 1e3, "iterations": n_d, "us_graph_replay": t_dg * 1e3,
                      "path": decode_path(w0, plans[0]), "hbm_gbs": dby / t_d / 1e6,
                      "frac_hbm": dby / t_d / 1e6 / hbm,
                      "frac_hbm_graph_replay": dby / t_dg / 1e6 / hbm, "algorithmic_bytes": dby},
        "clocks": summarize_clocks(rows),
    }
    del K, V, q, caches, plans, ws, out, phiT
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    import torch.distributed as dist

    import fourier_basis_attention_b200 as fa
    import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    base = workload_by_name(args.workload)
    if args.batch > 0:
        base = wl.shrink(base, B=args.batch)
    w = rank_workload(base, rank)
    mask = wl.dim_mask(base)
    dev = torch.device("cuda", local)
    K = wl.kv_cache(w, "K", device=dev)
    V = wl.kv_cache(w, "V", device=dev)
    q = wl.queries(w, device=dev)
    plan = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
    cache = fa.Cache(plan, device=dev)
    phiT = torch.empty(w.k, plan.phi_ld, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(fa.fa_decode_workspace_size(plan), dtype=torch.uint8, device=dev)
    out = torch.empty(w.B, w.Hq, 128, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.fa_build_basis(plan.P, w.k, phiT, plan.phi_ld, False, stream)
        fa.fa_compress(plan, K, V, phiT, cache, stream)
        fa.fa_decode(plan, q, cache, out, ws, 0, stream)

    for _ in range(max(args.warmup, 3)):
        step()
    fa.fa_device_status(stream)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize(dev)

    gpu_index = os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local if world > 1 else 0]
    sampler = ClockSampler(gpu_index)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    sampler.start()
    time.sleep(0.3)
    barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        e = ev[i]
        e[0].record(stream)
        fa.fa_build_basis(plan.P, w.k, phiT, plan.phi_ld, False, stream)
        e[1].record(stream)
        fa.fa_compress(plan, K, V, phiT, cache, stream)
        e[2].record(stream)
        fa.fa_decode(plan, q, cache, out, ws, 0, stream)
        e[3].record(stream)
    t_end.record(stream)
    barrier()
    total_ms = t_start.elapsed_time(t_end)
    rows = sampler.stop()
    clock_note = "sampled during the timed region"
    if len([r for r in rows if r["power"] > 200.0]) < 3 and not args.no_clock_probe:
        # timed region too short for the 100 ms sampler: sample the same step for ~1 s more
        sampler2 = ClockSampler(gpu_index)
        sampler2.start()
        time.sleep(0.3)
        t_end_probe = time.time() + 1.2
        while time.time() < t_end_probe:
            for _ in range(20):
                step()
            torch.cuda.synchronize(dev)
        rows = rows + sampler2.stop()
        clock_note = "timed region plus ~1.2 s more of the same step (region shorter than the sampler period)"
    fa.fa_device_status(stream)
    t_basis = [e[0].elapsed_time(e[1]) for e in ev]
    t_comp = [e[1].elapsed_time(e[2]) for e in ev]
    t_dec = [e[2].elapsed_time(e[3]) for e in ev]
    ms_step = total_ms / args.steps
    comp_ms = statistics.mean(t_comp)
    dec_ms = statistics.mean(t_dec)
    basis_ms = statistics.mean(t_basis)
    ms_step, comp_ms, dec_ms, basis_ms = max_over_ranks([ms_step, comp_ms, dec_ms, basis_ms], dev)

    # ---------------------------------------------------------------- end to end (host buffers)
    e2e_us = None
    h2d = d2h = 0
    if args.e2e_steps > 0:
        Kh = torch.empty(K.shape, dtype=K.dtype, pin_memory=True)
        Vh = torch.empty(V.shape, dtype=V.dtype, pin_memory=True)
        qh = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
        oh = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        Kh.copy_(K)
        Vh.copy_(V)
        qh.copy_(q)
        Kd, Vd, qd = torch.empty_like(K), torch.empty_like(V), torch.empty_like(q)
        del K, V
        torch.cuda.synchronize(dev)
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            Kd.copy_(Kh, non_blocking=True)
            Vd.copy_(Vh, non_blocking=True)
            qd.copy_(qh, non_blocking=True)
            fa.fa_build_basis(plan.P, w.k, phiT, plan.phi_ld, False, stream)
            fa.fa_compress(plan, Kd, Vd, phiT, cache, stream)
            fa.fa_decode(plan, qd, cache, out, ws, 0, stream)
            oh.copy_(out, non_blocking=True)
        b.record(stream)
        barrier()
        e2e_ms = a.elapsed_time(b) / args.e2e_steps
        e2e_ms = max_over_ranks([e2e_ms], dev)[0]
        e2e_us = e2e_ms * 1e3
        h2d = Kh.numel() * 2 + Vh.numel() * 2 + qh.numel() * 2
        d2h = oh.numel() * 2
        del Kh, Vh, Kd, Vd
    else:
        del K, V
    del cache, ws
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- roofline
    wm = work_model(w, plan)
    peaks, peak_src = load_peaks()
    hbm = peaks["hbm_gbs"]
    tc = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    traffic = compress_traffic()
    roof = roofline_entry("compress", wm["compress_bytes_alg"], wm["compress_flops"], comp_ms,
                          peaks, peak_src, "fa_compress (compress_kernel + copy_sink_recent_kernel)",
                          traffic["bytes_per_launch_scaled"] if traffic else None)
    roof_dec = roofline_entry("decode", wm["decode_bytes_alg"], wm["decode_flops"], dec_ms, peaks,
                              peak_src, "fa_decode (prologue + %s + combine)" % decode_path(w, plan),
                              decode_traffic())
    c_gbs = wm["compress_bytes_alg"] / (comp_ms * 1e-3) / 1e9
    c_tflops = wm["compress_flops"] / (comp_ms * 1e-3) / 1e12
    d_gbs = wm["decode_bytes_alg"] / (dec_ms * 1e-3) / 1e9

    line = {
        "metric": METRIC, "value": ms_step * 1e3, "unit": "us/step", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_step,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": config_dict(base, world),
        "components": {
            "fa_build_basis": {"us": basis_ms * 1e3},
            "fa_compress": {"us": comp_ms * 1e3, "tflops": c_tflops, "hbm_gbs": c_gbs,
                            "algorithmic_bytes": wm["compress_bytes_alg"],
                            "bytes_moved_fp32_C_and_F_copy": wm["compress_bytes"],
                            "algorithmic_flops": wm["compress_flops"],
                            "frac_hbm": c_gbs / hbm, "frac_tensor": c_tflops / tc},
            "fa_decode": {"us": dec_ms * 1e3, "hbm_gbs": d_gbs, "frac_hbm": d_gbs / hbm,
                          "path": decode_path(w, plan),
                          "algorithmic_bytes": wm["decode_bytes_alg"],
                          "bytes_moved_fp32_C": wm["decode_bytes"],
                          "algorithmic_flops": wm["decode_flops"]},
        },
        "roofline": roof,
        "roofline_fa_decode": roof_dec,
        "clocks": {**summarize_clocks(rows), "note": clock_note},
        "gpu_launches": launches_per_step(w, plan) * args.steps,
        "e2e": {"value": e2e_us, "unit": "us/step", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
    }
    if world == 1 and not args.no_configs:
        # every single-layer workload and one point of the 32-layer cache, measured apart
        # from the timed step above (not part of ``value``)
        per = {}
        for cw in wl.CONFIGS:
            per[cw.name] = measure_workload(cw, dev, stream, peaks, peak_src, gpu_index)
        per["llama3_8b_32_layers_b8_L32768_k255"] = measure_layers(8, 32768, dev, stream, peaks,
                                                                  gpu_index)
        line["per_workload"] = per
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        pairs = host_pairs(base, ORACLE_PAIRS)
        est = [oracle_step_seconds(base, pairs) for _ in range(3)]
        line["cpu_baseline"] = {
            "value": statistics.mean(est) * 1e6, "unit": "us/step", "cores": blas_threads(),
            "kind": "oracle",
            "sample": oracle_sample_note(base, len(pairs)) + "; mean of 3 sampled steps"}
    if prints_line(rank):
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()


def launches_per_step(w, plan):
    """Kernels one step launches: build_basis_kernel; copy_sink_recent_kernel (when there
    are sink / recent rows) and compress_kernel (when there is a middle span); then what
    fa_decode launches (the library's count: prologue, split kernel, combine)."""
    import fourier_basis_attention_b200 as fa
    n = 1 + (1 if plan.S + plan.R > 0 else 0) + (1 if plan.M > 0 else 0)
    return n + fa.fa_decode_describe(plan, 1).launches


def K_bytes(w):
    return w.B * w.Hkv * w.L * 128 * 2


def _time(fn, n, stream):
    import torch
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / n


def _time_graph(fn, n):
    """Per-replay device time of fn(stream) captured once in a CUDA graph (the way a serving
    loop runs a launch-bound step); CUDA events on the replaying stream."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn(side)
        fn(side)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn(torch.cuda.current_stream())
    g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        g.replay()
    b.record(stream)
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / n


APPEND_STEPS = 50


def append_bytes(plan):
    """Algorithmic bytes of one fa_append: per (batch, KV head) and K / V, the k x dc_ld
    coefficient block read and written, one E row written, the leaving ring row read, the
    new token read and written to the ring."""
    s = plan.shape
    per = sum(2 * plan.kk * plan.dc_ld[g] * 4 + plan.de_ld[g] * 2 + 3 * 128 * 2
              for g in range(s.Hkv))
    return 2 * s.B * per


def time_append(w, plan, K, V, stream):
    """Device time of one fa_append (one new token per sequence) on a copy of ``plan`` with
    room reserved for the warm-up and timed appends; returns (ms, bytes per launch)."""
    import torch

    import fourier_basis_attention_b200 as fa
    pa = fa.fa_plan.from_buffer_copy(plan)
    fa.fa_plan_reserve(pa, w.L + APPEND_STEPS + 3)
    cache = fa.Cache(pa, device=K.device)
    phiT = fa.basis_table(pa, device=K.device, stream=stream)
    fa.fa_compress(pa, K, V, phiT, cache, stream)
    kn = K[:, :, -1].contiguous()
    vn = V[:, :, -1].contiguous()
    app = lambda: fa.fa_append(pa, kn, vn, cache, stream)
    for _ in range(3):
        app()
    nbytes = append_bytes(pa)
    # each append timed alone after a 256 MB read that evicts the 126 MB L2 with clean lines,
    # as in a decode loop where the attention step streams the cache between two appends
    flush = torch.ones(64 << 20, dtype=torch.float32, device=K.device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(APPEND_STEPS)]
    for a, b in evs:
        flush.sum()
        a.record(stream)
        app()
        b.record(stream)
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in evs) / APPEND_STEPS
    fa.fa_device_status(stream)
    del cache, phiT, flush
    torch.cuda.empty_cache()
    return ms, nbytes


def time_sensitivity(w, K, q, stream):
    """Device time of one fa_dim_sensitivity over the workload's keys and a seeded noise
    tensor of the same shape; returns (ms, algorithmic bytes: K and noise read once)."""
    import torch

    import fourier_basis_attention_b200 as fa
    import workloads as wl
    noise = wl.value_noise(w, device=K.device)
    ws = torch.empty(fa.fa_dim_sensitivity_workspace_size(w.B, w.Hq, w.Hkv, w.L),
                     dtype=torch.uint8, device=K.device)
    scores = torch.empty(w.Hkv, 128, dtype=torch.float32, device=K.device)
    run = lambda: fa.fa_dim_sensitivity(q, K, noise, scores, ws, stream)
    for _ in range(2):
        run()
    ms = _time(run, 5, stream)
    fa.fa_device_status(stream)
    del noise, ws, scores
    torch.cuda.empty_cache()
    return ms, 2 * K_bytes(w)


def run_sweep(args):
    """Per-workload timings (1 GPU): the four single-layer workloads, then the 32-layer
    LLaMA-3-8B-shaped cache: compress every layer (distinct seeded masks), and time one
    decode step over all 32 layers for each batch x context point."""
    import torch

    import fourier_basis_attention_b200 as fa
    import workloads as wl

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks, _ = load_peaks()
    hbm = peaks["hbm_gbs"]
    tc = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    for w in wl.CONFIGS:
        mask = wl.dim_mask(w)
        K = wl.kv_cache(w, "K", device=dev)
        V = wl.kv_cache(w, "V", device=dev)
        q = wl.queries(w, device=dev)
        plan = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
        cache = fa.Cache(plan, device=dev)
        phiT = torch.empty(w.k, plan.phi_ld, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(fa.fa_decode_workspace_size(plan), dtype=torch.uint8, device=dev)
        out = torch.empty(w.B, w.Hq, 128, dtype=torch.bfloat16, device=dev)
        basis = lambda: fa.fa_build_basis(plan.P, w.k, phiT, plan.phi_ld, False, stream)
        comp = lambda: fa.fa_compress(plan, K, V, phiT, cache, stream)
        dec = lambda: fa.fa_decode(plan, q, cache, out, ws, 0, stream)
        for f in (basis, comp, dec):
            f(); f(); f()
        tb = _time(basis, 10, stream)
        tcmp = _time(comp, 10, stream)
        td_eager = _time(dec, 20, stream)
        td = _time_graph(lambda s: fa.fa_decode(plan, q, cache, out, ws, 0, s), 20)
        fa.fa_device_status(stream)
        del cache, ws
        ta, a_bytes = time_append(w, plan, K, V, stream)
        tsens, s_bytes = time_sensitivity(w, K, q, stream)
        wm = work_model(w, plan)
        print(json.dumps({"sweep": "single_layer", "workload": w.name, "basis_us": tb * 1e3,
                          "compress_us": tcmp * 1e3,
                          "compress_tflops": wm["compress_flops"] / tcmp / 1e9,
                          "compress_hbm_gbs": wm["compress_bytes"] / tcmp / 1e6,
                          "compress_frac_tensor": wm["compress_flops"] / tcmp / 1e9 / tc,
                          "compress_frac_hbm": wm["compress_bytes"] / tcmp / 1e6 / hbm,
                          "decode_us": td * 1e3, "decode_us_eager": td_eager * 1e3,
                          "decode_timing": "CUDA graph replay (eager launches in decode_us_eager)",
                          "decode_hbm_gbs": wm["decode_bytes"] / td / 1e6,
                          "decode_frac_hbm": wm["decode_bytes"] / td / 1e6 / hbm,
                          "decode_fp32_tflops": wm["decode_flops"] / td / 1e9,
                          "append_us": ta * 1e3, "append_hbm_gbs": a_bytes / ta / 1e6,
                          "append_frac_hbm": a_bytes / ta / 1e6 / hbm,
                          "sensitivity_us": tsens * 1e3, "sensitivity_hbm_gbs": s_bytes / tsens / 1e6,
                          "sensitivity_frac_hbm": s_bytes / tsens / 1e6 / hbm}), flush=True)
        del K, V, out, phiT
        torch.cuda.empty_cache()

    points = [(B, L) for L in wl.SWEEP_L for B in wl.SWEEP_BATCH]
    if args.sweep_points:
        points = [tuple(int(x) for x in p.split("x")) for p in args.sweep_points.split(",")]
    for B, L in points:
        w0 = wl.llama3_8b_layer(B, L, 0)
        K = wl.kv_cache(w0, "K", device=dev)
        V = wl.kv_cache(w0, "V", device=dev)
        q = wl.queries(w0, device=dev)
        plans, caches, t_comp = [], [], []
        free, _ = torch.cuda.mem_get_info(dev)
        phiT = None
        resident = 0
        for layer in range(32):
            wlay = wl.llama3_8b_layer(B, L, layer)
            plan = fa.fa_plan_init(B, 32, 8, L, wlay.S, wlay.R, wlay.k, wl.dim_mask(wlay))
            need = 2 * (plan.f_elems * 2 + plan.e_elems * 2 + plan.c_elems * 4)
            free, _ = torch.cuda.mem_get_info(dev)
            if need > free - (4 << 30) and resident > 0:
                plans.append(plan)  # cycled: reuses an earlier layer's buffers
                caches.append(caches[layer % resident])
            else:
                cache = fa.Cache(plan, device=dev)
                plans.append(plan)
                caches.append(cache)
                resident += 1
            if phiT is None:
                phiT = torch.empty(wlay.k, plan.phi_ld, dtype=torch.bfloat16, device=dev)
                fa.fa_build_basis(plan.P, wlay.k, phiT, plan.phi_ld, False, stream)
            # the K / V of every layer are the same synthetic draw (its mask differs); the
            # compress cost does not depend on the values
            fa.fa_compress(plan, K, V, phiT, caches[-1], stream)
            t_comp.append(_time(lambda: fa.fa_compress(plan, K, V, phiT, caches[-1], stream), 1, stream))
        del K, V
        torch.cuda.empty_cache()
        ws = torch.empty(max(fa.fa_decode_workspace_size(p) for p in plans), dtype=torch.uint8, device=dev)
        out = torch.empty(B, 32, 128, dtype=torch.bfloat16, device=dev)

        def step(s=stream):
            for p, c in zip(plans, caches):
                fa.fa_decode(p, q, c, out, ws, 0, s)
        step()
        n = 3 if B * L >= 32 * 131072 else 10
        td_eager = _time(step, n, stream)
        td = _time_graph(step, n)
        fa.fa_device_status(stream)
        wms = [work_model(wl.llama3_8b_layer(B, L, l), p) for l, p in enumerate(plans)]
        dbytes = sum(m["decode_bytes"] for m in wms)
        cflops = sum(m["compress_flops"] for m in wms)
        cbytes = sum(m["compress_bytes"] for m in wms)
        tcomp = sum(t_comp)
        print(json.dumps({"sweep": "llama3_8b_32_layers", "B": B, "L": L, "k": w0.k,
                          "layers_resident": resident, "layers": 32,
                          "compress_us_32_layers": tcomp * 1e3,
                          "compress_tflops": cflops / tcomp / 1e9,
                          "compress_frac_hbm": cbytes / tcomp / 1e6 / hbm,
                          "decode_us_per_step": td * 1e3,
                          "decode_us_per_step_eager": td_eager * 1e3,
                          "decode_timing": "CUDA graph replay of the 32 layer calls",
                          "decode_hbm_gbs": dbytes / td / 1e6,
                          "decode_frac_hbm": dbytes / td / 1e6 / hbm}), flush=True)
        del caches, plans, ws, out, q, phiT
        torch.cuda.empty_cache()


def run_fft_probe(args):
    """Measurement for the FFT variant of the decode (the skill page's Steps 2 and 4 use
    rfft / irfft). An O(M log M) decode of one layer would, per query head: synthesise the
    compressed-dim scores of all M middle tokens as one inverse real FFT of the zero-padded
    spectrum w (length P), add the exact-dim scores and take the softmax (one pass over the
    B Hq x M score matrix), and form u = Phi^T p as one forward real FFT of p. This times those
    three steps with cuFFT (torch.fft, fp32; the exact-dim stream is not included) at the
    plan's period P and at the next power of two, beside fa_decode on the same workload
    (CUDA-graph replays). Library FFTs are a lower bound for a hand-written one."""
    import torch

    import fourier_basis_attention_b200 as fa
    import workloads as wl
    dev = torch.device("cuda", 0)
    for w in (wl.LLAMA3_8B_GQA_32K, wl.LLAMA3_8B_GQA_128K):
        mask = wl.dim_mask(w)
        K = wl.kv_cache(w, "K", device=dev)
        V = wl.kv_cache(w, "V", device=dev)
        q = wl.queries(w, device=dev)
        plan = fa.fa_plan_init(w.B, w.Hq, w.Hkv, w.L, w.S, w.R, w.k, mask)
        cache = fa.Cache(plan, device=dev)
        fa.fa_compress(plan, K, V, fa.basis_table(plan), cache)
        del K, V
        ws = torch.empty(fa.fa_decode_workspace_size(plan), dtype=torch.uint8, device=dev)
        out = torch.empty(w.B, w.Hq, 128, dtype=torch.bfloat16, device=dev)
        t_dec = _time_graph(lambda s: fa.fa_decode(plan, q, cache, out, ws, 0, s), 30)
        fa.fa_device_status()
        del cache, ws
        torch.cuda.empty_cache()
        nh = w.B * w.Hq
        res = {"workload": w.name, "query_heads": nh, "M": plan.M, "k": w.k,
               "fa_decode_us": round(t_dec * 1e3, 1),
               "fa_decode_path": SPLIT_NAMES.get(fa.fa_decode_describe(plan, 0).split_kernel)}
        for P in (plan.P, 1 << (plan.P - 1).bit_length()):
            spec = torch.zeros(nh, P // 2 + 1, dtype=torch.complex64, device=dev)
            spec[:, :(w.k + 1) // 2 + 1] = torch.randn(nh, (w.k + 1) // 2 + 1, dtype=torch.complex64,
                                                      device=dev)
            sc = torch.empty(nh, P, dtype=torch.float32, device=dev)
            pr = torch.empty_like(sc)
            uu = torch.empty(nh, P // 2 + 1, dtype=torch.complex64, device=dev)

            def synth(s):
                with torch.cuda.stream(s):
                    torch.fft.irfft(spec, n=P, dim=1, out=sc)

            def softmax(s):
                with torch.cuda.stream(s):
                    pr.copy_(torch.softmax(sc, dim=1))

            def analyse(s):
                with torch.cuda.stream(s):
                    torch.fft.rfft(pr, dim=1, out=uu)

            ts = [_time_graph(f, 30) for f in (synth, softmax, analyse)]
            res[f"P{P}"] = {"irfft_scores_us": round(ts[0] * 1e3, 1), "softmax_us": round(ts[1] * 1e3, 1),
                            "rfft_values_us": round(ts[2] * 1e3, 1),
                            "sum_us": round(sum(ts) * 1e3, 1)}
            del spec, sc, pr, uu
            torch.cuda.empty_cache()
        print(json.dumps(res), flush=True)
        del q, out


SPLIT_NAMES = {0: "none", 1: "CUDA cores", 2: "tcgen05 token-major", 3: "warp MMA",
               4: "tcgen05 slot-split cluster"}


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.fft_probe:
        run_fft_probe(args)
    elif args.sweep:
        run_sweep(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
