#!/usr/bin/env python
"""Benchmark of the cluster-attention forward pass (libclusterattn on B200).

One step = one full forward (k-means, centroid attention, gather, window
attention, blend) over one batch of a seeded synthetic workload, inputs
already resident in HBM.  L2 is flushed (a 256 MiB write, outside the timed
event pairs) before every timed step.  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the fp64 CPU oracle arm

Under torchrun (N > 1) every rank runs its own full copy of the workload on
its own GPU (independent heads, no data-path collective: weak scaling); the
step time is the max over ranks.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "cluster-attention fwd tokens/s (B·H·L/s) and achieved HBM GB/s vs ~8 TB/s"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "l32k_dup_bf16"
# Timed beside the headline: the other workloads the roofline target is stated on.
DEFAULT_ALSO = "l4k_gmm_bf16,l512_bf16"
FALLBACK_HBM_GBS = 6650.0
# Heads of each workload the parity block re-checks against the fp64 oracle
# (every head: the oracle needs about a second per 32k-token head per thread).
PARITY_HEADS = {"small_f32": 24, "card_gmm_f32": 384, "l512_bf16": 768, "l4k_gmm_bf16": 96,
                "l32k_dup_bf16": 16}
PRECISION = {
    "bf16": ("bf16 Q/K/V and O in HBM; bf16 tensor-core operands with fp32 accumulation; "
             "k-means decisions exact on fp32 centroids (certified filter + fp64 re-measure, exact fp64 "
             "member sums); one rounding of O to bf16"),
    "f32": ("fp32 Q/K/V and O; fp32 FMA with fp64 re-measure for the k-means decisions, exact fp64 "
            "member sums; fp32 attention arithmetic"),
}
# Kernel whose launches the roofline object reports, per workload.
DOMINANT = {"small_f32": "window_blend", "card_gmm_f32": "window_blend", "l512_bf16": "fused_forward",
            "l4k_gmm_bf16": "tiled_assign", "l32k_dup_bf16": "tiled_assign"}


def workload_desc(w) -> dict:
    src = {"normal": "N(0,1)", "gmm": f"Q {w.gmm_components}-component Gaussian mixture (means N(0,4I), std {w.gmm_std}), K,V N(0,1)"}[w.q_kind]
    if w.dup_frac:
        src += f", {int(w.dup_frac * 100)}% of tokens duplicated (forced ties / empty clusters)"
    return {"workload": f"{w.name}: B={w.B}, H={w.H}, L={w.L}, d={w.d}, K={w.K}, iters={w.iters}, "
                        f"W={w.W}, alpha={w.alpha}; {w.dtype} {src}, seed 0",
            "B": w.B, "H": w.H, "L": w.L, "d": w.d, "K": w.K, "iters": w.iters, "W": w.W,
            "alpha": w.alpha, "io_dtype": w.dtype, "tokens_per_step": w.tokens,
            "l2": "flushed before every timed step (256 MiB write outside the timed events)"}


def dist_info():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(values, dist=None, device=None):
    """Element-wise max of a list of floats over all ranks (identity alone)."""
    if dist is None:
        return [float(x) for x in values]
    import torch
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_rate(tokens_per_rank: int, world: int, ms_per_step: float) -> float:
    """Weak scaling: every rank processes its own full workload; the job's
    throughput is all ranks' tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (ms_per_step / 1e3)


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or
    None when there is none or the kernel sources changed since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[workload][kernel]
        from means_cluster_attention_b200.build import source_hash
        if e.get("source_hash") != source_hash(kernel):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        with open(self.file.name) as f:
            rows = [r.strip().split(", ") for r in f if r.strip()]
        os.unlink(self.file.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < len(self.FIELDS):
                continue
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for n, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


_CALIBRATION = {}


def cpu_oracle_rate(w, target_s: float, max_heads=None):
    """Time the fp64 oracle (as it stands) on a bounded head sample of the
    workload on this host's cores.  Returns (tokens/s, cores, sample text)."""
    import oracle
    from means_cluster_attention_b200.inputs import make_inputs
    cores = oracle.default_threads()
    # calibrate on one head (once per workload), then size the sample to
    # about target_s
    if w.name not in _CALIBRATION:
        x1 = make_inputs(w, heads=1)
        t0 = time.perf_counter()
        oracle.forward(x1["q64"], x1["k64"], x1["v64"], K=w.K, iters=w.iters, W=w.W, alpha=w.alpha, nthreads=1)
        _CALIBRATION[w.name] = max(time.perf_counter() - t0, 1e-4)
    t1 = _CALIBRATION[w.name]
    heads = int(max(1, min(w.heads, (target_s / t1) * cores)))
    if max_heads:
        heads = min(heads, max_heads)
    heads = max(1, (heads // cores) * cores) if heads >= cores else heads
    x = make_inputs(w, heads=heads)
    used = min(cores, heads)
    t0 = time.perf_counter()
    oracle.forward(x["q64"], x["k64"], x["v64"], K=w.K, iters=w.iters, W=w.W, alpha=w.alpha, nthreads=used)
    dt = time.perf_counter() - t0
    passes = 1
    if heads == w.heads and dt < target_s:
        # the whole workload is shorter than the target: time repeated passes
        passes = int(min(1000, math.ceil(target_s / max(dt, 1e-3))))
        t0 = time.perf_counter()
        for _ in range(passes):
            oracle.forward(x["q64"], x["k64"], x["v64"], K=w.K, iters=w.iters, W=w.W, alpha=w.alpha,
                           nthreads=used)
        dt = time.perf_counter() - t0
    toks = heads * w.L * passes
    sample = (f"{passes} pass(es) over {heads} of {w.heads} heads (L={w.L}) of {w.name}, same recipe "
              f"and sizes, {toks} tokens in {dt:.2f} s on {used} threads")
    return toks / dt, used, sample, dt


def run_reference(args, w):
    ws, rank, local = dist_info()
    if rank != 0:
        return 0
    # Each step: a bounded head sample sized so warmup + steps end within ~3 min.
    per_step = max(0.5, min(10.0, args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup)))
    rates = []
    cores = sample = None
    for i in range(args.warmup + args.steps):
        rate, cores, sample, dt = cpu_oracle_rate(w, per_step)
        if i >= args.warmup:
            rates.append(rate)
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * w.tokens / value,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_desc(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _to_device(x, w, dev):
    import numpy as np
    import torch
    if w.dtype == "f32":
        conv = lambda a: torch.from_numpy(a).to(dev)
    else:
        conv = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    return conv(x["q"]), conv(x["k"]), conv(x["v"])


def time_workload(args, w, dev, pg, flush, clocks=None):
    """Warm up, then time exactly args.steps forwards of workload w (inputs
    resident in HBM, L2 flushed before every step outside the event pair).
    Returns the timing record and the device tensors."""
    import torch
    import means_cluster_attention_b200 as ca
    from means_cluster_attention_b200 import _lib
    from means_cluster_attention_b200.inputs import make_inputs

    x = make_inputs(w, seed=0)
    q, k, v = _to_device(x, w, dev)
    out = torch.empty_like(q)
    assign = torch.empty((w.B, w.H, w.L), dtype=torch.int32, device=dev)
    cent = torch.empty((w.B, w.H, w.K, w.d), dtype=torch.float32, device=dev)

    def step():
        ca.forward(q, k, v, w.K, w.iters, w.W, w.alpha, out=out, assign=assign, centroids=cent)

    for _ in range(args.warmup):
        step()
        flush.zero_()
    ca.sync_status()

    def timed_pass(profile_kernel):
        """args.steps steps between a barrier and a synchronize on both
        sides, each bracketed by CUDA events (L2 flushed before each, outside
        the events).  With profile_kernel, every launch of that kernel is
        also bracketed by CUDA events on its stream."""
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        if pg:
            pg.barrier()
        torch.cuda.synchronize()
        if profile_kernel:
            _lib.profile_start(profile_kernel)
        n0 = _lib.launch_count()
        for i in range(args.steps):
            flush.zero_()
            starts[i].record()
            step()
            ends[i].record()
        torch.cuda.synchronize()
        n_launch = _lib.launch_count() - n0
        kstat = _lib.profile_stop() if profile_kernel else None
        if pg:
            pg.barrier()
        return [s.elapsed_time(e) for s, e in zip(starts, ends)], n_launch, kstat

    # Headline pass: nothing but the forward between the step events.  An
    # event recorded between two launches ends the programmatic overlap of
    # the second with the first, so the per-kernel events of the roofline
    # figure are taken in a second pass of the same steps.
    if clocks:
        clocks.start()
    ms, n_launch, _ = timed_pass(None)
    clk = clocks.stop() if clocks else None
    dom = args.profile_kernel or DOMINANT.get(w.name, "kmeans_assign")
    ms_prof, _, kstat = timed_pass(dom)
    ca.sync_status()
    ms_step = sum(ms) / len(ms)
    ms_step_prof = sum(ms_prof) / len(ms_prof)
    k_ms = kstat.total_ms / max(1, kstat.launches)
    ms_step, k_ms, ms_step_prof = reduce_max([ms_step, k_ms, ms_step_prof], pg, dev)
    ws = dist_info()[0]
    value = whole_job_rate(w.tokens, ws, ms_step)

    peak, peak_kind = measured_peak()
    achieved = (kstat.algorithmic_bytes / max(1, kstat.launches)) / (k_ms / 1e3) / 1e9 if k_ms > 0 else 0.0
    step_bytes = 4.0 * w.tokens * w.d * w.elem_bytes
    roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "peak_kind": peak_kind,
                "traffic": ncu_traffic(dom, w.name),
                "kernel_ms_per_launch": k_ms, "launches_timed": int(kstat.launches),
                "kernel_timing": "second timed pass of the same steps with CUDA events around each launch "
                                 "of the kernel on its stream",
                "ms_per_step_kernel_pass": ms_step_prof,
                "alg_bytes_per_launch": kstat.algorithmic_bytes / max(1, kstat.launches),
                "step_alg_bytes": step_bytes, "step_achieved_gbs": step_bytes / (ms_step / 1e3) / 1e9,
                "step_frac": step_bytes / (ms_step / 1e3) / 1e9 / peak,
                "step_frac_of_8tbs": step_bytes / (ms_step / 1e3) / 8e12}
    rec = {"value": value, "unit": UNIT, "ms_per_step": ms_step, "step_ms_min": min(ms),
           "step_ms_median": statistics.median(ms), "roofline": roofline, "gpu_launches": int(n_launch),
           "config": workload_desc(w)}
    if clk is not None:
        rec["clocks"] = clk
    return rec, x, (q, k, v)


def parity_check(w, x, dev_inputs, n_heads):
    """Outside the timed region: one more forward with the per-iteration
    assignment history, then the fp64 oracle on the first n_heads heads.
    Reports the flip rate (final assignments that differ from the oracle's),
    per-iteration mismatches, centroid and output errors; the output error is
    taken against the oracle evaluated at the GPU's own assignments."""
    import numpy as np
    import torch
    import oracle
    import means_cluster_attention_b200 as ca
    from means_cluster_attention_b200.inputs import bf16_bits_to_f64

    q, k, v = dev_inputs
    B, H, L, d = q.shape
    hist = torch.full((B, H, max(w.iters, 1), L), -1, dtype=torch.int32, device=q.device)
    out, assign, cent = ca.forward(q, k, v, w.K, w.iters, w.W, w.alpha, assign_hist=hist, sync_check=True)
    torch.cuda.synchronize()
    heads = list(range(min(n_heads, B * H)))
    flat = lambda a: a.reshape((B * H,) + a.shape[2:])[heads][None]
    if out.dtype == torch.bfloat16:
        g_out = bf16_bits_to_f64(out.view(torch.int16).cpu().numpy().view(np.uint16))
    else:
        g_out = out.cpu().numpy().astype(np.float64)
    g_out, g_assign = flat(g_out), flat(assign.cpu().numpy())
    g_cent = flat(cent.cpu().numpy().astype(np.float64))
    g_hist = flat(hist.cpu().numpy()[:, :, :w.iters])
    xs = {n: np.ascontiguousarray(flat(x[n])) for n in ("q64", "k64", "v64")}
    t0 = time.perf_counter()
    r_out, r_assign, r_cent, r_hist = oracle.forward(xs["q64"], xs["k64"], xs["v64"], K=w.K, iters=w.iters,
                                                     W=w.W, alpha=w.alpha, hist=True)
    at_out, at_cent = oracle.forward_at(xs["q64"], xs["k64"], xs["v64"], g_assign, K=w.K, iters=w.iters,
                                        W=w.W, alpha=w.alpha)
    dt = time.perf_counter() - t0
    tokens = len(heads) * L
    flips = int((g_assign != r_assign).sum())
    denom = np.maximum(np.abs(at_cent), 1e-30)
    return {"heads_checked": len(heads), "of_heads": B * H, "tokens_checked": tokens,
            "flip_rate": flips / tokens, "final_assignment_flips": flips,
            "per_iteration_mismatches": int((g_hist != r_hist).sum()) if w.iters else 0,
            "centroids_bit_exact": bool(np.array_equal(g_cent, at_cent)),
            "centroid_max_rel_err": float((np.abs(g_cent - at_cent) / denom).max()),
            "max_abs_err_at_gpu_assign": float(np.abs(g_out - at_out).max()),
            "max_abs_err_vs_oracle": float(np.abs(g_out - r_out).max()),
            "tolerance": 2e-3 if w.dtype == "f32" else 2e-2, "oracle_seconds": round(dt, 2)}


def time_variants(args, w, dev_inputs, flush):
    """Step times of the module's variants (ca_forward_ex) on workload w, on
    the same device inputs: grouped key/value heads (H_kv = H / 4), the
    module's radius window (radius = W), key padding (the last 10% of every
    batch row invalid), the soft gather, and all of them together.  Each is
    timed like the headline (L2 flushed before every step, CUDA events around
    the forward), after its own warm-up; correctness of every variant is
    covered by the GPU tests against the oracle."""
    import torch
    import means_cluster_attention_b200 as ca
    q, k, v = dev_inputs
    B, H, L, d = q.shape
    hkv = max(1, H // 4)
    kg, vg = k[:, :hkv].contiguous(), v[:, :hkv].contiguous()
    valid = torch.ones((B, L), dtype=torch.uint8, device=q.device)
    valid[:, L - L // 10:] = 0
    cases = {
        "gqa_hkv_h_over_4": (q, kg, vg, w.W, {}),
        "radius_window_W": (q, k, v, w.W // 2, dict(window_mode=1)),
        "key_padding_10pct": (q, k, v, w.W, dict(key_valid=valid)),
        "soft_gather": (q, k, v, w.W, dict(gather_mode=1)),
        "all_together": (q, kg, vg, w.W // 2, dict(window_mode=1, key_valid=valid, gather_mode=1)),
    }
    out = {}
    for name, (qq, kk, vv, W, opts) in cases.items():
        def step():
            ca.forward_ex(qq, kk, vv, w.K, w.iters, W, w.alpha, **opts)
        for _ in range(args.warmup):
            step()
            flush.zero_()
        torch.cuda.synchronize()
        ms = []
        for _ in range(args.steps):
            flush.zero_()
            s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s_ev.record()
            step()
            e_ev.record()
            ms.append((s_ev, e_ev))
        torch.cuda.synchronize()
        t = sum(a.elapsed_time(b) for a, b in ms) / len(ms)
        out[name] = {"ms_per_step": t, "value": w.tokens / (t / 1e3), "unit": UNIT,
                     "window_arg_W": W, "options": sorted(opts)}
    ca.sync_status()
    return {"workload": w.name, **out}


def run_ours(args, w):
    import torch
    import means_cluster_attention_b200 as ca
    from means_cluster_attention_b200.inputs import WORKLOADS

    ws, rank, local = dist_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
        pg = dist

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    clocks = ClockSampler(local)
    rec, x, dev_inputs = time_workload(args, w, dev, pg, flush, clocks)
    q = dev_inputs[0]

    # End to end through the C ABI with host buffers (pinned), copies included.
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (t.cpu().pin_memory() for t in dev_inputs)
        oh = torch.empty_like(qh).pin_memory()
        n_e2e = max(3, min(args.steps, 10))
        for _ in range(2):
            ca.forward_host(qh, kh, vh, w.K, w.iters, w.W, w.alpha, out=oh)
        e_ms = []
        for _ in range(n_e2e):
            s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s_ev.record()
            ca.forward_host(qh, kh, vh, w.K, w.iters, w.W, w.alpha, out=oh)
            e_ev.record()
            torch.cuda.synchronize()
            e_ms.append(s_ev.elapsed_time(e_ev))
        e_step = reduce_max([sum(e_ms) / len(e_ms)], pg, dev)[0]
        nbytes = q.numel() * q.element_size()
        e2e = {"value": whole_job_rate(w.tokens, ws, e_step), "unit": UNIT, "h2d_bytes_per_step": 3 * nbytes,
               "d2h_bytes_per_step": nbytes, "ms_per_step": e_step}

    # The other bf16 workloads the HBM-roofline target is stated on: their own
    # timed lines (same steps / warm-up), context for the headline.
    others = {}
    extra = [n for n in (args.also.split(",") if args.also else []) if n and n != w.name]
    extra_inputs = {}
    for name in extra:
        ow = WORKLOADS[name]
        orec, ox, odev = time_workload(args, ow, dev, pg, flush)
        others[name] = orec
        extra_inputs[name] = (ow, ox, odev)

    line = {
        "metric": METRIC, "value": rec["value"], "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "precision": PRECISION[w.dtype], "data": "synthetic", "config": rec["config"],
        "roofline": rec["roofline"], "e2e": e2e, "gpu_launches": rec["gpu_launches"], "clocks": rec["clocks"],
        "step_ms_min": rec["step_ms_min"], "step_ms_median": rec["step_ms_median"],
    }
    if others:
        line["other_workloads"] = others
    if not args.no_variants and "l4k_gmm_bf16" in extra_inputs:
        ow, _, odev = extra_inputs["l4k_gmm_bf16"]
        line["variants"] = time_variants(args, ow, odev, flush)
    if pg:
        line["config"]["parallelism"] = f"replicas x{ws} (independent heads, no collective)"
    if rank == 0 and ws == 1 and not args.no_parity:
        par = {w.name: parity_check(w, x, dev_inputs, PARITY_HEADS.get(w.name, 8))}
        for name, (ow, ox, odev) in extra_inputs.items():
            par[name] = parity_check(ow, ox, odev, PARITY_HEADS.get(name, 8))
        line["parity"] = par
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        rate, cores, sample, _ = cpu_oracle_rate(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def main():
    from means_cluster_attention_b200.inputs import WORKLOADS
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--profile-kernel", default=None)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-parity", action="store_true")
    ap.add_argument("--no-variants", action="store_true",
                    help="skip the step times of the module's variants (on l4k_gmm_bf16)")
    ap.add_argument("--also", default=DEFAULT_ALSO,
                    help="comma-separated workloads timed beside the headline ('' for none)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
