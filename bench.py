#!/usr/bin/env python
"""Benchmark of the B200 DashAttention forward pass (prefill + decode), one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 16k|32k|96k] [--no-decode]
    python bench.py --impl reference ...      # the fp64 CPU oracle timed on this host

A step is one full prefill (block summaries, coarse scores + alpha-entmax thresholds +
block lists, prior-weighted fine attention) of the workload (default: the 16K prefill
at 75 % block sparsity).  The other prefill configurations (tiny, the 32K alpha sweep and
the 96K prefill at ~93.75 % block sparsity) are timed with the same steps and warm-up and
reported in `other_prefill_configs`.  `value` is prefill tokens/s over all ranks with inputs resident
in HBM; `e2e` is the same through the C ABI's host-buffer entry point (host<->device
copies inside the timed region).  The `decode` object times one decode step of the 96K
workload (B=8, cache 98304): its step is replayed from a CUDA graph, as a serving loop
runs it, and a profiled eager run gives the per-kernel split.  L2 is flushed before every
timed step (a 256 MiB write, then a 256 MiB read so that no dirty line of the flush is
written back inside the step); times are CUDA events on the launching stream, max over
ranks.

Multi-GPU: one process per GPU (torchrun), every rank runs its own replica of the
workload (work units are independent: weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill tok/s & decode tok/s at 16K–96K ctx; % of BF16 TC / HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def calibrated(name):
    with open(os.path.join(ROOT, "tests", "golden", "coarse_scale.json")) as f:
        return json.load(f)[name]


def source_sha(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "sparse_hierarchical_attention_pool_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, sha, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this workload
    and the kernel is unchanged since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel)
    if not d or d.get("source_sha256_16") != sha or d.get("workload_key") != workload:
        return None
    return d.get("traffic_bytes_per_launch")


class L2Flush:
    """Evicts the inputs from L2: a write pass over a buffer twice the L2 size, then a read
    pass over another, so the timed step starts with clean lines of unrelated data."""

    def __init__(self, nbytes=256 << 20):
        import torch
        self.w = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        self.r = torch.ones(nbytes // 4, dtype=torch.float32, device="cuda")

    def __call__(self):
        self.w.zero_()
        self.r.amax()


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms during a timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        import torch
        ident = str(self.dev)
        try:
            ident = str(torch.cuda.get_device_properties(self.dev).uuid)
            if not ident.startswith("GPU-"):
                ident = "GPU-" + ident
        except Exception:
            pass
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={ident}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = sorted(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if _num(r[3]))}


def _num(s):
    try:
        float(s)
        return True
    except ValueError:
        return False


# ------------------------------------------------------------------ distributed plumbing

_REPLICAS = None


def dist_setup(n_gpus):
    """One process per GPU (independent replicas, see replicas.py): (world, rank, local)."""
    global _REPLICAS
    from sparse_hierarchical_attention_pool_b200.replicas import Replicas
    _REPLICAS = Replicas(timeout_s=300.0)
    return _REPLICAS.world, _REPLICAS.rank, _REPLICAS.local


def barrier(ws):
    if _REPLICAS is not None:
        _REPLICAS.barrier()


def max_over_ranks(ws, x):
    return x if _REPLICAS is None else _REPLICAS.max(x)


# ------------------------------------------------------------------ GPU arms

def time_prefill(wl, qd, kd, vd, alpha, cs, steps, warmup, flush, ws, wsb=None, clocks_dev=None):
    """Times `steps` full prefills (after `warmup` untimed ones) of one workload with the
    profiled entry point (CUDA events between the three kernels, on the launching stream;
    L2 flushed before each step) and derives the roofline figures of the fine kernel and of
    the block-summary kernel from the call's own counters.  Returns a plain dict."""
    import torch
    from sparse_hierarchical_attention_pool_b200 import dash_attn as da
    B, Hq, Hkv, T, d = wl.B, wl.Hq, wl.Hkv, wl.T, wl.d
    out = torch.empty_like(qd)
    if wsb is None:
        wsb = da.alloc_workspace(da.prefill_workspace_size(B, Hq, Hkv, T, d))
    for _ in range(warmup):
        flush()
        da.dash_prefill(qd, kd, vd, out, alpha, cs, wsb)
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    clk = None
    if clocks_dev is not None:
        clk = ClockSampler(clocks_dev)
        clk.start()
        time.sleep(0.3)
    evs = []
    for _ in range(steps):
        flush()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        da.dash_prefill_profiled(qd, kd, vd, out, alpha, cs, wsb, e)
        evs.append(e)
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    clocks = clk.stop() if clk is not None else None
    mean = lambda xs: sum(xs) / len(xs)  # noqa: E731
    tot = [e[0].elapsed_time(e[3]) for e in evs]
    summ = [e[0].elapsed_time(e[1]) for e in evs]
    coarse = [e[1].elapsed_time(e[2]) for e in evs]
    fine = [e[2].elapsed_time(e[3]) for e in evs]
    step_ms = max_over_ranks(ws, mean(tot))
    st = da.dash_prefill_stats(wsb)
    if da.dash_get_device_status(wsb) != 0:
        raise RuntimeError(f"device status not clean after the timed prefill of {wl.name}")
    # algorithmic work: fine FLOPs = 4 d * sum_rows |L_row|; coarse FLOPs = 2 d * sum_rows bt
    diag_tokens = sum((t % 64) + 1 for t in range(T)) * B * Hq
    fine_alg = 4.0 * d * (64.0 * st["selected_pairs"] + diag_tokens)
    coarse_alg = 2.0 * d * st["scored_pairs"]
    # executed: every step of a 128-row tile multiplies 64 keys for all 128 rows
    fine_exec = 4.0 * d * 64.0 * 128.0 * st["fine_steps"]
    pk, pk_kind = peaks()
    peak = pk["bf16_tflops"]
    fine_ms = mean(fine)
    achieved = fine_alg / (fine_ms * 1e-3) / 1e12
    # block-summary kernel: reads K, writes the fp32 means and their bf16 hi/lo parts
    nb = T // 64
    sum_bytes = B * Hkv * T * d * 2 + B * Hkv * nb * d * (4 + 2 + 2)
    sum_gbs = sum_bytes / (mean(summ) * 1e-3) / 1e9
    G = Hq // Hkv
    fine_kernel = "fine_tc_kernel" if G <= 16 else "fine_mma_kernel"
    return {
        "workload": wl.name, "alpha": alpha, "coarse_scale": cs, "seed": wl.seed,
        "B": B, "Hq": Hq, "Hkv": Hkv, "T": T, "d": d,
        "steps": steps, "warmup": warmup,
        "step_ms": step_ms, "tok_s": ws * B * T / (step_ms * 1e-3),
        "stage_ms": {"block_summary": mean(summ), "coarse_select": mean(coarse), "fine_attention": fine_ms},
        "stats": st, "clocks": clocks,
        "sparsity": 1.0 - st["selected_pairs"] / max(1, st["scored_pairs"]),
        "roofline": {"bound": "tensor", "kernel": fine_kernel, "achieved": round(achieved, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": f"{pk_kind} bf16_tflops (burst)",
                     "algorithmic_flops_per_launch": fine_alg,
                     "executed_flops_per_launch": fine_exec,
                     "executed_tflops": round(fine_exec / (fine_ms * 1e-3) / 1e12, 2),
                     "executed_frac": round(fine_exec / (fine_ms * 1e-3) / 1e12 / peak, 4),
                     "inflation": round(fine_exec / fine_alg, 3)},
        "coarse_algorithmic_flops": coarse_alg,
        "summary_roofline": {"bound": "hbm", "kernel": "block_summary_kernel", "bytes_per_launch": sum_bytes,
                             "achieved": round(sum_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": round(sum_gbs / pk["hbm_gbs"], 4)},
        # block summary, coarse, fine; with selection-ordered tiles also the two ordering kernels
        "launches_per_step": 5 if (Hq // Hkv <= 16 and T >= 64 and os.environ.get("DASH_TILES") != "positions") else 3,
        "l2": "flushed before every timed step",
        "_wsb": wsb, "_out": out, "_fine_alg": fine_alg, "_fine_exec": fine_exec,
    }


def tau_start_timings(wl, qd, kd, vd, alpha, cs, steps, warmup, flush, ws, newton_ms):
    """The coarse stage with the histogram-started threshold solve (AdaSplash-2's
    initialisation) against the default start, same inputs and steps."""
    os.environ["DASH_ENTMAX_INIT"] = "histogram"
    try:
        r = time_prefill(wl, qd, kd, vd, alpha, cs, steps, warmup, flush, ws)
    finally:
        os.environ.pop("DASH_ENTMAX_INIT", None)
    return {"default_coarse_select_ms": newton_ms, "histogram_coarse_select_ms": r["stage_ms"]["coarse_select"],
            "note": "default: Newton from the root of a subset (the 16 group maxima of a row whose scores stay in TMEM, the 4 largest scores of each quarter of a streamed row)"}


def public(d):
    """The JSON-ready part of a time_prefill result."""
    return {k: v for k, v in d.items() if not k.startswith("_")}


def bench_prefill(args, ws, rank, local):
    import torch
    from sparse_hierarchical_attention_pool_b200 import dash_attn as da
    from sparse_hierarchical_attention_pool_b200 import inputs

    wl, (q, k, v) = inputs.make(args.workload)
    cal = calibrated(args.workload)
    cs, alpha = cal["coarse_scale"], wl.alpha
    B, Hq, Hkv, T, d = wl.B, wl.Hq, wl.Hkv, wl.T, wl.d
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    flush = L2Flush()
    core = time_prefill(wl, qd, kd, vd, alpha, cs, args.steps, args.warmup, flush, ws, clocks_dev=local)
    wsb, out = core["_wsb"], core["_out"]
    fine_alg, fine_exec = core["_fine_alg"], core["_fine_exec"]
    st = core["stats"]
    mean = lambda xs: sum(xs) / len(xs)  # noqa: E731
    # context only: dense causal attention FLOPs and torch's SDPA (flash) on the same tensors
    dense_flops = 4.0 * d * B * Hq * T * (T + 1) / 2
    import torch.nn.functional as F
    for _ in range(2):
        F.scaled_dot_product_attention(qd, kd, vd, is_causal=True, enable_gqa=True)
    sd = []
    for _ in range(5):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        F.scaled_dot_product_attention(qd, kd, vd, is_causal=True, enable_gqa=True)
        e1.record()
        sd.append((e0, e1))
    torch.cuda.synchronize()
    sdpa_ms = mean([a.elapsed_time(b) for a, b in sd])
    context = {"dense_causal_flops": dense_flops, "torch_sdpa_dense_causal_ms": round(sdpa_ms, 4),
               "torch_sdpa_tflops": round(dense_flops / (sdpa_ms * 1e-3) / 1e12, 1),
               "note": "library dense attention on the same inputs, for context only"}
    G = Hq // Hkv
    traffic = (recorded_traffic("fine_tc_kernel", source_sha("fine_tc.cu", "sm100.cuh", "common.cuh"), args.workload)
               if G <= 16 else recorded_traffic("fine_mma_kernel", source_sha("fine_mma.cu", "mma_sync.cuh", "common.cuh"),
                                                args.workload))
    core["roofline"]["traffic"] = traffic
    tau_start = tau_start_timings(wl, qd, kd, vd, alpha, cs, args.steps, args.warmup, flush, ws,
                                  core["stage_ms"]["coarse_select"])
    res = {
        "step_ms": core["step_ms"],
        "tok_s": core["tok_s"],
        "stage_ms": core["stage_ms"],
        "clocks": core["clocks"],
        "stats": st,
        "sparsity": core["sparsity"],
        "roofline": core["roofline"],
        "coarse_algorithmic_flops": core["coarse_algorithmic_flops"],
        "summary_roofline": core["summary_roofline"],
        "context": context,
        "launches_per_step": core["launches_per_step"],
        "tau_start": tau_start,
        "wl": wl, "cs": cs,
    }
    # end-to-end through the host-buffer entry point
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty_like(q).pin_memory()
    for _ in range(2):
        da.dash_prefill_host(qh, kh, vh, oh, qd, kd, vd, out, alpha, cs, wsb)
    torch.cuda.synchronize()
    barrier(ws)
    e2e_ms = []
    ne2e = max(3, min(args.steps, 20))
    for _ in range(ne2e):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        da.dash_prefill_host(qh, kh, vh, oh, qd, kd, vd, out, alpha, cs, wsb)
        e1.record()
        e2e_ms.append((e0, e1))
    torch.cuda.synchronize()
    e2e_step = max_over_ranks(ws, mean([a.elapsed_time(b) for a, b in e2e_ms]))
    res["e2e"] = {"value": ws * B * T / (e2e_step * 1e-3), "unit": "tok/s",
                  "h2d_bytes_per_step": q.numel() * 2 + k.numel() * 2 + v.numel() * 2,
                  "d2h_bytes_per_step": q.numel() * 2, "ms_per_step": e2e_step}
    if not args.no_backward:
        res["backward"] = bench_backward(args, ws, qd, kd, vd, out, wl, cs, st, fine_alg, fine_exec, flush)
    del flush, wsb
    return res


def bench_other_prefills(args, ws, rank):
    """The prefill configurations besides the headline one, each timed with the same steps
    and warm-up: the tiny configuration (its oracle timed in full on the host, rank 0 at
    N = 1), the 32K workload at alpha 1.25 / 1.5 / 2 with one coarse scale, and the 96K
    workload at ~93.75 % block sparsity (whose block-summary kernel reads 201 MB of keys, a
    size at which that kernel is not launch-bound)."""
    import torch
    from sparse_hierarchical_attention_pool_b200 import inputs
    flush = L2Flush()
    res = {}
    # tiny: B=1, Hq=Hkv=1, T=512, d=64, fp32 N(0, 1) rounded to bf16
    wl, (q, k, v) = inputs.make("tiny")
    cs = calibrated("tiny")["coarse_scale"]
    tiny = public(time_prefill(wl, q.cuda(), k.cuda(), v.cuda(), wl.alpha, cs, args.steps, args.warmup, flush, ws))
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        tiny["cpu_baseline"] = oracle_full_tiny(wl, q, k, v, cs)
    res["tiny"] = tiny
    # 32K: one input set and coarse scale, three alphas
    wl, (q, k, v) = inputs.make("32k")
    cs = calibrated("32k")["coarse_scale"]
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    del q, k, v
    sweep = {}
    wsb = None
    for alpha in (1.25, 1.5, 2.0):
        r = time_prefill(wl, qd, kd, vd, alpha, cs, args.steps, args.warmup, flush, ws, wsb=wsb)
        wsb = r["_wsb"]
        sweep[str(alpha)] = public(r)
    res["32k_alpha_sweep"] = sweep
    del qd, kd, vd, wsb, r
    torch.cuda.empty_cache()
    # 96K: B=1, Hq=32, Hkv=8, T=98304
    wl, (q, k, v) = inputs.make("96k")
    cs = calibrated("96k")["coarse_scale"]
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    del q, k, v
    r96 = public(time_prefill(wl, qd, kd, vd, wl.alpha, cs, args.steps, args.warmup, flush, ws))
    r96["tau_start"] = tau_start_timings(wl, qd, kd, vd, wl.alpha, cs, args.steps, args.warmup, flush, ws,
                                         r96["stage_ms"]["coarse_select"])
    res["96k"] = r96
    del qd, kd, vd
    torch.cuda.empty_cache()
    return res


def oracle_full_tiny(wl, q, k, v, cs):
    """The fp64 oracle over every row of the tiny configuration, timed on the host."""
    import oracle
    oracle.build()
    rows = [(0, 0, t) for t in range(wl.T)]
    qr = oracle.gather_q_rows(q, rows)
    threads = len(os.sched_getaffinity(0))
    oracle.forward_rows(qr, k, v, rows[:8], wl.Hq, 64, wl.alpha, cs, nthreads=threads)
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.forward_rows(qr, k, v, rows, wl.Hq, 64, wl.alpha, cs, nthreads=threads)
        reps += 1
        if time.perf_counter() - t0 > 1.0:
            break
    dt = (time.perf_counter() - t0) / reps
    return {"value": wl.T / dt, "unit": "tok/s", "cores": threads, "kind": "oracle",
            "ms_per_step": dt * 1e3,
            "sample": f"every row of the tiny configuration (T={wl.T}), fp64 C oracle with OpenMP over rows, "
                      f"mean of {reps} full passes"}


def backward_only(args, ws):
    """The backward measurement alone on the prefill workload (for profiling runs)."""
    import torch
    from sparse_hierarchical_attention_pool_b200 import dash_attn as da
    from sparse_hierarchical_attention_pool_b200 import inputs
    wl, (q, k, v) = inputs.make(args.workload)
    cs = calibrated(args.workload)["coarse_scale"]
    B, Hq, Hkv, T, d = wl.B, wl.Hq, wl.Hkv, wl.T, wl.d
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty_like(qd)
    wsb = da.alloc_workspace(da.prefill_workspace_size(B, Hq, Hkv, T, d))
    da.dash_prefill(qd, kd, vd, out, wl.alpha, cs, wsb)
    st = da.dash_prefill_stats(wsb)
    diag_tokens = sum((t % 64) + 1 for t in range(T)) * B * Hq
    fine_alg = 4.0 * d * (64.0 * st["selected_pairs"] + diag_tokens)
    fine_exec = 4.0 * d * 64.0 * 128.0 * st["fine_steps"]
    return bench_backward(args, ws, qd, kd, vd, out, wl, cs, st, fine_alg, fine_exec, L2Flush())


def bench_backward(args, ws, qd, kd, vd, out, wl, cs, st, fine_alg, fine_exec, flush):
    """Gradients of the same prefill (dash_prefill_backward: coarse stage again, then the
    D, query-major and key-major kernels) for an N(0, 1) upstream gradient."""
    import torch
    from sparse_hierarchical_attention_pool_b200 import dash_attn as da
    from sparse_hierarchical_attention_pool_b200 import inputs
    B, Hq, Hkv, T, d = wl.B, wl.Hq, wl.Hkv, wl.T, wl.d
    da.dash_prefill(qd, kd, vd, out, wl.alpha, cs)
    dout = inputs.out_grad(B, Hq, T, d, seed=wl.seed + 1).cuda()
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    bws = da.alloc_workspace(da.prefill_backward_workspace_size(B, Hq, Hkv, T, d))
    for _ in range(args.warmup):
        flush()
        da.dash_prefill_backward(qd, kd, vd, out, dout, wl.alpha, cs, dq, dk, dv, bws)
    torch.cuda.synchronize()
    barrier(ws)
    n = max(3, min(args.steps, 10))
    evs = []
    for _ in range(n):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        da.dash_prefill_backward(qd, kd, vd, out, dout, wl.alpha, cs, dq, dk, dv, bws)
        e1.record()
        evs.append((e0, e1))
    torch.cuda.synchronize()
    ms = max_over_ranks(ws, sum(a.elapsed_time(b) for a, b in evs) / n)
    if da.dash_get_device_status(bws) != 0 or not all(bool(torch.isfinite(t).all()) for t in (dq, dk, dv)):
        raise RuntimeError("backward: device status not clean or non-finite gradients")
    pk, pk_kind = peaks()
    # five products per (row, key) at minimum (S again, dP, dV, dK, dQ): 2.5x the forward's
    # four-flop-per-d count.  The tcgen05 kernels execute nine 2 d products per (row, key)
    # of the tiles' unions (S and dP in the statistics pass, S, dP and dQ in the dq pass,
    # S, dP, dV and dK in the key-major pass), 4.5x the forward's executed count; the
    # summary columns of S and the blocks a key-block pair carries for its partner are
    # not counted
    alg = 2.5 * fine_alg
    exe = 4.5 * fine_exec
    ach = alg / (ms * 1e-3) / 1e12
    return {"ms": round(ms, 4), "tok_s": ws * B * T / (ms * 1e-3), "steps": n,
            "kernels": ["block_summary_kernel", "coarse_tc_kernel", "bwd_rowdot_kernel",
                        "bwd_tc_kernel<statistics>", "bwd_tc_kernel<dq>", "bwd_dkv_tc_kernel"],
            "roofline": {"bound": "tensor", "achieved": round(ach, 2), "peak": pk["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(ach / pk["bf16_tflops"], 4),
                         "peak_source": f"{pk_kind} bf16_tflops (burst)",
                         "algorithmic_flops": alg, "executed_flops": exe,
                         "executed_tflops": round(exe / (ms * 1e-3) / 1e12, 2),
                         "note": "tcgen05 kernels (TMEM accumulators, TMA rings)"},
            "l2": "flushed before every timed call"}


def bench_decode(args, ws, rank, local):
    import torch
    from sparse_hierarchical_attention_pool_b200 import dash_attn as da
    from sparse_hierarchical_attention_pool_b200 import inputs

    over = {"B": args.decode_batch} if args.decode_batch else {}
    wl, (q, kc, vc, kv_len) = inputs.make("decode96k", **over)
    cs = calibrated("decode96k")["coarse_scale"]
    B, Hq, Hkv, T, d = wl.B, wl.Hq, wl.Hkv, wl.T, wl.d
    qd, kcd, vcd, lens = q.cuda(), kc.cuda(), vc.cuda(), kv_len.cuda()
    del kc, vc
    ksum = da.dash_block_summary(kcd)
    out = torch.empty_like(qd)
    wsb = da.alloc_workspace(da.decode_workspace_size(B, Hq, Hkv, T, d))
    flush = L2Flush()
    for _ in range(max(3, args.warmup)):
        flush()
        da.dash_decode(qd, kcd, vcd, ksum, lens, out, wl.alpha, cs, wsb)
    torch.cuda.synchronize()
    barrier(ws)
    steps = max(args.steps, 20)
    mean = lambda xs: sum(xs) / len(xs)  # noqa: E731
    # per-kernel split from a profiled eager run
    evs = []
    for _ in range(steps):
        flush()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        da.dash_decode_profiled(qd, kcd, vcd, ksum, lens, out, wl.alpha, cs, wsb, e)
        evs.append(e)
    torch.cuda.synchronize()
    st_ms = [mean([e[i].elapsed_time(e[i + 1]) for e in evs]) for i in range(3)]
    eager = mean([e[0].elapsed_time(e[3]) for e in evs])
    # the threshold solve started at the histogram edge instead of u = -1, for comparison
    os.environ["DASH_ENTMAX_INIT"] = "histogram"
    evn = []
    for _ in range(steps):
        flush()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        da.dash_decode_profiled(qd, kcd, vcd, ksum, lens, out, wl.alpha, cs, wsb, e)
        evn.append(e)
    torch.cuda.synchronize()
    del os.environ["DASH_ENTMAX_INIT"]
    coarse_hist_ms = mean([e[0].elapsed_time(e[1]) for e in evn])
    # the step as a serving loop runs it: one CUDA graph replay (header reset + 2 kernels)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        da.dash_decode(qd, kcd, vcd, ksum, lens, out, wl.alpha, cs, wsb)
    torch.cuda.current_stream().wait_stream(side)
    with torch.cuda.graph(graph):
        da.dash_decode(qd, kcd, vcd, ksum, lens, out, wl.alpha, cs, wsb)
    for _ in range(3):
        flush()
        graph.replay()
    torch.cuda.synchronize()
    barrier(ws)
    gev = []
    for _ in range(steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        gev.append((e0, e1))
    torch.cuda.synchronize()
    barrier(ws)
    tot = max_over_ranks(ws, mean([a.elapsed_time(b) for a, b in gev]))
    st = da.dash_decode_stats(wsb)
    if da.dash_get_device_status(wsb) != 0:
        raise RuntimeError("device status not clean after the timed decode")
    blk_bytes = 64 * d * 2 * 2
    gathered = (st["union_blocks"] + B * Hkv) * blk_bytes
    other = B * Hkv * (T // 64) * d * 4 + 2 * B * Hq * d * 2
    pk, pk_kind = peaks()
    attn_gbs = gathered / (st_ms[1] * 1e-3) / 1e9
    step_gbs = (gathered + other) / (tot * 1e-3) / 1e9
    traffic = recorded_traffic("decode_attn_tc_kernel",
                               source_sha("decode_tc.cu", "mma_sync.cuh", "sm100.cuh", "common.cuh"),
                               f"decode96k-b{B}")
    # end to end: the new query goes up, the graph runs, the output comes back (the cache
    # stays resident)
    qh, oh = q.pin_memory(), torch.empty_like(q).pin_memory()
    e2e = []
    for _ in range(steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        qd.copy_(qh, non_blocking=True)
        graph.replay()
        oh.copy_(out, non_blocking=True)
        e1.record()
        e2e.append((e0, e1))
    torch.cuda.synchronize()
    del graph
    e2e_ms = max_over_ranks(ws, mean([a.elapsed_time(b) for a, b in e2e]))
    return {
        "workload": wl.name, "coarse_scale": cs, "seed": wl.seed,
        "value": ws * B / (tot * 1e-3), "unit": "tok/s", "ms_per_step": tot,
        "timing": "CUDA graph replay of the step; stage_ms from an eager profiled run",
        "eager_ms_per_step": eager,
        "stage_ms": dict(zip(["coarse_select", "attention", "merge"], st_ms)),
        "tau_start": {"newton_from_minus_one_coarse_select_ms": st_ms[0],
                      "histogram_edge_coarse_select_ms": coarse_hist_ms},
        "sparsity": 1.0 - st["selected_pairs"] / max(1, st["scored_pairs"]),
        "union_blocks_per_group": st["union_blocks"] / (B * Hkv),
        "roofline": {"bound": "hbm", "kernel": "decode_attn_tc_kernel", "achieved": round(attn_gbs, 1),
                     "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(attn_gbs / pk["hbm_gbs"], 4),
                     "traffic": traffic, "peak_source": f"{pk_kind} hbm_gbs",
                     "algorithmic_bytes_per_launch": gathered,
                     "step_bytes": gathered + other, "step_frac": round(step_gbs / pk["hbm_gbs"], 4)},
        "e2e": {"value": ws * B / (e2e_ms * 1e-3), "unit": "tok/s", "h2d_bytes_per_step": q.numel() * 2,
                "d2h_bytes_per_step": q.numel() * 2},
        # block scores, threshold + lists, attention (with its in-kernel merge of split groups)
        "launches_per_step": 3,
        "stats": st,
    }


# ------------------------------------------------------------------ CPU oracle (baseline / reference arm)

def oracle_rows_per_s(workload, n_rows, seed, tensors=None):
    """Time the fp64 oracle on n_rows random rows of the workload; returns (rows/s, cores, wl)."""
    import oracle
    from sparse_hierarchical_attention_pool_b200 import inputs
    oracle.build()
    if tensors is None:
        wl, (q, k, v) = inputs.make(workload)
    else:
        wl, (q, k, v) = tensors
    cs = calibrated(workload)["coarse_scale"]
    rows = inputs.sample_rows(wl.B, wl.Hq, wl.T, n_rows, seed)
    qr = oracle.gather_q_rows(q, rows)
    threads = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    oracle.forward_rows(qr, k, v, rows, wl.Hq, 64, wl.alpha, cs, nthreads=threads)
    dt = time.perf_counter() - t0
    return n_rows / dt, threads, wl, dt


def cpu_baseline(args):
    from sparse_hierarchical_attention_pool_b200 import inputs
    tensors = inputs.make(args.workload)
    r, cores, wl, dt = oracle_rows_per_s(args.workload, 64, 1, tensors)
    n = int(max(64, min(20000, r * 10.0)))            # about 10 s of oracle work
    r, cores, wl, dt = oracle_rows_per_s(args.workload, n, 2, tensors)
    return {"value": r / wl.Hq, "unit": "tok/s", "cores": cores, "kind": "oracle",
            "rows_per_s": r, "rows_per_s_per_core": r / cores,
            "sample": f"{n} uniformly drawn rows (b, h, t) of the {wl.name} workload, fp64 C oracle "
                      f"with OpenMP over rows on {cores} threads, {dt:.1f} s; tok/s = rows/s / Hq "
                      "(extrapolated); per core = all-thread rate / threads"}


def run_reference(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from sparse_hierarchical_attention_pool_b200 import inputs
    tensors = inputs.make(args.workload)
    wl = tensors[0]
    r, cores, _, _ = oracle_rows_per_s(args.workload, 32, 1, tensors)
    n = int(max(16, min(5000, r * 2.0)))               # about 2 s per step
    for i in range(args.warmup):
        oracle_rows_per_s(args.workload, max(8, n // 4), 100 + i, tensors)
    times = []
    for i in range(args.steps):
        rr, cores, _, dt = oracle_rows_per_s(args.workload, n, 200 + i, tensors)
        times.append(dt)
    step_s = sum(times) / len(times)
    value = n / step_s / wl.Hq
    line = {"metric": METRIC, "value": value, "unit": "tok/s", "impl": "reference", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "T": wl.T, "d": wl.d,
                       "block": wl.block, "alpha": wl.alpha, "coarse_scale": calibrated(args.workload)["coarse_scale"],
                       "seed": wl.seed},
            "cpu_baseline": {"value": value, "unit": "tok/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step: {n} uniformly drawn rows of the workload (fp64 C oracle, "
                                       "OpenMP over rows); tok/s = rows/s / Hq (extrapolated)"},
            "e2e": {"value": value, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="16k", choices=["16k", "32k", "96k", "16k-coherent"],
                    help="16k-coherent is not a target workload: block-coherent query topics")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-backward", action="store_true", help="skip the prefill backward measurement")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the tiny, 32K alpha-sweep and 96K prefill measurements")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the prefill backward and print its object (for profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-only", action="store_true",
                    help="time only the decode step and print its object (for profiling runs)")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="decode batch other than the workload's 8 (smaller profiling captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    ws, rank, local = dist_setup(args.gpus)
    from sparse_hierarchical_attention_pool_b200 import build as _b
    if rank == 0:
        _b.build()
    barrier(ws)
    if args.backward_only:
        bwd = backward_only(args, ws)
        if rank == 0:
            print(json.dumps(bwd), flush=True)
        if ws > 1:
            barrier(ws)
            _REPLICAS.close()
        return
    if args.decode_only:
        dec = bench_decode(args, ws, rank, local)
        if rank == 0:
            print(json.dumps(dec), flush=True)
        if ws > 1:
            barrier(ws)
            _REPLICAS.close()
        return
    pre = bench_prefill(args, ws, rank, local)
    others = None if args.no_other_configs else bench_other_prefills(args, ws, rank)
    dec = None if args.no_decode else bench_decode(args, ws, rank, local)
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args)
    if rank == 0:
        wl = pre["wl"]
        line = {
            "metric": METRIC, "value": pre["tok_s"], "unit": "tok/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": pre["step_ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "T": wl.T, "d": wl.d,
                       "block": wl.block, "alpha": wl.alpha, "coarse_scale": pre["cs"], "seed": wl.seed,
                       "realised_sparsity": round(pre["sparsity"], 5),
                       "l2": "flushed before every timed step (256 MiB write + 256 MiB read, outside the step's events)",
                       "parallelism": f"independent replica per GPU x{ws}"},
            "roofline": pre["roofline"],
            "e2e": pre["e2e"],
            "cpu_baseline": cpu,
            "clocks": pre["clocks"],
            "gpu_launches": pre["launches_per_step"] * args.steps,
            "stage_ms": pre["stage_ms"],
            "tau_start": pre["tau_start"],
            "summary_roofline": pre["summary_roofline"],
            "context": pre["context"],
            "prefill_stats": pre["stats"],
            "backward": pre.get("backward"),
            "decode": dec,
            "other_prefill_configs": others,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        barrier(ws)
        _REPLICAS.close()


if __name__ == "__main__":
    main()
