"""Benchmark: one step = router + fine-stage forward + backward (sa_plan, sa_forward,
sa_backward) at the Wan2.1-14B-720p attention shape, 95% block sparsity.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 720p]

Prints ONE JSON line on rank 0.  ``value`` is effective TFLOP/s over the whole step
(all ranks' work / max-over-ranks device time), counting only the selected 64x64 tiles:
forward 4*D*64*64 and backward 10*D*64*64 FLOPs per selected tile (VSA page, FLOP
accounting: 4 * D * S * H * d * 3.5, i.e. forward 1 + backward 2.5).  Each rank runs an
independent problem of the same shape (weak scaling, no collective on the data path).
Inputs are larger than L2 and L2 is also flushed between steps (256 MiB write); every
time reported is the median over the timed steps (per-step values are on the line too).
Extra sections on the same line: ``fp8_forward`` (e4m3 Q/K configuration, 720p only) and
``gated`` (the coarse branch + gate layer: sa_plan_coarse, sa_forward_gated,
sa_backward_gated), skipped with ``--no-fp8`` / ``--no-gated``.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn fwd+bwd ms & effective TFLOPS at Wan-720p shape, 95% sparsity"
UNIT = "TFLOP/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def tile_flops(D: int, ntiles: int):
    fwd = 4.0 * D * 64 * 64 * ntiles
    return fwd, 2.5 * fwd


# ---------------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock/power/throttle samples every 200 ms in a temporary file.  Started
    before the warm-up (so its start-up is over long before the timed region) and
    summarised over the lines written between two ``mark()`` calls."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix="sa_clocks_", suffix=".csv")
        os.close(fd)

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={CLOCK_QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < 5.0:
            self.f.flush()
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.05)
        return self

    def mark(self) -> int:
        """Number of complete sample lines written so far."""
        if self.proc is None:
            return 0
        with open(self.path) as f:
            return sum(1 for line in f if line.endswith("\n"))

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self, first: int = 0, last: int | None = None):
        """Median SM clock under load and throttle reasons over sample lines [first, last]
        (one line past ``last`` is included: the sample that closes the interval)."""
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        lines = open(self.path).read().splitlines()
        try:
            os.remove(self.path)
        except OSError:
            pass
        window = lines[first:(None if last is None else last + 1)]
        rows = [[x.strip() for x in line.split(",")] for line in window]
        rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        under_load = [s for s, pw in zip(sm, power) if pw is not None and pw > 300] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip().lower() == "active"})
        return {"sm_mhz": statistics.median(under_load) if under_load else None,
                "sm_max_mhz": max(num(r[2]) or 0 for r in rows), "reasons": reasons, "samples": len(rows)}


def stats_ms(v):
    return {"median": round(statistics.median(v), 4), "mean": round(statistics.mean(v), 4),
            "min": round(min(v), 4), "max": round(max(v), 4)}


# ---------------------------------------------------------------------------------- ours
def run_ours(args, rank, world, dist):
    import torch

    import block_sparse_attention_cubes_b200 as sa
    import synth

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = synth.get_config(args.config)
    t_gen = time.time()
    host = synth.make_inputs(cfg, seed=rank_seed(rank))
    t_gen = time.time() - t_gen
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    npad, T = sa.geometry(p)
    x = {n: sa.tile(host[n].to(dev), p) for n in ("q", "k", "v", "do")}
    A = sa.Attention(p)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    launches = {"n": 0}

    def step(rec=None):
        if rec is not None:
            rec[0].record()
        idx, cnt = A.plan(x["q"], x["k"])
        launches["n"] += sa.last_launch_count()
        if rec is not None:
            rec[1].record()
        out, lse, out32 = A.forward(x["q"], x["k"], x["v"], idx, cnt)
        launches["n"] += sa.last_launch_count()
        if rec is not None:
            rec[2].record()
        g = A.backward(x["q"], x["k"], x["v"], out, lse, x["do"], idx, cnt, out_f32=out32)
        launches["n"] += sa.last_launch_count()
        if rec is not None:
            rec[3].record()
        return idx, cnt, out, lse, g

    def phases(recs):
        return [[r[i].elapsed_time(r[i + 1]) for r in recs] for i in range(3)]

    # the clock sampler runs from before the warm-up to after the timed steps; its samples
    # are summarised over the timed region only
    with ClockSampler(local) as clocks:
        wrecs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.warmup)]
        for w in range(args.warmup):
            flush.fill_(w & 0xff)
            last = step(wrecs[w])
        torch.cuda.synchronize()
        warm_phases = phases(wrecs)
        for op in (sa.OP_PLAN, sa.OP_FORWARD, sa.OP_BACKWARD):
            st = sa.device_status(A._ws[op])
            if st != 0:
                raise RuntimeError(f"device status {sa.STATUS_NAMES.get(st, st)} after warm-up")
        fallback_rows = sa.plan_fallback_rows(A._ws[sa.OP_PLAN])  # rows the last plan decided in fp64
        cnt = last[1]
        ntiles = int(cnt.sum().item())
        valid_fl = valid_only_flops(sa, p, cfg, last[0], cnt, dev)
        del last

        recs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        launches["n"] = 0
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        line0 = clocks.mark()
        for s in range(args.steps):
            flush.fill_(s & 0xff)     # evict L2 between steps (not timed)
            res = step(recs[s])
        torch.cuda.synchronize()
        line1 = clocks.mark()
        gpu_launches = launches["n"]
        if dist is not None:
            dist.barrier()
        # warm L2: the same step without the flush in between (context, not the headline)
        wl = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(5)]
        for s in range(5):
            step(wl[s])
        torch.cuda.synchronize()
    clock_summary = clocks.summary(line0, line1)
    balance = measure_balance(sa, p, x, res[0], res[1], flush)
    plan_ms, fwd_ms, bwd_ms = phases(recs)
    step_ms = [a + b + c for a, b, c in zip(plan_ms, fwd_ms, bwd_ms)]
    ms_per_step = max_over_ranks(statistics.median(step_ms), dist, dev)
    fwd_fl, bwd_fl = tile_flops(cfg.D, ntiles)
    step_flops = (fwd_fl + bwd_fl) * world
    value = step_flops / (ms_per_step * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    fwd_med, bwd_med, plan_med = (statistics.median(v) for v in (fwd_ms, bwd_ms, plan_ms))
    # dominant kernel: the forward kernel, timed with events around sa_forward on the launching
    # (current) stream inside the timed region; the call's two other launches (cube mask, query
    # pair union) are about 0.3% of its time, so this slightly understates the kernel's own rate.
    # A kernel timed on its own (tens of ms) takes the burst peak, measured with the same clocks free.
    fwd_tf = fwd_fl / (fwd_med * 1e-3) / 1e12
    fb_tf = (fwd_fl + bwd_fl) / ((fwd_med + bwd_med) * 1e-3) / 1e12
    peak_tf = peaks.get("bf16_tflops")
    roofline = {"kernel": "attn_fwd_kernel", "bound": "tensor", "achieved": round(fwd_tf, 2),
                "peak": peak_tf, "unit": "TFLOP/s", "frac": round(fwd_tf / peak_tf, 4),
                "traffic": traffic_for("attn_fwd_kernel", ntiles),
                "peak_source": f"{peak_src} bf16 dense, burst (cuBLAS, best of 10)",
                "algorithmic_flops_per_launch": fwd_fl,
                "fwd_bwd": {"achieved": round(fb_tf, 2), "frac": round(fb_tf / peak_tf, 4),
                            "frac_of_sustained": round(fb_tf / peaks.get("bf16_tflops_sustained", peak_tf), 4)},
                "run_sm_mhz": clock_summary.get("sm_mhz"),
                "peak_sustained_sm_mhz": (peaks.get("clocks_under_load") or {}).get("sm_mhz_median")}
    router_bytes = 2 * cfg.B * cfg.H * npad * cfg.D * 2 + 4 * (ntiles + cfg.B * cfg.H * T)
    router_gbs = router_bytes / (plan_med * 1e-3) / 1e9
    warm = phases(wl)

    result = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"Wan2.1-shaped attention ({args.config}): B={cfg.B}, H={cfg.H}, D={cfg.D}, latent "
                               f"{'x'.join(map(str, cfg.lat))} -> T={T} cubes of 64, Npad={npad}; top_k={cfg.top_k}, "
                               f"top_p={cfg.top_p}; step = sa_plan + sa_forward + sa_backward",
                   "B": cfg.B, "H": cfg.H, "D": cfg.D, "lat": list(cfg.lat), "T": T, "top_k": cfg.top_k,
                   "top_p": cfg.top_p, "density": round(ntiles / (cfg.B * cfg.H * T * T), 5), "selected_tiles": ntiles,
                   "l2": "inputs larger than L2; 256 MiB flush between steps",
                   "per_rank": "independent problem per rank (seed = rank)",
                   "timing": "median of the timed steps (CUDA events on the launching stream)"},
        "breakdown_ms": {"plan": round(plan_med, 4), "forward": round(fwd_med, 4), "backward": round(bwd_med, 4),
                         "fwd_plus_bwd": round(fwd_med + bwd_med, 4)},
        "step_ms": stats_ms(step_ms),
        "per_step_ms": {"plan": [round(v, 3) for v in plan_ms], "forward": [round(v, 3) for v in fwd_ms],
                        "backward": [round(v, 3) for v in bwd_ms]},
        "warmup_ms": {n: [round(v, 3) for v in vals] for n, vals in zip(("plan", "forward", "backward"), warm_phases)},
        "warm_l2_ms": {n: round(statistics.median(vals), 4) for n, vals in zip(("plan", "forward", "backward"), warm)},
        "fwd_bwd_tflops": round(fb_tf, 3),
        "valid_only": {"flops_fwd_bwd": valid_fl, "tflops": round(valid_fl / ((fwd_med + bwd_med) * 1e-3) / 1e12, 3),
                       "note": "4*D and 10*D FLOPs per valid (query row, key) pair of the selected tiles"},
        "router": {"achieved_gbs": round(router_gbs, 1), "peak_gbs": peaks.get("hbm_gbs"),
                   "frac": round(router_gbs / peaks.get("hbm_gbs"), 4), "algorithmic_bytes": router_bytes,
                   "fallback_rows": fallback_rows, "rows": int(cnt.numel())},
        "roofline": roofline,
        "gpu_launches": gpu_launches,
        "clocks": clock_summary,
        "cta_balance": balance,
        "gen_s": round(t_gen, 1),
    }
    if args.e2e_steps > 0:
        result["e2e"] = run_e2e(args, sa, A, p, host, dev, fwd_fl + bwd_fl, world, dist)
    gpu_sample = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gpu_sample = gpu_outputs_for_heads(res, cfg, oracle_heads(cfg.H))
    del res
    run_fp8 = args.config == "720p" and not args.no_fp8
    if run_fp8 or not args.no_gated:
        del x, A
    if run_fp8:
        result["fp8_forward"] = run_fp8_forward(args, sa, synth, rank, dev, flush, peak_tf, peaks.get("hbm_gbs"), dist)
    if not args.no_gated:
        result["gated"] = run_gated(args, sa, synth, cfg, host, rank, dev, flush, result["breakdown_ms"], dist)
    if args.extras:
        result["extras"] = run_extras(args, sa, cfg, host, dev, flush, dist)
    if gpu_sample is not None:
        result["cpu_baseline"], result["parity_sample"] = cpu_baseline(cfg, host, gpu_sample, ntiles,
                                                                       seconds=args.cpu_seconds)
    return result


def measure_balance(sa, p, x, idx, cnt, flush):
    """One more forward + backward (not timed) with per-CTA clock records: for each attention
    kernel, how long each CTA was busy (start to end, globaltimer) under the dynamic in-order
    item schedule, and how its items and pipeline steps were spread."""
    import torch
    res = {"source": "globaltimer at each CTA's start and end (SA_DEBUG_CTA_CLOCKS), one untimed forward + backward "
                     "per schedule, L2 flushed before each call"}
    for sched, flag in (("dynamic", 0), ("static", sa.DEBUG_STATIC_ITEMS)):
        pc = sa.make_params(p.B, p.H, p.D, (p.lat_t, p.lat_h, p.lat_w), p.top_k, p.top_p,
                            kv_capacity=p.kv_capacity, debug_flags=sa.DEBUG_CTA_CLOCKS | flag)
        wf, wb = sa.new_workspace(pc, sa.OP_FORWARD), sa.new_workspace(pc, sa.OP_BACKWARD)
        flush.fill_(7)
        out, lse, o32 = sa.forward(x["q"], x["k"], x["v"], idx, cnt, pc, ws=wf, with_f32=True)
        flush.fill_(8)
        sa.backward(x["q"], x["k"], x["v"], out, lse, x["do"], idx, cnt, pc, ws=wb, out_f32=o32)
        torch.cuda.synchronize()
        part = {"schedule": ("work items (cube pairs) in natural order from a per-launch counter, each to the next "
                             "free CTA (the library's schedule)") if flag == 0 else
                            "fixed round-robin share (CTA c: items c, c + grid, ...; SA_DEBUG_STATIC_ITEMS)"}
        for kernel, name, ws in ((0, "attn_fwd_kernel", wf), (1, "attn_dq_kernel", wb), (2, "attn_dkdv_kernel", wb)):
            r = sa.cta_clocks(ws, kernel).astype("float64")
            if len(r) == 0:
                continue
            busy = (r[:, 1] - r[:, 0]) / 1e6
            span = (r[:, 1].max() - r[:, 0].min()) / 1e6
            part[name] = {"ctas": len(r), "span_ms": round(span, 4), "busy_ms_max": round(busy.max(), 4),
                          "busy_ms_mean": round(busy.mean(), 4), "busy_ms_min": round(busy.min(), 4),
                          "max_over_mean": round(busy.max() / busy.mean(), 4),
                          "idle_frac": round(1.0 - busy.sum() / (len(r) * span), 4),
                          "items": [int(r[:, 2].min()), int(r[:, 2].max())],
                          "steps": [int(r[:, 3].min()), int(r[:, 3].max())],
                          "steps_max_over_mean": round(r[:, 3].max() / r[:, 3].mean(), 4)}
        res[sched] = part
        del wf, wb, out, lse, o32
    return res


def valid_only_flops(sa, p, cfg, idx, cnt, dev):
    """Forward + backward FLOPs counting only valid (query row, key) pairs of the selected
    tiles: sum over selected (i, j) of 14 * D * n_i * n_j, n = valid tokens of a cube."""
    import torch
    T = idx.shape[2]
    nv = torch.tensor(cube_valid_counts(cfg.lat), dtype=torch.float64, device=dev)
    total = 0.0
    for b in range(idx.shape[0]):
        for h in range(idx.shape[1]):
            used = torch.arange(idx.shape[3], device=dev)[None, :] < cnt[b, h][:, None]
            nk = torch.where(used, nv[idx[b, h].clamp(0, T - 1).long()], torch.zeros((), dtype=torch.float64,
                                                                                   device=dev)).sum(1)
            total += float((nk * nv).sum().item())
    return 14.0 * cfg.D * total


def cube_valid_counts(lat):
    """Valid tokens of every 4x4x4 cube of a latent grid, in cube order."""
    lt, lh, lw = lat
    out = []
    for ct in range((lt + 3) // 4):
        for ch in range((lh + 3) // 4):
            for cw in range((lw + 3) // 4):
                out.append(min(4, lt - 4 * ct) * min(4, lh - 4 * ch) * min(4, lw - 4 * cw))
    return out


def oracle_heads(H: int):
    """The heads the oracle leg runs on: the first two of each head type (uniform first half,
    sink second half)."""
    return sorted({0, min(1, H - 1), H // 2, min(H // 2 + 1, H - 1)})


def gpu_outputs_for_heads(res, cfg, heads):
    """Host copies of the last timed step's lists and outputs on the oracle leg's heads."""
    idx, cnt, out, lse, (dq, dk, dv) = res
    pick = lambda t: t[0, heads].cpu()
    return {"heads": heads, "idx": pick(idx), "cnt": pick(cnt), "out": pick(out).float(), "dq": pick(dq),
            "dk": pick(dk), "dv": pick(dv)}


def run_fp8_forward(args, sa, synth, rank, dev, flush, bf16_peak, hbm_peak, dist):
    """The e4m3 Q/K configuration (config "720p_fp8": k = 22, p = 0.9, ~97% sparsity):
    sa_plan + sa_forward with Q, K quantised per cube from the bf16 draws, V bf16.  The
    forward's S product runs at the fp8 rate and PV at the bf16 rate, so its tensor peak
    is 4/3 of the bf16 peak (half the FLOPs at twice the rate)."""
    import torch
    cfg = synth.get_config("720p_fp8")
    host = synth.make_inputs(cfg, seed=rank_seed(rank), names=("q", "k", "v"))
    pb = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p, qk_dtype=sa.FP8_E4M3)
    npad, T = sa.geometry(p)
    t = {n: sa.tile(host[n].to(dev), pb) for n in host}
    q8, qs = synth.quantize_e4m3_rows(t["q"])
    k8, ks = synth.quantize_e4m3_rows(t["k"])
    del t["q"], t["k"]
    A = sa.Attention(p)

    def step(rec=None):
        if rec is not None:
            rec[0].record()
        idx, cnt = A.plan(q8, k8, qs, ks)
        if rec is not None:
            rec[1].record()
        A.forward(q8, k8, t["v"], idx, cnt, qs, ks, with_f32=False)
        if rec is not None:
            rec[2].record()
        return cnt

    for _ in range(max(3, args.warmup)):
        cnt = step()
    torch.cuda.synchronize()
    for op in (sa.OP_PLAN, sa.OP_FORWARD):
        st = sa.device_status(A._ws[op])
        if st != 0:
            raise RuntimeError(f"fp8: device status {sa.STATUS_NAMES.get(st, st)}")
    ntiles = int(cnt.sum().item())
    steps = max(3, min(args.steps, 10))
    recs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    for s in range(steps):
        flush.fill_(s & 0xff)
        step(recs[s])
    torch.cuda.synchronize()
    plan_ms = statistics.median(r[0].elapsed_time(r[1]) for r in recs)
    fwd_ms = statistics.median(r[1].elapsed_time(r[2]) for r in recs)
    fwd_fl, _ = tile_flops(cfg.D, ntiles)
    tf = fwd_fl / (fwd_ms * 1e-3) / 1e12
    peak = bf16_peak * 4.0 / 3.0
    router_bytes = 2 * cfg.B * cfg.H * npad * cfg.D + 2 * 4 * cfg.B * cfg.H * T + 4 * (ntiles + cfg.B * cfg.H * T)
    return {"config": f"{cfg.name}: e4m3 Q/K with per-cube scales, V bf16, top_k={cfg.top_k}, top_p={cfg.top_p}",
            "density": round(ntiles / (cfg.B * cfg.H * T * T), 5), "selected_tiles": ntiles, "steps": steps,
            "plan_ms": round(plan_ms, 4), "forward_ms": round(fwd_ms, 4), "forward_tflops": round(tf, 2),
            "forward_peak_tflops": round(peak, 1), "forward_frac": round(tf / peak, 4),
            "router_gbs": round(router_bytes / (plan_ms * 1e-3) / 1e9, 1),
            "router_frac": round(router_bytes / (plan_ms * 1e-3) / 1e9 / hbm_peak, 4)}


def run_gated(args, sa, synth, cfg, host, rank, dev, flush, plain_ms, dist):
    """The full gated layer at the same shape: sa_plan_coarse (router + coarse branch),
    sa_forward_gated (fine stage + O = G * Repeat(Oc) + O_f) and sa_backward_gated (fine +
    coarse gradients, dG), timed like the main step.  Reports each phase and what the coarse
    branch adds to the plain step.  Its cube-level products (T x T x D per head: one in the
    forward, five in the backward) run on the fp32 FMA pipe."""
    import torch
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    npad, T = sa.geometry(p)
    t = {n: sa.tile(host[n].to(dev), p) for n in ("q", "k", "v", "do")}
    gate = synth.make_gate(cfg, seed=rank_seed(rank)).to(dev)
    ws = {op: sa.new_workspace(p, op, dev) for op in (sa.OP_PLAN_COARSE, sa.OP_FORWARD, sa.OP_BACKWARD_GATED)}
    co = sa.Coarse.empty(p, dev)
    shape = tuple(t["q"].shape)
    out = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    out32 = torch.empty(shape, dtype=torch.float32, device=dev)
    lse = torch.empty((cfg.B, cfg.H, npad), dtype=torch.float32, device=dev)
    grads = [torch.empty(shape, dtype=torch.float32, device=dev) for _ in range(3)]
    dgate = torch.empty((cfg.B, cfg.H, npad), dtype=torch.float32, device=dev)
    idx = torch.empty((cfg.B, cfg.H, T, p.kv_capacity), dtype=torch.int32, device=dev)
    cnt = torch.empty((cfg.B, cfg.H, T), dtype=torch.int32, device=dev)
    launches = {"n": 0}

    def step(rec=None):
        n = 0
        if rec is not None:
            rec[0].record()
        sa.plan_coarse(t["q"], t["k"], t["v"], p, kv_index=idx, kv_count=cnt, coarse=co, ws=ws[sa.OP_PLAN_COARSE])
        n += sa.last_launch_count()
        if rec is not None:
            rec[1].record()
        sa.forward_gated(t["q"], t["k"], t["v"], idx, cnt, p, co, gate, out=out, lse=lse, ws=ws[sa.OP_FORWARD],
                         out_f32=out32)
        n += sa.last_launch_count()
        if rec is not None:
            rec[2].record()
        sa.backward_gated(t["q"], t["k"], t["v"], out, lse, t["do"], gate, idx, cnt, p, co, dq=grads[0], dk=grads[1],
                          dv=grads[2], dgate=dgate, ws=ws[sa.OP_BACKWARD_GATED], out_f32=out32)
        n += sa.last_launch_count()
        if rec is not None:
            rec[3].record()
        launches["n"] += n

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    for op, w in ws.items():
        st = sa.device_status(w)
        if st != 0:
            raise RuntimeError(f"gated: device status {sa.STATUS_NAMES.get(st, st)} (op {op})")
    ntiles = int(cnt.sum().item())
    steps = max(3, min(args.steps, 10))
    recs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    launches["n"] = 0
    for s in range(steps):
        flush.fill_(s & 0xff)
        step(recs[s])
    torch.cuda.synchronize()
    per_step = [[r[i].elapsed_time(r[i + 1]) for r in recs] for i in range(3)]
    ms = [statistics.median(v) for v in per_step]
    fwd_fl, bwd_fl = tile_flops(cfg.D, ntiles)
    cube_fl = 2.0 * cfg.B * cfg.H * T * T * cfg.D      # one cube-level product
    total_ms = sum(ms)
    extra = {}
    if dist is None and not args.no_cpu_baseline:
        extra["cpu_baseline"] = cpu_baseline_gated(cfg, host, gate.cpu(), seconds=args.cpu_seconds)
    return {**extra, "config": f"{cfg.name}: O = G * Repeat(Oc) + O_f, gates tanh(N(0,1)), fp32 out kept",
            "steps": steps, "selected_tiles": ntiles,
            "plan_coarse_ms": round(ms[0], 4), "forward_gated_ms": round(ms[1], 4),
            "backward_gated_ms": round(ms[2], 4), "ms_per_step": round(total_ms, 4),
            "added_ms": {"plan": round(ms[0] - plain_ms["plan"], 4), "forward": round(ms[1] - plain_ms["forward"], 4),
                         "backward": round(ms[2] - plain_ms["backward"], 4)},
            "cube_level_gflop": round(6 * cube_fl / 1e9, 2),
            "effective_tflops": round((fwd_fl + bwd_fl + 6 * cube_fl) / (total_ms * 1e-3) / 1e12, 3),
            "gpu_launches_per_step": launches["n"] // steps,
            "per_step_ms": {n: [round(v, 3) for v in vals]
                            for n, vals in zip(("plan_coarse", "forward_gated", "backward_gated"), per_step)}}


def run_extras(args, sa, cfg, host, dev, flush, dist):
    """The other routers at the same shape (off by default, ``--extras``): sa_plan_bq128
    (128-token query blocks) timed with the fine forward and backward on its lists, like the
    main step; and the recall diagnostic, sa_recall on the lse of the forward with the cube
    router's lists and with every block (the dense forward is not timed), with its result."""
    import torch
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    npad, T = sa.geometry(p)
    t = {n: sa.tile(host[n].to(dev), p) for n in ("q", "k", "v", "do")}
    ws = {op: sa.new_workspace(p, op, dev) for op in (sa.OP_PLAN_BQ128, sa.OP_FORWARD, sa.OP_BACKWARD)}

    def step(rec=None):
        if rec is not None:
            rec[0].record()
        idx, cnt = sa.plan_bq128(t["q"], t["k"], p, ws=ws[sa.OP_PLAN_BQ128])
        if rec is not None:
            rec[1].record()
        out, lse, o32 = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p, ws=ws[sa.OP_FORWARD], with_f32=True)
        if rec is not None:
            rec[2].record()
        sa.backward(t["q"], t["k"], t["v"], out, lse, t["do"], idx, cnt, p, ws=ws[sa.OP_BACKWARD], out_f32=o32)
        if rec is not None:
            rec[3].record()
        return cnt

    for _ in range(max(3, args.warmup)):
        cnt = step()
    torch.cuda.synchronize()
    for op, w in ws.items():
        st = sa.device_status(w)
        if st != 0:
            raise RuntimeError(f"extras: device status {sa.STATUS_NAMES.get(st, st)} (op {op})")
    ntiles = int(cnt.sum().item())
    steps = max(3, min(args.steps, 5))
    recs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    torch.cuda.synchronize()
    for s in range(steps):
        flush.fill_(s & 0xff)
        step(recs[s])
    torch.cuda.synchronize()
    ms = [statistics.median(r[i].elapsed_time(r[i + 1]) for r in recs) for i in range(3)]
    fwd_fl, bwd_fl = tile_flops(cfg.D, ntiles)
    bq = {"plan_ms": round(ms[0], 4), "forward_ms": round(ms[1], 4), "backward_ms": round(ms[2], 4),
          "selected_tiles": ntiles, "density": round(ntiles / (cfg.B * cfg.H * T * T), 5),
          "effective_tflops": round((fwd_fl + bwd_fl) / (sum(ms) * 1e-3) / 1e12, 3)}
    # recall of the cube router's selection
    idx, cnt = sa.plan(t["q"], t["k"], p)
    _, lse_kept = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p)
    every = torch.arange(T, dtype=torch.int32, device=dev).expand(cfg.B, cfg.H, T, T).contiguous()
    full = torch.full((cfg.B, cfg.H, T), T, dtype=torch.int32, device=dev)
    _, lse_all = sa.forward(t["q"], t["k"], t["v"], every, full, p)
    del every
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    sa.recall(lse_kept, lse_all, p)
    ev[0].record()
    tau, cube = sa.recall(lse_kept, lse_all, p)
    ev[1].record()
    torch.cuda.synchronize()
    cube_cpu = cube.float().cpu()
    rec = {"recall_ms": round(ev[0].elapsed_time(ev[1]), 4), "mean_cube_recall": round(float(cube_cpu.mean()), 4),
           "min_cube_recall": round(float(cube_cpu.min()), 4),
           "cubes_below_half": round(float((cube_cpu < 0.5).float().mean()), 4),
           "mean_blocks_per_row": round(float(cnt.float().mean()), 2)}
    # P_oracle (token-level softmax mass per block pair) and the best recall at the router's counts
    pblock = sa.block_mass(t["q"], t["k"], lse_all, p)
    best = sa.best_recall(pblock, cnt, p)
    sel = torch.zeros_like(pblock)
    ar = torch.arange(idx.shape[-1], device=dev)
    keep = ar.view(1, 1, 1, -1) < cnt.unsqueeze(-1)
    sel.scatter_(3, torch.where(keep, idx.long(), 0), keep.float())
    got = (pblock * sel).sum(-1)
    ratio = (got / best.clamp_min(1e-30)).float().cpu()
    rec.update({"mean_oracle_recall": round(float(got.mean()), 4), "mean_best_recall": round(float(best.mean()), 4),
                "mean_recall_over_best": round(float(ratio.mean()), 4),
                "min_recall_over_best": round(float(ratio.min()), 4)})
    del pblock, sel, lse_all
    fine = run_fine_router(sa, cfg, t, p, T, dev, flush, steps)
    return {"config": f"{cfg.name}: sa_plan_bq128 + fine stage on its lists; recall of sa_plan's lists "
                      f"(token-level and against P_oracle's best at the same counts); VSA2 fine router",
            "steps": steps, "bq128": bq, "recall": rec, "fine_router": fine}


def run_fine_router(sa, cfg, t, p, T, dev, flush, steps, R=(2, 2, 2)):
    """VSA2's fine-grained router (sa_plan_fine, group pooling R) timed alone and with the fine
    forward and backward on its per-sequence Top-K lists."""
    import torch
    ws = {op: sa.new_workspace(p, op, dev) for op in (sa.OP_FORWARD, sa.OP_BACKWARD)}
    idx = torch.empty((cfg.B, cfg.H, T, p.kv_capacity), dtype=torch.int32, device=dev)
    cnt = torch.empty((cfg.B, cfg.H, T), dtype=torch.int32, device=dev)
    n = int(sa.load_library().sa_plan_fine_workspace_size(ctypes.byref(p), *R))
    wsf = torch.empty(n, dtype=torch.uint8, device=dev)

    def step(rec=None):
        if rec is not None:
            rec[0].record()
        sa.plan_fine(t["q"], t["k"], p, R=R, kv_index=idx, kv_count=cnt, ws=wsf)
        if rec is not None:
            rec[1].record()
        out, lse, o32 = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p, ws=ws[sa.OP_FORWARD], with_f32=True)
        if rec is not None:
            rec[2].record()
        sa.backward(t["q"], t["k"], t["v"], out, lse, t["do"], idx, cnt, p, ws=ws[sa.OP_BACKWARD], out_f32=o32)
        if rec is not None:
            rec[3].record()

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    for w in list(ws.values()) + [wsf]:
        st = sa.device_status(w)
        if st != 0:
            raise RuntimeError(f"fine router: device status {sa.STATUS_NAMES.get(st, st)}")
    recs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for s in range(steps):
        flush.fill_(s & 0xff)
        step(recs[s])
    torch.cuda.synchronize()
    ms = [statistics.median(r[i].elapsed_time(r[i + 1]) for r in recs) for i in range(3)]
    ntiles = int(cnt.sum().item())
    fwd_fl, bwd_fl = tile_flops(cfg.D, ntiles)
    c = cnt.float()
    return {"R": list(R), "plan_fine_ms": round(ms[0], 4), "forward_ms": round(ms[1], 4),
            "backward_ms": round(ms[2], 4), "selected_tiles": ntiles,
            "density": round(ntiles / (cfg.B * cfg.H * T * T), 5),
            "blocks_per_row": {"mean": round(float(c.mean()), 2), "min": int(c.min()), "max": int(c.max())},
            "effective_tflops": round((fwd_fl + bwd_fl) / (sum(ms) * 1e-3) / 1e12, 3)}


def cta_balance(masks, sms: int):
    """Per-CTA work of the persistent attention kernels, from the selection alone.

    ``masks``: one boolean [T, T] matrix per (b, h), M[i, j] = query cube i selected key
    cube j.  The forward and dQ kernels take query-cube pairs (rows 2p, 2p+1), the dK/dV
    kernel key-cube pairs (columns 2p, 2p+1); item it = bh * ceil(T/2) + pair goes to CTA
    it mod G with G = min(items, sms); one step covers two union entries (128 keys).
    Returns max/mean of per-CTA steps and tiles for both kernels, and the union
    inflation (union entries walked per selected tile)."""
    import numpy as np

    def pair_items(M):
        T = M.shape[0]
        if T % 2:
            M = np.concatenate([M, np.zeros((1, M.shape[1]), bool)])
        a, b = M[0::2], M[1::2]
        return (((a | b).sum(1) + 1) // 2), a.sum(1) + b.sum(1), (a | b).sum(1)

    def stats(item_steps, item_tiles):
        n = len(item_steps)
        G = min(n, sms)
        st = np.bincount(np.arange(n) % G, weights=item_steps, minlength=G)
        tl = np.bincount(np.arange(n) % G, weights=item_tiles, minlength=G)
        return {"ctas": G, "steps_max_over_mean": round(float(st.max() / st.mean()), 4),
                "tiles_max_over_mean": round(float(tl.max() / tl.mean()), 4),
                "steps_per_cta_mean": round(float(st.mean()), 1), "steps_per_cta_max": int(st.max())}

    q = [pair_items(M) for M in masks]
    k = [pair_items(M.T) for M in masks]
    qs, qt, qu = (np.concatenate([x[c] for x in q]) for c in range(3))
    ks, kt, _ = (np.concatenate([x[c] for x in k]) for c in range(3))
    return {"forward_dq": stats(qs, qt), "dkdv": stats(ks, kt),
            "union_entries_per_tile": round(float(qu.sum() / max(1, qt.sum())), 4)}


def selection_masks(idx, cnt):
    """[B,H,T,cap] index lists + counts -> one boolean [T, T] selection matrix per (b, h)."""
    import numpy as np
    ic, cc = idx.cpu().numpy(), cnt.cpu().numpy()
    B, H, T, cap = ic.shape
    masks = []
    for b in range(B):
        for h in range(H):
            M = np.zeros((T, T), bool)
            used = np.arange(cap)[None, :] < cc[b, h][:, None]
            rows = np.broadcast_to(np.arange(T)[:, None], (T, cap))
            M[rows[used], ic[b, h][used]] = True
            masks.append(M)
    return masks


def run_sweep(args):
    """Config-4 sweep at the 720p shape: k = 4, p in {0.8, 0.9, 0.95}, locality amplitude calibrated
    (at p = 0.9) for 80..98% sparsity.  One JSON line per point: step timings, the per-CTA load
    balance of the persistent attention kernels predicted from the lists under a fixed
    round-robin share, and the measured per-CTA busy times under the dynamic and the fixed
    schedules."""
    import torch

    import block_sparse_attention_cubes_b200 as sa
    import synth
    dev = torch.device("cuda", 0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    for sp in (80, 85, 90, 95, 98):
        for pp in (0.8, 0.9, 0.95):
            cfg = synth.get_config(f"sweep_{pp}_{sp}")
            host = synth.make_inputs(cfg, seed=0)
            p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
            npad, T = sa.geometry(p)
            x = {n: sa.tile(host[n].to(dev), p) for n in ("q", "k", "v", "do")}
            A = sa.Attention(p)

            def step(rec=None):
                if rec is not None:
                    rec[0].record()
                idx, cnt = A.plan(x["q"], x["k"])
                if rec is not None:
                    rec[1].record()
                out, lse, out32 = A.forward(x["q"], x["k"], x["v"], idx, cnt)
                if rec is not None:
                    rec[2].record()
                A.backward(x["q"], x["k"], x["v"], out, lse, x["do"], idx, cnt, out_f32=out32)
                if rec is not None:
                    rec[3].record()
                return idx, cnt

            for _ in range(3):
                idx, cnt = step()
            torch.cuda.synchronize()
            for op in (sa.OP_PLAN, sa.OP_FORWARD, sa.OP_BACKWARD):
                if sa.device_status(A._ws[op]) != 0:
                    raise RuntimeError(f"sweep {cfg.name}: device status {sa.device_status(A._ws[op])}")
            recs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
            for s in range(args.steps):
                flush.fill_(s & 0xff)
                step(recs[s])
            torch.cuda.synchronize()
            ms = [statistics.median(r[k].elapsed_time(r[k + 1]) for r in recs) for k in range(3)]
            ntiles = int(cnt.sum().item())
            fwd_fl, bwd_fl = tile_flops(cfg.D, ntiles)
            masks = selection_masks(idx, cnt)
            row_n = cnt[0].cpu().numpy().astype(float)
            line = {"config": cfg.name, "top_k": cfg.top_k, "top_p": cfg.top_p,
                    "sparsity": round(1 - ntiles / (cfg.H * T * T), 4), "selected_tiles": ntiles,
                    "blocks_per_row": {"mean": round(float(row_n.mean()), 1), "min": int(row_n.min()),
                                       "max": int(row_n.max())},
                    "plan_ms": round(ms[0], 3), "forward_ms": round(ms[1], 3), "backward_ms": round(ms[2], 3),
                    "forward_tflops": round(fwd_fl / (ms[1] * 1e-3) / 1e12, 1),
                    "backward_tflops": round(bwd_fl / (ms[2] * 1e-3) / 1e12, 1),
                    "balance": cta_balance(masks, sms),
                    "measured_balance": measure_balance(sa, p, x, idx, cnt, flush)}
            print(json.dumps(line), flush=True)
            del x, A


def run_one_pass(args):
    """One pass of every hot kernel on the seeded inputs of --config, nothing timed: sa_plan,
    sa_forward (fp32 copy), sa_backward, sa_plan_fine (R = 2x2x2), sa_plan_coarse,
    sa_forward_gated, sa_backward_gated.  Prints the selected tile counts."""
    import torch

    import block_sparse_attention_cubes_b200 as sa
    import synth
    cfg = synth.get_config(args.config)
    host = synth.make_inputs(cfg, 0)
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    x = {n: sa.tile(host[n].cuda(), p) for n in ("q", "k", "v", "do")}
    idx, cnt = sa.plan(x["q"], x["k"], p)
    out, lse, o32 = sa.forward(x["q"], x["k"], x["v"], idx, cnt, p, with_f32=True)
    sa.backward(x["q"], x["k"], x["v"], out, lse, x["do"], idx, cnt, p, out_f32=o32)
    _, fcnt = sa.plan_fine(x["q"], x["k"], p, R=(2, 2, 2))
    idx2, cnt2, co = sa.plan_coarse(x["q"], x["k"], x["v"], p)
    gate = synth.make_gate(cfg, 0).cuda()
    og, lg, o32g = sa.forward_gated(x["q"], x["k"], x["v"], idx2, cnt2, p, co, gate)
    sa.backward_gated(x["q"], x["k"], x["v"], og, lg, x["do"], gate, idx2, cnt2, p, co, out_f32=o32g)
    torch.cuda.synchronize()
    print(json.dumps({"one_pass": cfg.name, "tiles": int(cnt.sum()), "fine_tiles": int(fcnt.sum())}), flush=True)


def max_over_ranks(x: float, dist, device) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(rank: int) -> int:
    """Each rank draws an independent problem of the same shape."""
    return rank


def traffic_for(kernel: str, ntiles: int):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f).get(kernel)
    if not d or d.get("source_sha") != source_sha():
        return None
    # scale by selected tiles when the capture ran a smaller case
    per_tile = d["dram_bytes"] / d["tiles"]
    return int(per_tile * ntiles)


# What decides the forward kernel's DRAM traffic: its own source and device headers, and in
# the C ABI the tensor-map encoding, the argument setup and the forward entry point.
FWD_SOURCES = ("attn_fwd.cu", "attn_common.cuh", "geometry.cuh", "ptx.cuh")
FWD_ABI_FUNCTIONS = ("bool make_map(", "sa::AttnArgs base_args(", "sa_status forward_impl(", "sa_status sa_forward(")


def source_sha() -> str:
    """Hash of the forward kernel's sources (see FWD_SOURCES, FWD_ABI_FUNCTIONS)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "block_sparse_attention_cubes_b200", "csrc")
    for fn in FWD_SOURCES:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    with open(os.path.join(csrc, "api.cu")) as f:
        api = f.read()
    for sig in FWD_ABI_FUNCTIONS:
        i = api.index(sig)
        h.update(api[i:api.index("\n}\n", i) + 3].encode())
    return h.hexdigest()[:16]


def run_e2e(args, sa, A, p, host, dev, flops, world, dist):
    """Same step through the public API with host buffers (sa_step_host): pinned latent-order
    inputs are copied in, tiled, routed, run forward and backward, and out/dq/dk/dv are untiled
    and copied back, all inside the timed region, the copies of one chunk of heads overlapping
    the work on the neighbouring chunks.  The results of the last timed step are then compared
    with the device entry points run on the same inputs (they must be equal bit for bit)."""
    import torch
    pinned = {n: host[n].contiguous().pin_memory() for n in ("q", "k", "v", "do")}
    L = p.lat_t * p.lat_h * p.lat_w
    outs = [torch.empty((p.B, p.H, L, p.D), dtype=torch.bfloat16).pin_memory()]
    outs += [torch.empty((p.B, p.H, L, p.D), dtype=torch.float32).pin_memory() for _ in range(3)]
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = sum(t.numel() * t.element_size() for t in outs)
    chunk = max(1, min(args.e2e_chunk, p.B * p.H))
    ws = torch.empty(sa.step_host_workspace_size(p, chunk), dtype=torch.uint8, device=dev)

    def e2e_step():
        sa.step_host(pinned["q"], pinned["k"], pinned["v"], pinned["do"], p, chunk, *outs, ws=ws)

    e2e_step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, dist, dev)
    status = sa.device_status(ws)
    # the device path on the same inputs
    x = {n: sa.tile(pinned[n].to(dev), p) for n in pinned}
    idx, cnt = A.plan(x["q"], x["k"])
    out, lse, out32 = A.forward(x["q"], x["k"], x["v"], idx, cnt)
    grads = A.backward(x["q"], x["k"], x["v"], out, lse, x["do"], idx, cnt, out_f32=out32)
    same = all(torch.equal(sa.untile(r, p).cpu(), o) for r, o in zip((out, *grads), outs))
    del x, idx, cnt, out, lse, out32, grads
    return {"value": round(flops * world / (ms * 1e-3) / 1e12, 3), "unit": UNIT, "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "how": f"sa_step_host, {chunk} heads per chunk: chunk c copied in while c-1 is computed and c-2 "
                   f"copied out (pinned host buffers)",
            "device_status": sa.STATUS_NAMES.get(status, status), "equals_device_path": bool(same)}


# ---------------------------------------------------------------------------------- oracle
def oracle_sample(cfg, host, head: int, frac: float, seed: int = 0):
    """Run the fp64 oracle on one head: the full router, then forward and backward for a
    fixed sample of query blocks.  Returns (seconds, effective FLOPs of the sampled tiles)."""
    import numpy as np

    import oracle as O
    lay = O.cube_layout(cfg.lat)
    t = {n: O.tile(host[n][0, head].double().numpy(), lay) for n in ("q", "k", "v", "do")}
    T = lay.n_cubes
    rng = np.random.default_rng(seed)
    sample = np.sort(rng.choice(T, size=max(1, int(round(frac * T))), replace=False))
    t0 = time.perf_counter()
    tr = O.route_head(t["q"], t["k"], lay.valid, cfg.top_k, cfg.top_p)
    O.attention_forward_head(t["q"], t["k"], t["v"], tr.lists, lay.valid, q_blocks=sample)
    O.attention_backward_head(t["q"], t["k"], t["v"], t["do"], tr.lists, lay.valid, q_blocks=sample,
                              kv_blocks=range(T), visit=sample)
    secs = time.perf_counter() - t0
    ntiles = sum(len(tr.lists[i]) for i in sample)
    f, b = tile_flops(cfg.D, ntiles)
    return secs, f + b, len(sample)


def oracle_gated_sample(cfg, host, gate, head: int, frac: float, seed: int = 0):
    """The fp64 oracle's gated layer on one head: the full router and cube-level branch,
    the fine forward and backward on a fixed sample of query blocks (as ``oracle_sample``).
    Returns (seconds, effective FLOPs: the sampled tiles plus the six cube-level products)."""
    import numpy as np

    import oracle as O
    lay = O.cube_layout(cfg.lat)
    t = {n: O.tile(host[n][0, head].double().numpy(), lay) for n in ("q", "k", "v", "do")}
    g = gate[0, head].double().numpy()
    T = lay.n_cubes
    rng = np.random.default_rng(seed)
    sample = np.sort(rng.choice(T, size=max(1, int(round(frac * T))), replace=False))
    t0 = time.perf_counter()
    tr = O.route_head(t["q"], t["k"], lay.valid, cfg.top_k, cfg.top_p)
    O.gated_forward_head(t["q"], t["k"], t["v"], g, tr.lists, lay.valid, q_blocks=sample)
    O.gated_backward_head(t["q"], t["k"], t["v"], t["do"], g, tr.lists, lay.valid, q_blocks=sample,
                          kv_blocks=range(T), visit=sample)
    secs = time.perf_counter() - t0
    ntiles = sum(len(tr.lists[i]) for i in sample)
    f, b = tile_flops(cfg.D, ntiles)
    return secs, f + b + 6 * 2.0 * T * T * cfg.D, len(sample)


def cpu_baseline_gated(cfg, host, gate, seconds: float = 15.0):
    s0, _, _ = oracle_gated_sample(cfg, host, gate, head=0, frac=0.02)
    frac = min(1.0, max(0.02, 0.02 * seconds / max(s0, 1e-3)))
    secs, flops, n = oracle_gated_sample(cfg, host, gate, head=0, frac=frac, seed=1)
    T = (cfg.lat[0] + 3) // 4 * ((cfg.lat[1] + 3) // 4) * ((cfg.lat[2] + 3) // 4)
    cores = cpu_cores()
    return {"value": round(flops / secs / 1e12, 6), "unit": UNIT, "cores": cores["used"], "host_cpus": cores["host"],
            "kind": "oracle",
            "sample": f"head 0 of {cfg.name}: full fp64 router and coarse branch, gated forward and backward of "
                      f"{n} of {T} query cubes ({secs:.1f} s)"}


def cpu_cores():
    """Threads the oracle's BLAS uses, and the host's logical CPUs (nproc)."""
    used = None
    try:
        from threadpoolctl import threadpool_info
        used = max((i.get("num_threads", 1) for i in threadpool_info()), default=None)
    except Exception:
        pass
    host = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    return {"used": int(used or host), "host": int(host)}


def cpu_baseline(cfg, host, gpu, ntiles_total: int, seconds: float = 15.0):
    """The fp64 oracle on the host cores, on a bounded sample of the timed workload: the full
    router of the heads ``gpu["heads"]`` (two near-uniform, two sink heads) and the forward and
    backward of one fixed sample of query cubes on each.  Returns (baseline, parity):

    * baseline: the measured seconds, and the whole step (all heads, every selected tile)
      extrapolated linearly (router time per head x heads, attention time per tile x tiles);
      ``value`` is the step's FLOPs over that extrapolated time.
    * parity: the last timed step's lists, outputs and gradients on the same heads against the
      oracle: tie rows (the tie band of ``oracle.parity``), mismatching rows, and max/mean abs
      errors of out and dQ on the sampled query cubes and of dK, dV on a few key cubes (over
      every query cube that selects them).  Cubes touched by a row whose lists differ are left
      out of the error figures."""
    import numpy as np

    import oracle as O
    heads = gpu["heads"]
    lay = O.cube_layout(cfg.lat)
    T = lay.n_cubes
    per_head = {h: {n: O.tile(host[n][0, h].double().numpy(), lay) for n in ("q", "k", "v", "do")} for h in heads}
    # size the query-cube sample from a 1% calibration run on the first head (not counted)
    t = per_head[heads[0]]
    tr0 = O.route_head(t["q"], t["k"], lay.valid, cfg.top_k, cfg.top_p)
    cal = np.arange(0, T, 100)
    c0 = time.perf_counter()
    O.attention_forward_head(t["q"], t["k"], t["v"], tr0.lists, lay.valid, q_blocks=cal)
    O.attention_backward_head(t["q"], t["k"], t["v"], t["do"], tr0.lists, lay.valid, q_blocks=cal,
                              kv_blocks=range(T), visit=cal)
    per_cube = (time.perf_counter() - c0) / len(cal)
    n_sample = int(min(T, max(4, seconds / len(heads) / max(per_cube, 1e-4))))
    rng = np.random.default_rng(1)
    sample = np.sort(rng.choice(T, size=n_sample, replace=False))
    router_s, attn_s, tiles = 0.0, 0.0, 0
    rows = eq = ties = mism = 0
    err = {n: [0.0, 0.0, 0] for n in ("out", "dq", "dk", "dv")}    # max, sum, count
    for hi, h in enumerate(heads):
        t = per_head[h]
        c0 = time.perf_counter()
        tr = O.route_head(t["q"], t["k"], lay.valid, cfg.top_k, cfg.top_p)
        c1 = time.perf_counter()
        o_ref, _ = O.attention_forward_head(t["q"], t["k"], t["v"], tr.lists, lay.valid, q_blocks=sample)
        dq_ref, _, _ = O.attention_backward_head(t["q"], t["k"], t["v"], t["do"], tr.lists, lay.valid,
                                                 q_blocks=sample, kv_blocks=range(T), visit=sample)
        c2 = time.perf_counter()
        router_s += c1 - c0
        attn_s += c2 - c1
        tiles += sum(len(tr.lists[i]) for i in sample)
        # ---- parity of the GPU's last timed step on this head
        ci, cc = gpu["idx"][hi].numpy(), gpu["cnt"][hi].numpy()
        got = [ci[i, :cc[i]].astype(np.int64) for i in range(T)]
        m, tie, _ = O.parity.classify_router_rows(tr, got, cfg.top_p)
        same = np.array([len(a) == len(b) and np.array_equal(a, b) for a, b in zip(tr.lists, got)])
        rows += T
        eq += int(same.sum())
        ties += tie
        mism += m

        def acc(name, got_rows, ref_rows):
            if got_rows.size == 0:
                return
            e = np.abs(got_rows.astype(np.float64) - ref_rows)
            err[name][0] = max(err[name][0], float(e.max()))
            err[name][1] += float(e.sum())
            err[name][2] += e.size
        qc = [i for i in sample if same[i]]
        rws = np.concatenate([np.arange(i * 64, i * 64 + 64) for i in qc]) if qc else np.zeros(0, np.int64)
        acc("out", gpu["out"][hi].numpy()[rws], o_ref[rws])
        acc("dq", gpu["dq"][hi].numpy()[rws], dq_ref[rws])
        # dK, dV of a few key cubes whose selecting query cubes all have equal lists
        sel_by = [[] for _ in range(T)]
        for i, l in enumerate(tr.lists):
            for j in l:
                sel_by[int(j)].append(i)
        kc = [j for j in rng.choice(T, size=min(T, 16), replace=False) if all(same[i] for i in sel_by[j])][:4]
        if kc:
            _, dk_ref, dv_ref = O.attention_backward_head(t["q"], t["k"], t["v"], t["do"], tr.lists, lay.valid,
                                                          q_blocks=[], kv_blocks=kc)
            kr = np.concatenate([np.arange(j * 64, j * 64 + 64) for j in kc])
            acc("dk", gpu["dk"][hi].numpy()[kr], dk_ref[kr])
            acc("dv", gpu["dv"][hi].numpy()[kr], dv_ref[kr])
    H = cfg.B * cfg.H
    est_s = router_s / len(heads) * H + attn_s / max(tiles, 1) * ntiles_total
    fwd, bwd = tile_flops(cfg.D, ntiles_total)
    cores = cpu_cores()
    sample_txt = (f"heads {heads} of {cfg.name}: full fp64 router of each, forward and backward of the same "
                  f"{n_sample} of {T} query cubes on each ({tiles} tiles); measured {router_s:.1f} s router + "
                  f"{attn_s:.1f} s attention; the whole step ({H} heads, {ntiles_total} tiles) extrapolated "
                  f"linearly to {est_s:.0f} s")
    baseline = {"value": round((fwd + bwd) / est_s / 1e12, 6), "unit": UNIT, "cores": cores["used"],
                "host_cpus": cores["host"], "kind": "oracle", "sample": sample_txt,
                "measured_s": {"router": round(router_s, 2), "attention": round(attn_s, 2)},
                "sampled_tflops": round(tile_flops(cfg.D, tiles)[0] * 3.5 / attn_s / 1e12, 6),
                "extrapolated_step_s": round(est_s, 1), "extrapolated": True}
    parity = {"heads": heads, "rows": rows, "equal_rows": eq, "tie_rows": ties, "mismatch_rows": mism,
              "tie_band": O.parity.TIE_REL,
              "max_abs": {n: round(v[0], 6) for n, v in err.items() if v[2]},
              "mean_abs": {n: round(v[1] / v[2], 7) for n, v in err.items() if v[2]},
              "bounds": {"max_abs": 2e-2, "mean_abs": 2e-3},
              "sample": f"last timed step; out and dq on {n_sample} query cubes per head, dk and dv on up to 4 "
                        f"key cubes per head (over every query cube selecting them)"}
    return baseline, parity


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle as it stands, on the host cores.  Step s runs the
    full router of one head (cycling over the two near-uniform and two sink heads the oracle
    leg uses) and the forward and backward of a fixed-size sample of its query cubes."""
    import synth
    cfg = synth.get_config(args.config)
    heads = oracle_heads(cfg.H)
    host = synth.make_inputs(cfg, seed=0, heads=heads)
    # make_inputs(heads=...) returns only those heads, in that order
    # sample size: the whole run (warm-up + timed) should take about two minutes
    s0, _, _ = oracle_sample(cfg, host, head=0, frac=0.02)
    per_step = 120.0 / max(1, args.steps + args.warmup)
    frac = min(1.0, max(0.005, 0.02 * per_step / max(s0, 1e-3)))
    for w in range(args.warmup):
        oracle_sample(cfg, host, w % len(heads), frac, seed=100 + w)
    tot_s, tot_f, n = 0.0, 0.0, 0
    for s in range(args.steps):
        secs, fl, n = oracle_sample(cfg, host, s % len(heads), frac, seed=s)
        tot_s += secs
        tot_f += fl
    value = tot_f / tot_s / 1e12
    cores = cpu_cores()
    sample = (f"per step: one of heads {heads} of {cfg.name} in turn, full fp64 router + forward and backward "
              f"of {n} query cubes")
    return {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": f"Wan2.1-14B-720p-shaped attention ({args.config}), fp64 CPU oracle sample",
                       "sample": sample},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores["used"],
                             "host_cpus": cores["host"], "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="720p")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--e2e-chunk", type=int, default=2,
                    help="(batch, head) problems per chunk of the end-to-end step (sa_step_host)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the e4m3 Q/K forward section")
    ap.add_argument("--no-gated", action="store_true", help="skip the gated (coarse + fine) layer section")
    ap.add_argument("--extras", action="store_true",
                    help="also time the 128-token query-block router and the recall diagnostic")
    ap.add_argument("--sweep", action="store_true",
                    help="config-4 sweep (k=4, p x sparsity grid): one JSON line per point with load balance")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--one-pass", action="store_true",
                    help="one untimed pass of every hot kernel at --config (router, forward with the fp32 copy, "
                         "backward, fine router, coarse branch and gated layer) and exit: the command the "
                         "kernel profiles are captured on")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.sweep:
        if rank == 0:
            run_sweep(args)
        return
    if args.one_pass:
        if rank == 0:
            run_one_pass(args)
        return
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, rank, world)), flush=True)
        return
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    try:
        res = run_ours(args, rank, world, dist)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
