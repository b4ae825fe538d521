"""Benchmark: one step = router + fine-stage forward + backward (sa_plan, sa_forward,
sa_backward) at the Wan2.1-14B-720p attention shape, 95% block sparsity.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 720p]

Prints ONE JSON line on rank 0.  ``value`` is effective TFLOP/s over the whole step
(all ranks' work / max-over-ranks device time), counting only the selected 64x64 tiles:
forward 4*D*64*64 and backward 10*D*64*64 FLOPs per selected tile (VSA page, FLOP
accounting: 4 * D * S * H * d * 3.5, i.e. forward 1 + backward 2.5).  Each rank runs an
independent problem of the same shape (weak scaling, no collective on the data path).
Inputs are larger than L2 and L2 is also flushed between steps (256 MiB write).
Extra sections on the same line: ``fp8_forward`` (e4m3 Q/K configuration, 720p only) and
``gated`` (the coarse branch + gate layer: sa_plan_coarse, sa_forward_gated,
sa_backward_gated), skipped with ``--no-fp8`` / ``--no-gated``.
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
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join(ROOT, "gpurun_out" if os.path.isdir(os.path.join(ROOT, "gpurun_out")) else "",
                                 f".clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={CLOCK_QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        # wait for the first sample, so nvidia-smi's start-up (NVML initialisation) is over
        # before the timed region begins
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < 5.0:
            self.f.flush()
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.05)
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
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

    for _ in range(args.warmup):
        idx, cnt, *_ = step()
    torch.cuda.synchronize()
    for op in (sa.OP_PLAN, sa.OP_FORWARD, sa.OP_BACKWARD):
        st = sa.device_status(A._ws[op])
        if st != 0:
            raise RuntimeError(f"device status {sa.STATUS_NAMES.get(st, st)} after warm-up")
    ntiles = int(cnt.sum().item())
    density = ntiles / (cfg.B * cfg.H * T * T)
    fwd_fl, bwd_fl = tile_flops(cfg.D, ntiles)

    recs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    launches["n"] = 0
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for s in range(args.steps):
            flush.fill_(s & 0xff)     # evict L2 between steps (not timed)
            step(recs[s])
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    plan_ms = [r[0].elapsed_time(r[1]) for r in recs]
    fwd_ms = [r[1].elapsed_time(r[2]) for r in recs]
    bwd_ms = [r[2].elapsed_time(r[3]) for r in recs]
    step_ms = [a + b + c for a, b, c in zip(plan_ms, fwd_ms, bwd_ms)]
    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    ms_per_step = total_ms / args.steps
    step_flops = (fwd_fl + bwd_fl) * world
    value = step_flops / (ms_per_step * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    fwd_avg = statistics.mean(fwd_ms)
    bwd_avg = statistics.mean(bwd_ms)
    plan_avg = statistics.mean(plan_ms)
    # dominant kernel: the forward kernel, timed with events around sa_forward on the launching
    # (current) stream inside the timed region; the call's two other launches (cube mask, query
    # pair union) are about 0.3% of its time, so this slightly understates the kernel's own rate
    fwd_tf = fwd_fl / (fwd_avg * 1e-3) / 1e12
    peak_tf = peaks.get("bf16_tflops_sustained") or peaks.get("bf16_tflops")
    roofline = {"kernel": "attn_fwd_kernel", "bound": "tensor", "achieved": round(fwd_tf, 2),
                "peak": peak_tf, "unit": "TFLOP/s", "frac": round(fwd_tf / peak_tf, 4),
                "traffic": traffic_for("attn_fwd_kernel", ntiles),
                "peak_source": f"{peak_src} bf16 dense, sustained",
                "algorithmic_flops_per_launch": fwd_fl}
    router_bytes = 2 * cfg.B * cfg.H * npad * cfg.D * 2 + 4 * (ntiles + cfg.B * cfg.H * T)
    router_gbs = router_bytes / (plan_avg * 1e-3) / 1e9

    result = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"Wan2.1-shaped attention ({args.config}): B={cfg.B}, H={cfg.H}, D={cfg.D}, latent "
                               f"{'x'.join(map(str, cfg.lat))} -> T={T} cubes of 64, Npad={npad}; top_k={cfg.top_k}, "
                               f"top_p={cfg.top_p}; step = sa_plan + sa_forward + sa_backward",
                   "B": cfg.B, "H": cfg.H, "D": cfg.D, "lat": list(cfg.lat), "T": T, "top_k": cfg.top_k,
                   "top_p": cfg.top_p, "density": round(density, 5), "selected_tiles": ntiles,
                   "l2": "inputs larger than L2; 256 MiB flush between steps",
                   "per_rank": "independent problem per rank (seed = rank)"},
        "breakdown_ms": {"plan": round(plan_avg, 4), "forward": round(fwd_avg, 4), "backward": round(bwd_avg, 4),
                         "fwd_plus_bwd": round(fwd_avg + bwd_avg, 4)},
        "per_step_ms": {"plan": [round(v, 3) for v in plan_ms], "forward": [round(v, 3) for v in fwd_ms],
                        "backward": [round(v, 3) for v in bwd_ms]},
        "fwd_bwd_tflops": round((fwd_fl + bwd_fl) / ((fwd_avg + bwd_avg) * 1e-3) / 1e12, 3),
        "router": {"achieved_gbs": round(router_gbs, 1), "peak_gbs": peaks.get("hbm_gbs"),
                   "frac": round(router_gbs / peaks.get("hbm_gbs"), 4), "algorithmic_bytes": router_bytes},
        "roofline": roofline,
        "gpu_launches": launches["n"],
        "clocks": clocks.summary(),
        "gen_s": round(t_gen, 1),
    }
    if args.e2e_steps > 0:
        result["e2e"] = run_e2e(args, sa, A, p, host, dev, fwd_fl + bwd_fl, world, dist)
    run_fp8 = args.config == "720p" and not args.no_fp8
    if run_fp8 or not args.no_gated:
        del x, A
    if run_fp8:
        result["fp8_forward"] = run_fp8_forward(args, sa, synth, rank, dev, flush, peak_tf, peaks.get("hbm_gbs"), dist)
    if not args.no_gated:
        result["gated"] = run_gated(args, sa, synth, cfg, host, rank, dev, flush, result["breakdown_ms"], dist)
    if args.extras:
        result["extras"] = run_extras(args, sa, cfg, host, dev, flush, dist)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, host, seconds=args.cpu_seconds)
    return result


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
    plan_ms = statistics.mean(r[0].elapsed_time(r[1]) for r in recs)
    fwd_ms = statistics.mean(r[1].elapsed_time(r[2]) for r in recs)
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
    ms = [statistics.mean(v) for v in per_step]
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
    ms = [statistics.mean(r[i].elapsed_time(r[i + 1]) for r in recs) for i in range(3)]
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
    return {"config": f"{cfg.name}: sa_plan_bq128 + fine stage on its lists; recall of sa_plan's lists",
            "steps": steps, "bq128": bq, "recall": rec}


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
    (at p = 0.9) for 80..98% sparsity.  One JSON line per point: step timings and the per-CTA
    load balance of the persistent attention kernels."""
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
            ms = [statistics.mean(r[k].elapsed_time(r[k + 1]) for r in recs) for k in range(3)]
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
                    "balance": cta_balance(masks, sms)}
            print(json.dumps(line), flush=True)
            del x, A


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
FWD_ABI_FUNCTIONS = ("bool make_map(", "sa::AttnArgs base_args(", "sa_status sa_forward(")


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
    """Same step through the public API with host buffers: pinned latent-order inputs are
    copied in, tiled, routed, run forward and backward, and out/dq/dk/dv are untiled and
    copied back, all inside the timed region."""
    import torch
    pinned = {n: host[n].pin_memory() for n in ("q", "k", "v", "do")}
    L = p.lat_t * p.lat_h * p.lat_w
    outs = {"out": torch.empty((p.B, p.H, L, p.D), dtype=torch.bfloat16).pin_memory()}
    for n in ("dq", "dk", "dv"):
        outs[n] = torch.empty((p.B, p.H, L, p.D), dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pinned.values())
    d2h = sum(t.numel() * t.element_size() for t in outs.values())

    def e2e_step():
        d = {n: t.to(dev, non_blocking=True) for n, t in pinned.items()}
        x = {n: sa.tile(d[n], p) for n in d}
        idx, cnt = A.plan(x["q"], x["k"])
        out, lse, out32 = A.forward(x["q"], x["k"], x["v"], idx, cnt)
        dq, dk, dv = A.backward(x["q"], x["k"], x["v"], out, lse, x["do"], idx, cnt, out_f32=out32)
        for n, t in (("out", out), ("dq", dq), ("dk", dk), ("dv", dv)):
            outs[n].copy_(sa.untile(t, p), non_blocking=True)

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
    return {"value": round(flops * world / (ms * 1e-3) / 1e12, 3), "unit": UNIT, "ms_per_step": round(ms, 3),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


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
    return {"value": round(flops / secs / 1e12, 6), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"head 0 of {cfg.name}: full fp64 router and coarse branch, gated forward and backward of "
                      f"{n} of {T} query cubes ({secs:.1f} s)"}


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((i.get("num_threads", 1) for i in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(cfg, host, seconds: float = 15.0):
    # calibrate the sample size on a small piece, then run ~`seconds` of oracle work
    s0, _, n0 = oracle_sample(cfg, host, head=0, frac=0.02)
    frac = min(1.0, max(0.02, 0.02 * seconds / max(s0, 1e-3)))
    secs, flops, n = oracle_sample(cfg, host, head=0, frac=frac, seed=1)
    return {"value": round(flops / secs / 1e12, 6), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"head 0 of {cfg.name}: full fp64 router + forward and backward of {n} of "
                      f"{(cfg.lat[0]+3)//4*((cfg.lat[1]+3)//4)*((cfg.lat[2]+3)//4)} query cubes ({secs:.1f} s)"}


def run_reference(args, rank, world):
    import synth
    cfg = synth.get_config(args.config)
    host = synth.make_inputs(cfg, seed=0, heads=[0])
    # sample size: the whole run (warm-up + timed) should take about two minutes
    s0, _, _ = oracle_sample(cfg, host, head=0, frac=0.02)
    per_step = 120.0 / max(1, args.steps + args.warmup)
    frac = min(1.0, max(0.005, 0.02 * per_step / max(s0, 1e-3)))
    for w in range(args.warmup):
        oracle_sample(cfg, host, 0, frac, seed=100 + w)
    tot_s, tot_f, n = 0.0, 0.0, 0
    for s in range(args.steps):
        secs, fl, n = oracle_sample(cfg, host, 0, frac, seed=s)
        tot_s += secs
        tot_f += fl
    value = tot_f / tot_s / 1e12
    cores = cpu_cores()
    sample = f"per step: head 0 of {cfg.name}, full fp64 router + forward and backward of {n} query cubes"
    return {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": f"Wan2.1-14B-720p-shaped attention ({args.config}), fp64 CPU oracle sample",
                       "sample": sample},
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="720p")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the e4m3 Q/K forward section")
    ap.add_argument("--no-gated", action="store_true", help="skip the gated (coarse + fine) layer section")
    ap.add_argument("--extras", action="store_true",
                    help="also time the 128-token query-block router and the recall diagnostic")
    ap.add_argument("--sweep", action="store_true",
                    help="config-4 sweep (k=4, p x sparsity grid): one JSON line per point with load balance")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.sweep:
        if rank == 0:
            run_sweep(args)
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
