"""Choose the input recipe's locality amplitude per head type so that the fp64 oracle
router reaches each workload's target block density (TEST INFRASTRUCTURE: it runs the
oracle and writes ``synth/calibration.json``, which the input generator reads).

    python -m oracle.calibrate [config ...]

For each configuration with a sparsity target and each head type ("uniform", "sink"),
alpha is found by bisection on seed 0 so that the mean density of that type's heads
(kept blocks / T^2, every row, the oracle's hybrid Top-k U Top-p) is within 0.25
percentage points of the target.  Density falls as alpha grows (sharper block scores).
"""
import json
import math
import os
import sys
from concurrent.futures import ProcessPoolExecutor
import multiprocessing as mp

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from oracle import attention as O  # noqa: E402

OUT = os.path.join(ROOT, "synth", "calibration.json")

def _head_density(args):
    cfg_name, h, alpha, top_k, top_p = args
    cfg = synth.get_config(cfg_name)
    comp = {n: synth.components(cfg, 0, n, 0, h) for n in ("q", "k")}
    ht = cfg.head_types[h]
    ht = synth.HeadType(ht.name, alpha, ht.kscale, ht.sink)
    lay = O.cube_layout(cfg.lat)
    q = O.tile(synth.combine("q", *comp["q"], ht).double().numpy(), lay)
    k = O.tile(synth.combine("k", *comp["k"], ht).double().numpy(), lay)
    tr = O.route_head(q, k, lay.valid, top_k, top_p)
    return sum(len(l) for l in tr.lists) / lay.n_cubes ** 2


def density(pool, cfg, heads, alpha):
    return float(np.mean(list(pool.map(_head_density, [(cfg.name, h, alpha, cfg.top_k, cfg.top_p) for h in heads]))))


def calibrate(pool, cfg_name, tol=0.0025):
    cfg = synth.get_config(cfg_name)
    target = cfg.target_density
    result = {}
    for typ in ("uniform", "sink"):
        heads = [h for h, ht in enumerate(cfg.head_types) if ht.name == typ]
        lo, hi = 0.0, 4.0
        d_hi = density(pool, cfg, heads, hi)
        while d_hi > target and hi < 64:
            lo, hi = hi, hi * 2
            d_hi = density(pool, cfg, heads, hi)
        best = (hi, d_hi)
        for _ in range(30):
            mid = 0.5 * (lo + hi)
            d = density(pool, cfg, heads, mid)
            if abs(d - target) < abs(best[1] - target):
                best = (mid, d)
            if abs(d - target) <= tol * 0.5:
                break
            if d > target:
                lo = mid
            else:
                hi = mid
        result[typ] = round(best[0], 6)
        result[f"{typ}_density"] = round(best[1], 6)
        print(cfg_name, typ, result[typ], result[f"{typ}_density"], flush=True)
    result["target"] = target
    return result


def main(names):
    table = json.load(open(OUT)) if os.path.exists(OUT) else {}
    ctx = mp.get_context("spawn")
    with ProcessPoolExecutor(max_workers=min(6, os.cpu_count() or 1), mp_context=ctx) as pool:
        for name in names:
            key = name if not name.startswith("sweep") else "sweep_" + name.split("_")[2]
            table[key] = calibrate(pool, name)
            with open(OUT, "w") as f:
                json.dump(table, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main(sys.argv[1:] or ["720p", "480p", "720p_fp8", "sweep_0.9_80", "sweep_0.9_85", "sweep_0.9_90",
                          "sweep_0.9_95", "sweep_0.9_98"])
