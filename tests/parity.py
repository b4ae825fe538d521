"""Helpers shared by the GPU parity tests: run the CUDA path and the oracle on the same
seeded inputs and compare the results.  Test infrastructure only."""
import math

import numpy as np
import torch

import block_sparse_attention_cubes_b200 as sa
import oracle as O
import synth

ATOL_MAX = 2e-2    # max-abs error bound for bf16 inputs with fp32 accumulation
ATOL_MEAN = 2e-3   # mean-abs error bound
TIE_REL = O.parity.TIE_REL   # block-score tie band at the k / p boundary
classify_router_rows = O.parity.classify_router_rows


def gpu_inputs(cfg, seed=0, names=("q", "k", "v", "do"), heads=None):
    x = synth.make_inputs(cfg, seed, names=names, heads=heads)
    H = len(heads) if heads is not None else cfg.H
    p = sa.make_params(cfg.B, H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    dev = torch.device("cuda")
    tiled = {n: sa.tile(x[n].to(dev), p) for n in names}
    return x, p, tiled


def oracle_head(x, name, b, h, lay):
    return O.tile(x[name][b, h].double().numpy(), lay)


def gpu_lists(idx, cnt, b, h):
    idx = idx[b, h].cpu().numpy()
    cnt = cnt[b, h].cpu().numpy()
    return [idx[i, :cnt[i]].astype(np.int64) for i in range(len(cnt))]


def errs(got: np.ndarray, ref: np.ndarray):
    e = np.abs(got.astype(np.float64) - ref)
    return float(e.max()) if e.size else 0.0, float(e.mean()) if e.size else 0.0


def assert_close(name, got, ref, atol_max=ATOL_MAX, atol_mean=ATOL_MEAN):
    mx, mn = errs(got, ref)
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    assert mx <= atol_max and mn <= atol_mean, f"{name}: max abs {mx:.3g} (<= {atol_max}), mean abs {mn:.3g} (<= {atol_mean})"
    return mx, mn


def lists_to_device(lists_per_head, B, H, T, cap, dev="cuda"):
    """Oracle lists [(b,h) -> T arrays] -> kv_index [B,H,T,cap], kv_count [B,H,T] int32."""
    idx = np.full((B, H, T, cap), -7, np.int32)
    cnt = np.zeros((B, H, T), np.int32)
    for (b, h), lists in lists_per_head.items():
        for i, l in enumerate(lists):
            idx[b, h, i, :len(l)] = l
            cnt[b, h, i] = len(l)
    return torch.from_numpy(idx).to(dev), torch.from_numpy(cnt).to(dev)


def scale_of(D):
    return 1.0 / math.sqrt(D)
