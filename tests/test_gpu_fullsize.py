"""Parity at the benchmark sizes, in the launch configuration bench.py times.

Router: every row of every head against the fp64 oracle (tie rows counted).
Fine stage: sampled query cubes (out, lse, dq) and key cubes (dk, dv), each computed by
the oracle on its own, using the GPU's own index lists.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_cubes_b200 as sa
import oracle as O
import synth
from parity import assert_close, classify_router_rows, gpu_lists

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    from block_sparse_attention_cubes_b200 import build
    build.build()
    yield


def _full(name, sample_heads, nq=12, nkv=6):
    cfg = synth.get_config(name)
    x = synth.make_inputs(cfg, 0)
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    dev = torch.device("cuda")
    t = {n: sa.tile(x[n].to(dev), p) for n in x}
    A = sa.Attention(p)
    idx, cnt = A.plan(t["q"], t["k"])
    out, lse, out32 = A.forward(t["q"], t["k"], t["v"], idx, cnt)
    dq, dk, dv = A.backward(t["q"], t["k"], t["v"], out, lse, t["do"], idx, cnt, out_f32=out32)
    torch.cuda.synchronize()
    for op in (sa.OP_PLAN, sa.OP_FORWARD, sa.OP_BACKWARD):
        assert sa.device_status(A._ws[op]) == 0
    lay = O.cube_layout(cfg.lat)
    T = lay.n_cubes
    ties = 0
    dens = []
    for h in range(cfg.H):
        q = O.tile(x["q"][0, h].double().numpy(), lay)
        k = O.tile(x["k"][0, h].double().numpy(), lay)
        tr = O.route_head(q, k, lay.valid, cfg.top_k, cfg.top_p)
        lists = gpu_lists(idx, cnt, 0, h)
        mis, tie, bad = classify_router_rows(tr, lists, cfg.top_p)
        assert mis == 0, f"head {h}: rows {bad[:5]}"
        ties += tie
        dens.append(sum(len(l) for l in lists) / T / T)
        if h not in sample_heads:
            continue
        rng = np.random.default_rng(h)
        qb = np.sort(rng.choice(T, nq, replace=False))
        qb[0] = T - 1                      # the last cube holds padding (ragged tail)
        kb = np.sort(rng.choice(T, nkv, replace=False))
        v = O.tile(x["v"][0, h].double().numpy(), lay)
        do = O.tile(x["do"][0, h].double().numpy(), lay)
        o_ref, lse_ref = O.attention_forward_head(q, k, v, lists, lay.valid, q_blocks=qb)
        g = O.attention_backward_head(q, k, v, do, lists, lay.valid, q_blocks=qb, kv_blocks=kb)
        rows = np.concatenate([np.arange(i * 64, (i + 1) * 64) for i in qb])
        rows = rows[lay.valid[rows]]
        cols = np.concatenate([np.arange(j * 64, (j + 1) * 64) for j in kb])
        cols = cols[lay.valid[cols]]
        assert_close(f"out h{h}", out[0, h].float().cpu().numpy()[rows], o_ref[rows])
        assert np.max(np.abs(lse[0, h].cpu().numpy()[rows] - lse_ref[rows])) < 1e-3
        assert_close(f"dq h{h}", dq[0, h].cpu().numpy()[rows], g[0][rows])
        assert_close(f"dk h{h}", dk[0, h].cpu().numpy()[cols], g[1][cols])
        assert_close(f"dv h{h}", dv[0, h].cpu().numpy()[cols], g[2][cols])
    assert ties <= max(2, 1e-3 * cfg.H * T)
    return float(np.mean(dens))


def test_480p_full_router_sampled_attention():
    _full("480p", sample_heads=(0, 6))


def test_720p_full_router_sampled_attention():
    _full("720p", sample_heads=(0, 20), nq=8, nkv=4)


def test_720p_fp8_full_router_sampled_forward():
    """The e4m3 Q/K configuration: Q and K quantised per cube from the same bf16 draws;
    router and forward against the oracle on the dequantised values (V stays bf16)."""
    cfg = synth.get_config("720p_fp8")
    x = synth.make_inputs(cfg, 0, names=("q", "k", "v"))
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p, qk_dtype=sa.FP8_E4M3)
    pb = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    dev = torch.device("cuda")
    t = {n: sa.tile(x[n].to(dev), pb) for n in x}
    q8, qs = synth.quantize_e4m3_rows(t["q"])
    k8, ks = synth.quantize_e4m3_rows(t["k"])
    A = sa.Attention(p)
    idx, cnt = A.plan(q8, k8, qs, ks)
    out, lse, _ = A.forward(q8, k8, t["v"], idx, cnt, qs, ks, with_f32=False)
    torch.cuda.synchronize()
    for op in (sa.OP_PLAN, sa.OP_FORWARD):
        assert sa.device_status(A._ws[op]) == 0
    lay = O.cube_layout(cfg.lat)
    T = lay.n_cubes
    q8n, k8n, qsn, ksn = (a.cpu().numpy() for a in (q8, k8, qs, ks))
    ties = 0
    for h in range(cfg.H):
        q = O.dequantize_rows(q8n[0, h], qsn[0, h])
        k = O.dequantize_rows(k8n[0, h], ksn[0, h])
        tr = O.route_head(q, k, lay.valid, cfg.top_k, cfg.top_p)
        lists = gpu_lists(idx, cnt, 0, h)
        mis, tie, bad = classify_router_rows(tr, lists, cfg.top_p)
        assert mis == 0, f"head {h}: rows {bad[:5]}"
        ties += tie
        if h not in (0, 20):
            continue
        rng = np.random.default_rng(h)
        qb = np.sort(rng.choice(T, 8, replace=False))
        qb[0] = T - 1
        v = O.tile(x["v"][0, h].double().numpy(), lay)
        o_ref, lse_ref = O.attention_forward_head(q, k, v, lists, lay.valid, q_blocks=qb)
        rows = np.concatenate([np.arange(i * 64, (i + 1) * 64) for i in qb])
        rows = rows[lay.valid[rows]]
        assert_close(f"out h{h}", out[0, h].float().cpu().numpy()[rows], o_ref[rows])
        assert np.max(np.abs(lse[0, h].cpu().numpy()[rows] - lse_ref[rows])) < 1e-3
    assert ties <= max(2, 1e-3 * cfg.H * T)


def test_sweep_densest_full_router_sampled_attention():
    """Config-4 sweep point with the longest lists (k = 4, p = 0.8 at the amplitude
    calibrated for 80% sparsity): ragged unions of up to min(2 cap, T) entries."""
    _full("sweep_0.8_80", sample_heads=(0, 20), nq=6, nkv=3)


def test_t4096_ragged_router_and_sampled_attention():
    """T = 4096 cubes (latent 63 x 62 x 61: every axis ragged), D = 64, one head: every router
    row against the oracle, and forward / backward of sampled cubes (among them the last,
    partial cube) with the GPU's lists."""
    cfg = synth.small_config("t4096", 1, 1, 64, (63, 62, 61), 8, 0.5)
    x = synth.make_inputs(cfg, 0)
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    npad, T = sa.geometry(p)
    assert T == 4096
    dev = torch.device("cuda")
    t = {n: sa.tile(x[n].to(dev), p) for n in x}
    A = sa.Attention(p)
    idx, cnt = A.plan(t["q"], t["k"])
    out, lse, out32 = A.forward(t["q"], t["k"], t["v"], idx, cnt)
    dq, dk, dv = A.backward(t["q"], t["k"], t["v"], out, lse, t["do"], idx, cnt, out_f32=out32)
    torch.cuda.synchronize()
    for op in (sa.OP_PLAN, sa.OP_FORWARD, sa.OP_BACKWARD):
        assert sa.device_status(A._ws[op]) == 0
    lay = O.cube_layout(cfg.lat)
    q, k, v, do = (O.tile(x[n][0, 0].double().numpy(), lay) for n in ("q", "k", "v", "do"))
    tr = O.route_head(q, k, lay.valid, cfg.top_k, cfg.top_p)
    lists = gpu_lists(idx, cnt, 0, 0)
    mis, ties, bad = classify_router_rows(tr, lists, cfg.top_p)
    assert mis == 0, f"rows {bad[:5]}"
    assert ties <= max(2, 1e-3 * T)
    rng = np.random.default_rng(7)
    qb = np.sort(rng.choice(T, 6, replace=False))
    qb[-1] = T - 1
    kb = np.sort(rng.choice(T, 4, replace=False))
    kb[-1] = T - 1
    o_ref, lse_ref = O.attention_forward_head(q, k, v, lists, lay.valid, q_blocks=qb)
    g = O.attention_backward_head(q, k, v, do, lists, lay.valid, q_blocks=qb, kv_blocks=kb)
    rows = np.concatenate([np.arange(i * 64, (i + 1) * 64) for i in qb])
    rows = rows[lay.valid[rows]]
    cols = np.concatenate([np.arange(j * 64, (j + 1) * 64) for j in kb])
    cols = cols[lay.valid[cols]]
    assert_close("out", out[0, 0].float().cpu().numpy()[rows], o_ref[rows])
    assert np.max(np.abs(lse[0, 0].cpu().numpy()[rows] - lse_ref[rows])) < 1e-3
    assert_close("dq", dq[0, 0].cpu().numpy()[rows], g[0][rows])
    assert_close("dk", dk[0, 0].cpu().numpy()[cols], g[1][cols])
    assert_close("dv", dv[0, 0].cpu().numpy()[cols], g[2][cols])
