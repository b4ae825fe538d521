"""CUDA path vs the fp64 oracle on the same seeded inputs, through the C ABI.

Index lists must match bit for bit except tie rows (counted); outputs and gradients
must be within max-abs 2e-2 and mean-abs 2e-3.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_cubes_b200 as sa
import oracle as O
import synth
from parity import (assert_close, classify_router_rows, gpu_inputs, gpu_lists, lists_to_device, oracle_head)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    from block_sparse_attention_cubes_b200 import build
    build.build()
    yield


def _check_layout(cfg, x, tiled):
    lay = O.cube_layout(cfg.lat)
    for n, t in tiled.items():
        ref = O.tile(x[n][0].float().numpy(), lay)
        assert np.array_equal(t[0].float().cpu().numpy(), ref), n
        back = sa.untile(t, sa.make_params(cfg.B, t.shape[1], cfg.D, cfg.lat, 1, 0.5))
        assert torch.equal(back.cpu(), x[n]), n


def _router_case(cfg, heads=None, allow_tie_frac=1e-3, names=("q", "k")):
    x, p, t = gpu_inputs(cfg, names=names, heads=heads)
    idx, cnt = sa.plan(t["q"], t["k"], p)
    torch.cuda.synchronize()
    lay = O.cube_layout(cfg.lat)
    tot_mis, tot_ties, rows = 0, 0, 0
    for hh in range(p.H):
        tr = O.route_head(oracle_head(x, "q", 0, hh, lay), oracle_head(x, "k", 0, hh, lay), lay.valid,
                          cfg.top_k, cfg.top_p)
        mis, ties, bad = classify_router_rows(tr, gpu_lists(idx, cnt, 0, hh), cfg.top_p)
        assert mis == 0, f"head {hh}: {mis} mismatching rows, e.g. {bad[:5]}"
        tot_ties += ties
        rows += lay.n_cubes
    assert tot_ties <= max(2, allow_tie_frac * rows)
    return x, p, t, idx, cnt


def test_tile_matches_oracle_layout():
    cfg = synth.small_config("pad", 1, 2, 64, (5, 6, 7), 2, 0.5)
    x, p, t = gpu_inputs(cfg, names=("q", "v"))
    _check_layout(cfg, x, t)


@pytest.mark.parametrize("name", ["tiny"])
def test_router_tiny(name):
    _router_case(synth.get_config(name))


@pytest.mark.parametrize("lat,k,pp", [((4, 4, 4), 1, 0.9), ((5, 8, 12), 3, 0.9), ((8, 8, 8), 0, 0.0),
                                      ((8, 12, 16), 2, 0.5), ((9, 9, 9), 50, 0.3), ((8, 8, 8), 4, 1.0)])
def test_router_small_edge(lat, k, pp):
    _router_case(synth.small_config("e", 1, 2, 128, lat, k, pp))


def _fwd_case(cfg, lists_src="oracle", heads=None, q_blocks=None):
    x, p, t = gpu_inputs(cfg, heads=heads)
    lay = O.cube_layout(cfg.lat)
    H = p.H
    trs = {}
    for hh in range(H):
        trs[(0, hh)] = O.route_head(oracle_head(x, "q", 0, hh, lay), oracle_head(x, "k", 0, hh, lay), lay.valid,
                                    cfg.top_k, cfg.top_p).lists
    idx, cnt = lists_to_device(trs, 1, H, lay.n_cubes, p.kv_capacity)
    out, lse, out32 = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p, with_f32=True)
    out_inf, lse_inf = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p)      # inference path: single bf16 P
    torch.cuda.synchronize()
    assert torch.equal(out32.to(torch.bfloat16), out)
    assert torch.equal(lse_inf, lse)
    for hh in range(H):
        q, k, v = (oracle_head(x, n, 0, hh, lay) for n in ("q", "k", "v"))
        o_ref, lse_ref = O.attention_forward_head(q, k, v, trs[(0, hh)], lay.valid, q_blocks=q_blocks)
        rows = lay.valid.copy()
        if q_blocks is not None:
            m = np.zeros_like(rows)
            for i in q_blocks:
                m[i * 64:(i + 1) * 64] = True
            rows &= m
        got = out[0, hh].float().cpu().numpy()
        assert_close(f"out h{hh}", got[rows], o_ref[rows])
        assert_close(f"out (bf16 P) h{hh}", out_inf[0, hh].float().cpu().numpy()[rows], o_ref[rows])
        assert np.all(got[~lay.valid] == 0)
        gl = lse[0, hh].cpu().numpy()
        assert np.max(np.abs(gl[rows] - lse_ref[rows])) < 1e-3
        assert np.all(gl[~lay.valid] == 0)
    return x, p, t, idx, cnt, out, lse, out32, trs


def test_forward_tiny():
    _fwd_case(synth.get_config("tiny"))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("lat,k,pp", [((4, 4, 4), 1, 0.9), ((5, 8, 12), 3, 0.9), ((8, 12, 16), 2, 0.5),
                                      ((9, 9, 9), 50, 0.3), ((8, 8, 8), 8, 1.0)])
def test_forward_small(D, lat, k, pp):
    _fwd_case(synth.small_config("f", 1, 2, D, lat, k, pp))


def _bwd_case(cfg):
    x, p, t, idx, cnt, out, lse, out32, trs = _fwd_case(cfg)
    dq, dk, dv = sa.backward(t["q"], t["k"], t["v"], out, lse, t["do"], idx, cnt, p, out_f32=out32)
    torch.cuda.synchronize()
    lay = O.cube_layout(cfg.lat)
    for hh in range(p.H):
        q, k, v, do = (oracle_head(x, n, 0, hh, lay) for n in ("q", "k", "v", "do"))
        g = O.attention_backward_head(q, k, v, do, trs[(0, hh)], lay.valid)
        for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), g):
            a = got[0, hh].cpu().numpy()
            assert_close(f"{name} h{hh}", a, ref)
            assert np.all(a[~lay.valid] == 0)


def test_backward_tiny():
    _bwd_case(synth.get_config("tiny"))


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("lat,k,pp", [((4, 4, 4), 1, 0.9), ((5, 8, 12), 3, 0.9), ((8, 12, 16), 2, 0.5),
                                      ((9, 9, 9), 50, 0.3)])
def test_backward_small(D, lat, k, pp):
    _bwd_case(synth.small_config("b", 1, 2, D, lat, k, pp))


@pytest.mark.parametrize("D", [64, 128])
def test_fp16_and_bf16_operand_paths(D):
    """The backward multiplies P and dS as single fp16 values when Q, K, V and dO all fit fp16
    and the bound |dS| <= 2 D max|dO| max|V| stays within 2^15, else as bf16 hi + lo pairs (the
    forward with the fp32 output likewise takes P in fp16 when V fits); the choice is made on
    the device for each call.  (a) dO scaled by 2^12 (exact in bf16, still inside fp16) breaks
    the dS bound: the gradients, scaled back, must still match the oracle.  (b) one padding
    slot of V set to 2^17 (outside fp16; padding keys never take part) forces the bf16 path in
    both forward and backward with results inside the same bounds."""
    cfg = synth.small_config("bp", 1, 2, D, (5, 8, 12), 3, 0.9)
    x, p, t, idx, cnt, out, lse, out32, trs = _fwd_case(cfg)
    lay = O.cube_layout(cfg.lat)
    refs = {hh: O.attention_backward_head(*(oracle_head(x, n, 0, hh, lay) for n in ("q", "k", "v", "do")),
                                          trs[(0, hh)], lay.valid) for hh in range(p.H)}
    s = 2.0 ** 12
    assert float(t["do"].abs().max()) * s < 65504.0
    ga = sa.backward(t["q"], t["k"], t["v"], out, lse, t["do"] * s, idx, cnt, p, out_f32=out32)
    pad = int(np.flatnonzero(~lay.valid)[0])
    v_pad = t["v"].clone()
    v_pad[0, :, pad, 0] = 2.0 ** 17
    out_b, lse_b, o32_b = sa.forward(t["q"], t["k"], v_pad, idx, cnt, p, with_f32=True)
    gb = sa.backward(t["q"], t["k"], v_pad, out_b, lse_b, t["do"], idx, cnt, p, out_f32=o32_b)
    torch.cuda.synchronize()
    for hh in range(p.H):
        o_ref, _ = O.attention_forward_head(*(oracle_head(x, n, 0, hh, lay) for n in ("q", "k", "v")),
                                            trs[(0, hh)], lay.valid)
        assert_close(f"out (V out of fp16 range) h{hh}", out_b[0, hh].float().cpu().numpy()[lay.valid],
                     o_ref[lay.valid])
        for name, g_a, g_b, ref in zip(("dq", "dk", "dv"), ga, gb, refs[hh]):
            assert_close(f"{name} (dO x 2^12) h{hh}", g_a[0, hh].cpu().numpy() / s, ref)
            b_ = g_b[0, hh].cpu().numpy()
            assert_close(f"{name} (V out of fp16 range) h{hh}", b_, ref)
            assert np.all(b_[~lay.valid] == 0)


def test_end_to_end_with_gpu_lists():
    cfg = synth.small_config("e2e", 1, 4, 128, (8, 16, 20), 4, 0.9)
    x, p, t, idx, cnt = _router_case(cfg, names=("q", "k", "v", "do"))
    out, lse, out32 = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p, with_f32=True)
    dq, dk, dv = sa.backward(t["q"], t["k"], t["v"], out, lse, t["do"], idx, cnt, p, out_f32=out32)
    torch.cuda.synchronize()
    lay = O.cube_layout(cfg.lat)
    for hh in range(p.H):
        lists = gpu_lists(idx, cnt, 0, hh)
        q, k, v, do = (oracle_head(x, n, 0, hh, lay) for n in ("q", "k", "v", "do"))
        o_ref, _ = O.attention_forward_head(q, k, v, lists, lay.valid)
        assert_close("out", out[0, hh].float().cpu().numpy(), o_ref)
        g = O.attention_backward_head(q, k, v, do, lists, lay.valid)
        for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), g):
            assert_close(name, got[0, hh].cpu().numpy(), ref)


def test_deterministic_repeat():
    cfg = synth.small_config("det", 1, 2, 128, (8, 12, 16), 3, 0.9)
    x, p, t = gpu_inputs(cfg)
    r1 = sa.plan(t["q"], t["k"], p)
    r2 = sa.plan(t["q"], t["k"], p)
    assert torch.equal(r1[1], r2[1])
    used = torch.arange(p.kv_capacity, device="cuda") < r1[1][..., None]   # entries past the count are unspecified
    assert torch.equal(r1[0][used], r2[0][used])
    o1 = sa.forward(t["q"], t["k"], t["v"], *r1, p, with_f32=True)
    o2 = sa.forward(t["q"], t["k"], t["v"], *r1, p, with_f32=True)
    assert all(torch.equal(a, b) for a, b in zip(o1, o2))
    g1 = sa.backward(t["q"], t["k"], t["v"], o1[0], o1[1], t["do"], *r1, p, out_f32=o1[2])
    g2 = sa.backward(t["q"], t["k"], t["v"], o1[0], o1[1], t["do"], *r1, p, out_f32=o1[2])
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)
    # without the fp32 copy Delta comes from the bf16 output: same as passing it upcast
    g3 = sa.backward(t["q"], t["k"], t["v"], o1[0], o1[1], t["do"], *r1, p)
    g4 = sa.backward(t["q"], t["k"], t["v"], o1[0], o1[1], t["do"], *r1, p, out_f32=o1[0].float())
    for a, b in zip(g3, g4):
        assert torch.equal(a, b)


def test_empty_lists_and_unselected_key_cubes():
    """Caller-supplied lists with runs of empty query-cube pairs and of key-cube pairs that
    no query selects: with 8 heads x 128 pairs every CTA walks several items per stream,
    empty ones among them.  Empty rows give out = 0, lse = -inf, dQ = 0 (the header's
    contract for a count of 0); all other rows match the oracle restricted to them."""
    cfg = synth.small_config("holes", 1, 8, 128, (16, 32, 32), 6, 0.9)
    x, p, t = gpu_inputs(cfg)
    lay = O.cube_layout(cfg.lat)
    T = lay.n_cubes
    drop_q = {i for i in range(T) if (i // 2) % 3 != 0}
    drop_k = {j for j in range(T) if (j // 2) % 3 == 1}
    trs = {}
    for hh in range(p.H):
        lists = O.route_head(oracle_head(x, "q", 0, hh, lay), oracle_head(x, "k", 0, hh, lay), lay.valid,
                             cfg.top_k, cfg.top_p).lists
        trs[(0, hh)] = [np.array([], np.int64) if i in drop_q else np.array([j for j in l if j not in drop_k],
                                                                            np.int64) for i, l in enumerate(lists)]
    idx, cnt = lists_to_device(trs, 1, p.H, T, p.kv_capacity)
    out, lse, out32 = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p, with_f32=True)
    dq, dk, dv = sa.backward(t["q"], t["k"], t["v"], out, lse, t["do"], idx, cnt, p, out_f32=out32)
    torch.cuda.synchronize()
    for hh in range(p.H):
        lists = trs[(0, hh)]
        live = [i for i in range(T) if len(lists[i]) > 0]
        assert 0 < len(live) < T
        empty_rows = np.zeros(lay.valid.shape, bool)
        for i in range(T):
            if len(lists[i]) == 0:
                empty_rows[i * 64:(i + 1) * 64] = True
        empty_rows &= lay.valid
        q, k, v, do = (oracle_head(x, n, 0, hh, lay) for n in ("q", "k", "v", "do"))
        o_ref, lse_ref = O.attention_forward_head(q, k, v, lists, lay.valid, q_blocks=live)
        rows = lay.valid & ~empty_rows
        got = out[0, hh].float().cpu().numpy()
        assert_close(f"out h{hh}", got[rows], o_ref[rows])
        assert np.all(got[empty_rows] == 0)
        gl = lse[0, hh].cpu().numpy()
        assert np.max(np.abs(gl[rows] - lse_ref[rows])) < 1e-3
        assert np.all(np.isneginf(gl[empty_rows]))
        g = O.attention_backward_head(q, k, v, do, lists, lay.valid, visit=live)
        for name, got_g, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), g):
            a = got_g[0, hh].cpu().numpy()
            assert_close(f"{name} h{hh}", a, ref)
        assert np.all(dq[0, hh].cpu().numpy()[empty_rows] == 0)
        unselected = sorted(set(range(T)) - {int(j) for l in lists for j in l})
        assert len(unselected) >= 4
        for j in unselected:
            assert np.all(dk[0, hh, j * 64:(j + 1) * 64].cpu().numpy() == 0)
            assert np.all(dv[0, hh, j * 64:(j + 1) * 64].cpu().numpy() == 0)


@pytest.mark.parametrize("lat,k,pp", [((4, 4, 4), 1, 0.9), ((5, 8, 12), 3, 0.9), ((9, 9, 9), 50, 0.3)])
def test_fp8_router_and_forward_small(lat, k, pp):
    """e4m3 Q/K with one scale per cube (quantised from the bf16 draws): router lists and
    forward against the oracle run on the dequantised Q and K."""
    cfg = synth.small_config("f8", 1, 2, 128, lat, k, pp)
    x, pb, t = gpu_inputs(cfg, names=("q", "k", "v"))
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p, qk_dtype=sa.FP8_E4M3)
    q8, qs = synth.quantize_e4m3_rows(t["q"])
    k8, ks = synth.quantize_e4m3_rows(t["k"])
    idx, cnt = sa.plan(q8, k8, p, qs, ks)
    out, lse = sa.forward(q8, k8, t["v"], idx, cnt, p, qs, ks)
    out_f, lse_f, out32 = sa.forward(q8, k8, t["v"], idx, cnt, p, qs, ks, with_f32=True)
    torch.cuda.synchronize()
    assert torch.equal(out32.to(torch.bfloat16), out_f)
    lay = O.cube_layout(cfg.lat)
    q8n, k8n, qsn, ksn = (a.cpu().numpy() for a in (q8, k8, qs, ks))
    for hh in range(p.H):
        q = O.dequantize_rows(q8n[0, hh], qsn[0, hh])
        kk = O.dequantize_rows(k8n[0, hh], ksn[0, hh])
        tr = O.route_head(q, kk, lay.valid, cfg.top_k, cfg.top_p)
        lists = gpu_lists(idx, cnt, 0, hh)
        mis, ties, bad = classify_router_rows(tr, lists, cfg.top_p)
        assert mis == 0, f"head {hh}: rows {bad[:5]}"
        v = oracle_head(x, "v", 0, hh, lay)
        o_ref, lse_ref = O.attention_forward_head(q, kk, v, lists, lay.valid)
        rows = lay.valid
        for name, o in (("out", out), ("out (split P)", out_f)):
            got = o[0, hh].float().cpu().numpy()
            assert_close(f"{name} h{hh}", got[rows], o_ref[rows])
            assert np.all(got[~rows] == 0)
        assert np.max(np.abs(lse[0, hh].cpu().numpy()[rows] - lse_ref[rows])) < 1e-3


def test_fp8_host_checks(cuda_ok):
    p = sa.make_params(1, 1, 64, (4, 4, 4), 1, 0.5, qk_dtype=sa.FP8_E4M3)   # e4m3 needs D = 128
    z8 = torch.zeros(1, 1, 64, 64, dtype=torch.uint8, device="cuda")
    zb = torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16, device="cuda")
    sc = torch.ones(1, 1, 1, device="cuda")
    idx = torch.zeros(1, 1, 1, 1, dtype=torch.int32, device="cuda")
    cnt = torch.ones(1, 1, 1, dtype=torch.int32, device="cuda")
    with pytest.raises(RuntimeError, match="UNSUPPORTED"):
        sa.forward(z8, z8, zb, idx, cnt, p, sc, sc)


@pytest.mark.parametrize("D", [64, 128])
def test_batch2_odd_heads_router_forward_backward(D):
    """B = 2 with an odd head count: router lists, forward and backward of every (b, h)
    against the oracle (the kernels index rows by b * H + h)."""
    cfg = synth.small_config("b2", 2, 3, D, (6, 9, 10), 3, 0.9)
    x, p, t = gpu_inputs(cfg)
    lay = O.cube_layout(cfg.lat)
    T = lay.n_cubes
    idx, cnt = sa.plan(t["q"], t["k"], p)
    trs = {}
    for b in range(cfg.B):
        for hh in range(cfg.H):
            tr = O.route_head(oracle_head(x, "q", b, hh, lay), oracle_head(x, "k", b, hh, lay), lay.valid,
                              cfg.top_k, cfg.top_p)
            mis, ties, bad = classify_router_rows(tr, gpu_lists(idx, cnt, b, hh), cfg.top_p)
            assert mis == 0, f"b{b} h{hh}: rows {bad[:5]}"
            trs[(b, hh)] = tr.lists
    idx_o, cnt_o = lists_to_device(trs, cfg.B, cfg.H, T, p.kv_capacity)
    out, lse, out32 = sa.forward(t["q"], t["k"], t["v"], idx_o, cnt_o, p, with_f32=True)
    dq, dk, dv = sa.backward(t["q"], t["k"], t["v"], out, lse, t["do"], idx_o, cnt_o, p, out_f32=out32)
    torch.cuda.synchronize()
    for b in range(cfg.B):
        for hh in range(cfg.H):
            q, k, v, do = (oracle_head(x, n, b, hh, lay) for n in ("q", "k", "v", "do"))
            o_ref, lse_ref = O.attention_forward_head(q, k, v, trs[(b, hh)], lay.valid)
            assert_close(f"out b{b}h{hh}", out[b, hh].float().cpu().numpy()[lay.valid], o_ref[lay.valid])
            assert np.max(np.abs(lse[b, hh].cpu().numpy()[lay.valid] - lse_ref[lay.valid])) < 1e-3
            g = O.attention_backward_head(q, k, v, do, trs[(b, hh)], lay.valid)
            for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), g):
                assert_close(f"{name} b{b}h{hh}", got[b, hh].cpu().numpy(), ref)
