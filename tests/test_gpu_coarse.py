"""Coarse branch and gated combination on the GPU against the fp64 oracle.

The router half of sa_plan_coarse must equal sa_plan bit for bit (same kernels); the
cube-level tensors are fp32 arithmetic on exactly pooled inputs and are held to 1e-4; the
gated output and every gradient to the attention bounds (max abs 2e-2, mean abs 2e-3).
Padding slots of the output and of dG must be exactly 0.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_cubes_b200 as sa
import oracle as O
import synth
from parity import assert_close, classify_router_rows, gpu_inputs, gpu_lists, lists_to_device, oracle_head

pytestmark = pytest.mark.gpu

CUBE_ATOL = 1e-4

SMALL = {
    # B = 2 with an odd head count (rows indexed by b * H + h), D = 64, every cube axis ragged
    "b2h3_d64": ("b2h3", 2, 3, 64, (6, 9, 10), 3, 0.9),
    # T = 90 cubes: the cube-level products span two 64-wide tiles with a ragged tail
    "t90_d128": ("t90", 1, 2, 128, (12, 19, 23), 4, 0.8),
}


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    from block_sparse_attention_cubes_b200 import build
    build.build()
    yield


def _check_coarse(co, x, lay, b, h, tag):
    q, k, v = (oracle_head(x, n, b, h, lay) for n in ("q", "k", "v"))
    ref = O.coarse_forward_head(q, k, v, lay.valid)
    for name, got, r in zip(("qbar", "kbar", "vbar", "oc", "lse"),
                            (co.qbar, co.kbar, co.vbar, co.oc, co.lse), ref[:5]):
        err = float(np.max(np.abs(got[b, h].cpu().numpy().astype(np.float64) - r)))
        assert err <= CUBE_ATOL, f"{tag} {name}: max abs {err:.3g}"
    return ref


def _lists_equal(idx_a, cnt_a, idx_b, cnt_b):
    assert torch.equal(cnt_a, cnt_b)
    cap = idx_a.shape[-1]
    keep = torch.arange(cap, device=idx_a.device)[None, None, None, :] < cnt_a[..., None]
    assert torch.equal(torch.where(keep, idx_a, 0), torch.where(keep, idx_b, 0))


@pytest.mark.parametrize("case", sorted(SMALL))
def test_plan_coarse_lists_and_cube_tensors(case):
    cfg = synth.small_config(*SMALL[case])
    x, p, t = gpu_inputs(cfg)
    lay = O.cube_layout(cfg.lat)
    idx, cnt, co = sa.plan_coarse(t["q"], t["k"], t["v"], p)
    idx2, cnt2 = sa.plan(t["q"], t["k"], p)
    torch.cuda.synchronize()
    _lists_equal(idx, cnt, idx2, cnt2)
    for b in range(cfg.B):
        for h in range(cfg.H):
            tr = O.route_head(oracle_head(x, "q", b, h, lay), oracle_head(x, "k", b, h, lay), lay.valid,
                              cfg.top_k, cfg.top_p)
            mis, _, bad = classify_router_rows(tr, gpu_lists(idx, cnt, b, h), cfg.top_p)
            assert mis == 0, f"b{b} h{h}: rows {bad[:5]}"
            _check_coarse(co, x, lay, b, h, f"b{b}h{h}")


@pytest.mark.parametrize("case", sorted(SMALL))
def test_gated_forward_backward(case):
    cfg = synth.small_config(*SMALL[case])
    x, p, t = gpu_inputs(cfg)
    gate = synth.make_gate(cfg).cuda()
    lay = O.cube_layout(cfg.lat)
    T = lay.n_cubes
    _, _, co = sa.plan_coarse(t["q"], t["k"], t["v"], p)
    # the oracle's own lists (no boundary ties can separate the two sides)
    lists = {}
    for b in range(cfg.B):
        for h in range(cfg.H):
            lists[(b, h)] = O.route_head(oracle_head(x, "q", b, h, lay), oracle_head(x, "k", b, h, lay), lay.valid,
                                         cfg.top_k, cfg.top_p).lists
    idx, cnt = lists_to_device(lists, cfg.B, cfg.H, T, p.kv_capacity)
    out, lse, out32 = sa.forward_gated(t["q"], t["k"], t["v"], idx, cnt, p, co, gate)
    dq, dk, dv, dg = sa.backward_gated(t["q"], t["k"], t["v"], out, lse, t["do"], gate, idx, cnt, p, co,
                                       out_f32=out32)
    torch.cuda.synchronize()
    pad = ~lay.valid
    for b in range(cfg.B):
        for h in range(cfg.H):
            q, k, v, do = (oracle_head(x, n, b, h, lay) for n in ("q", "k", "v", "do"))
            g = gate[b, h].cpu().numpy().astype(np.float64)
            o_ref, _, lse_ref, _ = O.gated_forward_head(q, k, v, g, lists[(b, h)], lay.valid)
            tag = f"b{b}h{h}"
            o = out[b, h].float().cpu().numpy()
            assert_close(f"out {tag}", o[lay.valid], o_ref[lay.valid])
            assert np.all(o[pad] == 0), tag
            assert_close(f"out_f32 {tag}", out32[b, h].cpu().numpy()[lay.valid], o_ref[lay.valid])
            # the bf16 output is the rounding of the fp32 one
            assert torch.equal(out[b, h], out32[b, h].to(torch.bfloat16))
            assert np.max(np.abs(lse[b, h].cpu().numpy()[lay.valid] - lse_ref[lay.valid])) < 1e-3
            grads = O.gated_backward_head(q, k, v, do, g, lists[(b, h)], lay.valid)
            for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), grads[:3]):
                gg = got[b, h].cpu().numpy()
                assert_close(f"{name} {tag}", gg, ref)
                assert np.all(gg[pad] == 0), (name, tag)
            dgt = dg[b, h].cpu().numpy()
            assert_close(f"dgate {tag}", dgt, grads[3])
            assert np.all(dgt[pad] == 0), tag


def test_zero_gate_reproduces_the_fine_stage():
    """G = 0 (VSA's zero-initialised coarse gate): the gated output is the fine output bit
    for bit; the gradients equal sa_backward's up to the order of Delta's sum.  dS enters
    the tensor-core products as one fp16 value (11 significant bits) when every operand fits
    fp16, as here, else as a bf16 hi + lo pair (about 16 bits); both calls take the same path.
    A last-bit change in Delta can flip the rounding of dS, moving a gradient by about 2^-11
    of its magnitude: the bound is 2^-9 of the largest gradient (measured 4.3e-4 on O(1)
    gradients)."""
    cfg = synth.small_config(*SMALL["b2h3_d64"])
    x, p, t = gpu_inputs(cfg)
    idx, cnt, co = sa.plan_coarse(t["q"], t["k"], t["v"], p)
    zero = torch.zeros((cfg.B, cfg.H, t["q"].shape[2]), dtype=torch.float32, device="cuda")
    out_g, lse_g, o32_g = sa.forward_gated(t["q"], t["k"], t["v"], idx, cnt, p, co, zero)
    out_f, lse_f, o32_f = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p, with_f32=True)
    torch.cuda.synchronize()
    assert torch.equal(out_g, out_f) and torch.equal(o32_g, o32_f) and torch.equal(lse_g, lse_f)
    gq, gk, gv, gg = sa.backward_gated(t["q"], t["k"], t["v"], out_g, lse_g, t["do"], zero, idx, cnt, p, co,
                                       out_f32=o32_g)
    fq, fk, fv = sa.backward(t["q"], t["k"], t["v"], out_f, lse_f, t["do"], idx, cnt, p, out_f32=o32_f)
    torch.cuda.synchronize()
    for a, b in ((gq, fq), (gk, fk), (gv, fv)):
        assert float((a - b).abs().max()) <= 2.0 ** -9 * max(1.0, float(b.abs().max()))
    # dG = <dO, Oc^> still flows with G = 0
    lay = O.cube_layout(cfg.lat)
    q, k, v, do = (oracle_head(x, n, 1, 2, lay) for n in ("q", "k", "v", "do"))
    oc = O.coarse_forward_head(q, k, v, lay.valid)[3]
    assert_close("dgate", gg[1, 2].cpu().numpy(), (do * O.repeat_cubes(oc, lay.valid)).sum(axis=1))


def test_720p_gated_sampled():
    """The 720p shape (40 heads, T = 1440) in the launch configuration the bench times: lists
    equal to sa_plan's, cube-level tensors of two heads in full, gated output, dq and dG on
    sampled query cubes and dk, dv on sampled key cubes (the oracle on the GPU's own lists)."""
    cfg = synth.get_config("720p")
    x = synth.make_inputs(cfg, 0)
    gate = synth.make_gate(cfg).cuda()
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    t = {n: sa.tile(x[n].cuda(), p) for n in x}
    ws = {op: sa.new_workspace(p, op) for op in (sa.OP_PLAN_COARSE, sa.OP_FORWARD, sa.OP_BACKWARD_GATED)}
    idx, cnt, co = sa.plan_coarse(t["q"], t["k"], t["v"], p, ws=ws[sa.OP_PLAN_COARSE])
    out, lse, out32 = sa.forward_gated(t["q"], t["k"], t["v"], idx, cnt, p, co, gate, ws=ws[sa.OP_FORWARD])
    dq, dk, dv, dg = sa.backward_gated(t["q"], t["k"], t["v"], out, lse, t["do"], gate, idx, cnt, p, co,
                                       ws=ws[sa.OP_BACKWARD_GATED], out_f32=out32)
    torch.cuda.synchronize()
    for w in ws.values():
        assert sa.device_status(w) == 0
    idx2, cnt2 = sa.plan(t["q"], t["k"], p)
    _lists_equal(idx, cnt, idx2, cnt2)
    lay = O.cube_layout(cfg.lat)
    T = lay.n_cubes
    for h in (0, 23):
        _check_coarse(co, x, lay, 0, h, f"h{h}")
        q, k, v, do = (oracle_head(x, n, 0, h, lay) for n in ("q", "k", "v", "do"))
        lists = gpu_lists(idx, cnt, 0, h)
        rng = np.random.default_rng(h)
        qb = np.sort(rng.choice(T, 6, replace=False))
        qb[0] = T - 1                                  # a cube with padding
        kb = np.sort(rng.choice(T, 3, replace=False))
        g = gate[0, h].cpu().numpy().astype(np.float64)
        o_ref, _, _, _ = O.gated_forward_head(q, k, v, g, lists, lay.valid, q_blocks=qb)
        grads = O.gated_backward_head(q, k, v, do, g, lists, lay.valid, q_blocks=qb, kv_blocks=kb)
        rows = np.concatenate([np.arange(i * 64, (i + 1) * 64) for i in qb])
        rows = rows[lay.valid[rows]]
        cols = np.concatenate([np.arange(j * 64, (j + 1) * 64) for j in kb])
        cols = cols[lay.valid[cols]]
        assert_close(f"out h{h}", out32[0, h].cpu().numpy()[rows], o_ref[rows])
        assert_close(f"dq h{h}", dq[0, h].cpu().numpy()[rows], grads[0][rows])
        assert_close(f"dk h{h}", dk[0, h].cpu().numpy()[cols], grads[1][cols])
        assert_close(f"dv h{h}", dv[0, h].cpu().numpy()[cols], grads[2][cols])
        assert_close(f"dgate h{h}", dg[0, h].cpu().numpy(), grads[3])
