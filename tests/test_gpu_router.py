"""The tensor-core router's two paths against the fp64 oracle (GPU, through the C ABI).

sa_plan decides each row from exact integer limb products turned into fixed-point keys, and
hands the rows whose decision lies within its error bounds to an fp64 path.  These tests force
every row through the fp64 path (SA_DEBUG_ROUTER_FALLBACK), check both paths against the oracle
and against each other, count the rows the normal path hands over, and run inputs whose pooled
values span very different magnitudes (the limbs follow each row's binary exponent) and a head
whose scores are all equal (every row a tie, decided by block id).
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_cubes_b200 as sa
import oracle as O
import synth
from parity import classify_router_rows, gpu_inputs, gpu_lists, oracle_head

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    from block_sparse_attention_cubes_b200 import build
    build.build()
    yield


def _oracle_traces(cfg, x, H):
    lay = O.cube_layout(cfg.lat)
    return lay, [O.route_head(oracle_head(x, "q", 0, h, lay), oracle_head(x, "k", 0, h, lay), lay.valid,
                              cfg.top_k, cfg.top_p) for h in range(H)]


def _plan(t, p, debug=0):
    q = sa.Params.from_buffer_copy(p)
    q.debug_flags = debug
    ws = sa.new_workspace(q, sa.OP_PLAN)
    idx, cnt = sa.plan(t["q"], t["k"], q, ws=ws)
    return idx, cnt, sa.plan_fallback_rows(ws)


CASES = [synth.get_config("tiny"), synth.small_config("rag", 1, 3, 128, (5, 9, 13), 3, 0.8),
         synth.small_config("d64", 2, 2, 64, (8, 12, 16), 2, 0.5), synth.small_config("k0p0", 1, 2, 128, (8, 8, 8), 0, 0.0)]


@pytest.mark.parametrize("cfg", CASES, ids=lambda c: c.name)
def test_fallback_path_matches_oracle_and_fast_path(cfg):
    x, p, t = gpu_inputs(cfg, names=("q", "k"))
    idx_f, cnt_f, nf = _plan(t, p)
    idx_s, cnt_s, ns = _plan(t, p, debug=sa.DEBUG_ROUTER_FALLBACK)
    torch.cuda.synchronize()
    rows = cfg.B * cfg.H * idx_f.shape[2]
    assert ns == rows                       # every row went through the fp64 path
    assert 0 <= nf <= rows
    lay, _ = _oracle_traces(cfg, x, 0)
    for b in range(cfg.B):
        for h in range(cfg.H):
            tr = O.route_head(oracle_head(x, "q", b, h, lay), oracle_head(x, "k", b, h, lay), lay.valid,
                              cfg.top_k, cfg.top_p)
            for idx, cnt in ((idx_f, cnt_f), (idx_s, cnt_s)):
                mis, _, bad = classify_router_rows(tr, gpu_lists(idx, cnt, b, h), cfg.top_p)
                assert mis == 0, (b, h, bad[:5])
    # the two paths agree wherever the fast path kept its decision (both are the fp64 decision)
    assert torch.equal(cnt_f, cnt_s)
    used = torch.arange(idx_f.shape[3], device=idx_f.device) < cnt_f[..., None]
    assert torch.equal(idx_f[used], idx_s[used])


def test_fallback_rows_are_rare_at_480p():
    cfg = synth.get_config("480p")
    x, p, t = gpu_inputs(cfg, names=("q", "k"))
    _, cnt, nf = _plan(t, p)
    rows = cnt.numel()
    assert nf <= 0.05 * rows, f"{nf} of {rows} rows needed the fp64 path"


@pytest.mark.parametrize("mag", [1e-3, 37.0])
def test_magnitudes_follow_row_exponents(mag):
    cfg = synth.small_config("mag", 1, 2, 128, (8, 12, 20), 4, 0.9)
    x = synth.make_inputs(cfg, 0, names=("q", "k"))
    # scale q and k of head 1 and the keys of head 0 (bf16 keeps the relative values)
    x["q"][:, 1] = (x["q"][:, 1].float() * mag).to(torch.bfloat16)
    x["k"] = (x["k"].float() * torch.tensor([mag, 1.0 / mag]).view(1, 2, 1, 1)).to(torch.bfloat16)
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    t = {n: sa.tile(x[n].cuda(), p) for n in ("q", "k")}
    idx, cnt, _ = _plan(t, p)
    torch.cuda.synchronize()
    lay, trs = _oracle_traces(cfg, x, cfg.H)
    for h in range(cfg.H):
        mis, _, bad = classify_router_rows(trs[h], gpu_lists(idx, cnt, 0, h), cfg.top_p)
        assert mis == 0, (h, bad[:5])


def test_equal_scores_everywhere():
    # q = 0 on head 0: every block score is 0, every row a tie broken by block id
    cfg = synth.small_config("flat", 1, 2, 128, (8, 8, 12), 3, 0.5)
    x = synth.make_inputs(cfg, 0, names=("q", "k"))
    x["q"][:, 0] = 0
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    t = {n: sa.tile(x[n].cuda(), p) for n in ("q", "k")}
    idx, cnt, nf = _plan(t, p)
    torch.cuda.synchronize()
    T = idx.shape[2]
    assert nf >= T                          # the flat head's rows all went to the fp64 path
    lay, trs = _oracle_traces(cfg, x, cfg.H)
    # uniform rows with p = 0.5: the smallest ids, ceil(T / 2) of them (one more is a tie at the
    # Top-p crossing, where p * Z equals a prefix sum)
    n = max(cfg.top_k, int(np.ceil(0.5 * T)))
    for i, lst in enumerate(gpu_lists(idx, cnt, 0, 0)):
        assert list(lst) == list(range(len(lst))) and len(lst) in (n, n + 1), (i, lst)
    for h in range(cfg.H):
        mis, _, bad = classify_router_rows(trs[h], gpu_lists(idx, cnt, 0, h), cfg.top_p)
        assert mis == 0, (h, bad[:5])
