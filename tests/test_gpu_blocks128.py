"""Router with 128-token query blocks on the GPU against the fp64 oracle, and the fine stage
on its lists (both cubes of a pair share one list).

Lists are compared per query block with the cube router's tie rule (rows that differ only
within the 1e-6 score band at the k / p boundary are counted, not failed); outputs and
gradients to the attention bounds.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_cubes_b200 as sa
import oracle as O
import synth
from oracle import blocks128 as Bq
from parity import assert_close, classify_router_rows, gpu_inputs, gpu_lists, oracle_head

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    from block_sparse_attention_cubes_b200 import build
    build.build()
    yield


@pytest.mark.parametrize("name,B,H,D,lat,k,pp", [
    ("b2h3", 2, 3, 64, (6, 9, 10), 3, 0.9),        # T = 18, every axis ragged, B = 2 with odd H
    ("t90", 1, 2, 128, (12, 19, 21), 4, 0.8),      # T = 90: score tiles with a ragged tail
    ("t12", 1, 2, 64, (5, 8, 12), 2, 0.6),         # T = 12, ragged in t
    ("t15", 1, 2, 128, (4, 12, 20), 3, 0.7),       # T = 15: the last block is one cube
])
def test_plan_bq128_and_attention(name, B, H, D, lat, k, pp):
    cfg = synth.small_config(name, B, H, D, lat, k, pp)
    x, p, t = gpu_inputs(cfg)
    lay = O.cube_layout(cfg.lat)
    T = lay.n_cubes
    M = (T + 1) // 2
    idx, cnt = sa.plan_bq128(t["q"], t["k"], p)
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(H):
            q, kk = oracle_head(x, "q", b, h, lay), oracle_head(x, "k", b, h, lay)
            lists_blk, pbar = Bq.route_head_bq128(q, kk, lay.valid, cfg.top_k, cfg.top_p)
            got = gpu_lists(idx, cnt, b, h)
            for c in range(T):                       # both cubes of a block carry its list
                assert np.array_equal(got[c], got[2 * (c // 2)])
            got_blk = [got[2 * i] for i in range(M)]
            # the cube router's tie classification, on the block rows
            tr = O.RouterTrace(pbar=pbar, lists=lists_blk, n_k=np.full(M, min(cfg.top_k, T)),
                               n_p=np.array([O.topp_count(r, cfg.top_p) for r in pbar]), qbar=None, kbar=None)
            mis, _, bad = classify_router_rows(tr, got_blk, cfg.top_p)
            assert mis == 0, f"b{b} h{h}: block rows {bad[:5]}"
    # the fine stage on the GPU's lists, forward and backward
    out, lse, out32 = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p, with_f32=True)
    dq, dk, dv = sa.backward(t["q"], t["k"], t["v"], out, lse, t["do"], idx, cnt, p, out_f32=out32)
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(H):
            q, kk, v, do = (oracle_head(x, n, b, h, lay) for n in ("q", "k", "v", "do"))
            lists = gpu_lists(idx, cnt, b, h)
            o_ref, _ = O.attention_forward_head(q, kk, v, lists, lay.valid)
            assert_close(f"out b{b}h{h}", out[b, h].float().cpu().numpy()[lay.valid], o_ref[lay.valid])
            g = O.attention_backward_head(q, kk, v, do, lists, lay.valid)
            for n, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), g):
                assert_close(f"{n} b{b}h{h}", got[b, h].cpu().numpy(), ref)
