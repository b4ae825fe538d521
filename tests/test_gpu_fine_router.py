"""VSA2's fine-grained router with per-sequence Top-K on the GPU (sa_plan_fine) against the
oracle (oracle/vsa2_router.py), through the C ABI.

P_r is compared entry by entry: the scores are exact limb products, the softmax runs on fp32
exponentials, so P_r is held to 5e-6 absolute plus 5e-5 relative.  The selection is taken from
that fp32 P_r; it must equal the oracle's except at ties: every entry of the symmetric
difference must have an oracle P_r within 1e-5 relative of the oracle's boundary value (the
budget-th largest entry).  Ties are counted.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_cubes_b200 as sa
import oracle as O
import synth
from oracle import vsa2_router as V
from parity import gpu_inputs, gpu_lists, oracle_head

pytestmark = pytest.mark.gpu

PR_ATOL, PR_RTOL, TIE_REL = 5e-6, 5e-5, 1e-5


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    from block_sparse_attention_cubes_b200 import build
    build.build()
    yield


CASES = [(synth.small_config("fr", 1, 2, 128, (8, 8, 12), 4, 0.9), (2, 2, 2)),
         (synth.small_config("frrag", 2, 1, 128, (5, 9, 13), 3, 0.9), (2, 2, 2)),
         (synth.get_config("tiny"), (4, 2, 2)),
         (synth.small_config("fr16", 1, 2, 64, (8, 8, 8), 2, 0.9), (2, 2, 1))]


def _selection(lists, T):
    return {(i, int(j)) for i in range(T) for j in lists[i]}


@pytest.mark.parametrize("cfg,R", CASES, ids=[c[0].name + "-" + "".join(map(str, c[1])) for c in CASES])
def test_fine_router_matches_oracle(cfg, R):
    x, p, t = gpu_inputs(cfg, names=("q", "k"))
    idx, cnt, pr = sa.plan_fine(t["q"], t["k"], p, R=R, with_scores=True)
    torch.cuda.synchronize()
    lay = O.cube_layout(cfg.lat)
    T = lay.n_cubes
    ties = 0
    for b in range(cfg.B):
        for h in range(cfg.H):
            q, k = oracle_head(x, "q", b, h, lay), oracle_head(x, "k", b, h, lay)
            ref, _ = V.fine_grained_scores(q, k, lay.valid, R)
            got = pr[b, h].cpu().numpy().astype(np.float64)
            err = np.abs(got - ref)
            assert np.all(err <= PR_ATOL + PR_RTOL * ref), (b, h, float(err.max()))
            ref_lists = V.per_sequence_topk(ref, cfg.top_k)
            budget = min(cfg.top_k * T, T * T)
            assert int(cnt[b, h].sum()) == budget
            sg, sr = _selection(gpu_lists(idx, cnt, b, h), T), _selection(ref_lists, T)
            bval = np.sort(ref.reshape(-1))[::-1][budget - 1]
            diff = sg ^ sr
            assert all(abs(ref[i, j] - bval) <= TIE_REL * bval for i, j in diff), sorted(diff)[:5]
            ties += len(diff) > 0
            for i in range(T):  # ascending ids in each row
                row = gpu_lists(idx, cnt, b, h)[i]
                assert np.all(np.diff(row) > 0)
    assert ties <= max(1, cfg.B * cfg.H // 2)


def test_fine_router_budget_edges():
    cfg = synth.small_config("fredge", 1, 2, 128, (8, 8, 8), 0, 0.9)   # T = 8
    x, p, t = gpu_inputs(cfg, names=("q", "k"))
    idx, cnt = sa.plan_fine(t["q"], t["k"], p, R=(2, 2, 2))          # K = 0: nothing kept
    torch.cuda.synchronize()
    assert int(cnt.sum()) == 0
    p2 = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, 100, 0.9)     # K * T >= T^2: every block
    idx, cnt = sa.plan_fine(t["q"], t["k"], p2, R=(2, 2, 2))
    torch.cuda.synchronize()
    assert torch.all(cnt == 8)
    assert torch.equal(idx, torch.arange(8, dtype=torch.int32, device="cuda").expand_as(idx))
    with pytest.raises(sa.SAError):
        sa.plan_fine(t["q"], t["k"], p, R=(1, 1, 1))                 # G = 64: not built
