"""Router recall on the GPU against the oracle (tau of the SpargeAttention2 page's equation 8).

tau = exp(lse_kept - lse_all) from two forward calls; each lse is held to 1e-3 of the oracle's
by the forward tests, so tau (at most 1) is held to exp(2e-3) - 1 < 2.1e-3.
"""
import numpy as np
import pytest
import torch

import block_sparse_attention_cubes_b200 as sa
import oracle as O
import synth
from oracle import blocks128 as Bq
from parity import gpu_inputs, gpu_lists, oracle_head

pytestmark = pytest.mark.gpu

TAU_ATOL = 2.1e-3


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    from block_sparse_attention_cubes_b200 import build
    build.build()
    yield


@pytest.mark.parametrize("D", [64, 128])
def test_recall_matches_oracle(D):
    cfg = synth.small_config("recall", 2, 3, D, (5, 8, 12), 2, 0.6)     # T = 12, ragged in t
    x, p, t = gpu_inputs(cfg, names=("q", "k", "v"))
    lay = O.cube_layout(cfg.lat)
    T = lay.n_cubes
    idx, cnt = sa.plan(t["q"], t["k"], p)
    _, lse_kept = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p)
    every = torch.arange(T, dtype=torch.int32, device="cuda").expand(cfg.B, cfg.H, T, T).contiguous()
    full = torch.full((cfg.B, cfg.H, T), T, dtype=torch.int32, device="cuda")
    _, lse_all = sa.forward(t["q"], t["k"], t["v"], every, full, p)
    tau, cube = sa.recall(lse_kept, lse_all, p)
    tau_all, cube_all = sa.recall(lse_all, lse_all, p)
    torch.cuda.synchronize()
    pad = ~lay.valid
    for b in range(cfg.B):
        for h in range(cfg.H):
            q, k = oracle_head(x, "q", b, h, lay), oracle_head(x, "k", b, h, lay)
            lists = gpu_lists(idx, cnt, b, h)
            ref = Bq.selected_mass(q, k, lists, lay.valid)
            got = tau[b, h].cpu().numpy()
            assert np.max(np.abs(got - ref)) <= TAU_ATOL, (b, h)
            assert np.all(got[pad] == 0)
            ref_cube, best = Bq.cube_recall(q, k, lists, lay.valid)
            assert np.max(np.abs(cube[b, h].cpu().numpy() - ref_cube)) <= TAU_ATOL
            assert np.all(best >= ref_cube - 1e-12)
    # every block kept: all of the mass, exactly
    assert torch.all(tau_all[:, :, torch.from_numpy(lay.valid).cuda()] == 1.0)
    assert torch.all(cube_all == 1.0)
