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
from oracle import vsa2_router as V
from parity import gpu_inputs, lists_to_device, oracle_head

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
    # the oracle router's lists feed both sides (the router itself is checked elsewhere)
    lists = {(b, h): O.route_head(oracle_head(x, "q", b, h, lay), oracle_head(x, "k", b, h, lay), lay.valid,
                                  cfg.top_k, cfg.top_p).lists for b in range(cfg.B) for h in range(cfg.H)}
    idx, cnt = lists_to_device(lists, cfg.B, cfg.H, T, p.kv_capacity)
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
            ref = Bq.selected_mass(q, k, lists[(b, h)], lay.valid)
            got = tau[b, h].cpu().numpy()
            assert np.max(np.abs(got - ref)) <= TAU_ATOL, (b, h)
            assert np.all(got[pad] == 0)
            ref_cube, best = Bq.cube_recall(q, k, lists[(b, h)], lay.valid)
            assert np.max(np.abs(cube[b, h].cpu().numpy() - ref_cube)) <= TAU_ATOL
            assert np.all(best >= ref_cube - 1e-12)
    # every block kept: all of the mass, exactly
    assert torch.all(tau_all[:, :, torch.from_numpy(lay.valid).cuda()] == 1.0)
    assert torch.all(cube_all == 1.0)


# P_oracle entries come from bf16 products with fp32 accumulation and ex2.approx exponentials
# of (s * scale - lse), with lse from the forward kernel (held to 1e-3 by the forward tests, but
# far closer in practice): held here to 2e-5 absolute plus 2e-4 relative.
PB_ATOL, PB_RTOL = 2e-5, 2e-4


@pytest.mark.parametrize("cfg", [synth.small_config("pbr", 1, 2, 64, (5, 8, 12), 2, 0.6),
                                 synth.small_config("pbr128", 2, 1, 128, (7, 9, 10), 3, 0.8),
                                 synth.get_config("tiny")], ids=["ragged-d64", "ragged-d128-B2", "tiny"])
def test_block_mass_and_best_recall(cfg):
    x, p, t = gpu_inputs(cfg, names=("q", "k", "v"))
    lay = O.cube_layout(cfg.lat)
    T = lay.n_cubes
    every = torch.arange(T, dtype=torch.int32, device="cuda").expand(cfg.B, cfg.H, T, T).contiguous()
    full = torch.full((cfg.B, cfg.H, T), T, dtype=torch.int32, device="cuda")
    _, lse_all = sa.forward(t["q"], t["k"], t["v"], every, full, p)
    pb = sa.block_mass(t["q"], t["k"], lse_all, p)
    lists = {(b, h): O.route_head(oracle_head(x, "q", b, h, lay), oracle_head(x, "k", b, h, lay), lay.valid,
                                  cfg.top_k, cfg.top_p).lists for b in range(cfg.B) for h in range(cfg.H)}
    cnt = torch.tensor([[[len(l) for l in lists[(b, h)]] for h in range(cfg.H)] for b in range(cfg.B)],
                       dtype=torch.int32, device="cuda")
    best = sa.best_recall(pb, cnt, p)
    torch.cuda.synchronize()
    for b in range(cfg.B):
        for h in range(cfg.H):
            q, k = oracle_head(x, "q", b, h, lay), oracle_head(x, "k", b, h, lay)
            ref = V.oracle_block_scores(q, k, lay.valid)
            got = pb[b, h].cpu().numpy().astype(np.float64)
            assert np.all(np.abs(got - ref) <= PB_ATOL + PB_RTOL * np.abs(ref)), (b, h, float(np.abs(got - ref).max()))
            assert np.allclose(got.sum(axis=1), 1.0, atol=1e-4)
            _, ref_best = Bq.cube_recall(q, k, lists[(b, h)], lay.valid)
            assert np.max(np.abs(best[b, h].cpu().numpy() - ref_best)) <= 1e-4, (b, h)
    # n = T keeps the whole row; n = 0 keeps nothing
    assert torch.allclose(sa.best_recall(pb, full, p), torch.ones_like(best), atol=1e-4)
    assert torch.all(sa.best_recall(pb, torch.zeros_like(full), p) == 0)
