"""Pins for the oracle's 128-token query blocks and the router recall diagnostic (CPU only).

Independent checks: queries duplicated across the two cubes of a block reproduce the
64-token router (pinned separately); pooled block means against plain token loops; the fine
stage against torch SDPA with a token-level mask built from the block lists; recall three
ways (equation 8's tau, exp(lse over the kept keys - lse over all keys), and the identity
with the cube-level P_oracle).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
from oracle import blocks128 as Bq


def _case(lat, D, seed):
    rng = np.random.default_rng(seed)
    lay = O.cube_layout(lat)
    q, k, v = (rng.standard_normal((lay.n_pad, D)) for _ in range(3))
    for x in (q, k, v):
        x[~lay.valid] = 0.0
    return lay, q, k, v


def test_pair_duplicated_queries_match_the_cube_router():
    lay, q, k, _ = _case((8, 8, 8), 8, 1)                 # T = 8 full cubes
    T = lay.n_cubes
    qd = q.reshape(T, 64, 8).copy()
    qd[1::2] = qd[0::2]                                   # cube 2i+1 carries cube 2i's tokens
    qd = qd.reshape(-1, 8)
    lists128, _ = Bq.route_head_bq128(qd, k, lay.valid, 2, 0.5)
    ref = O.route_head(qd, k, lay.valid, 2, 0.5).lists
    for i in range(T // 2):
        assert np.array_equal(lists128[i], ref[2 * i]) and np.array_equal(lists128[i], ref[2 * i + 1])


@pytest.mark.parametrize("lat", [(5, 6, 7), (4, 4, 12)])   # ragged cubes; T = 8, and T = 3 (odd)
def test_block_means_against_token_loops(lat):
    lay, q, _, _ = _case(lat, 4, 2)
    T = lay.n_cubes
    got = Bq.pool_query_pairs(q, lay.valid)
    assert got.shape == ((T + 1) // 2, 4)
    for i in range((T + 1) // 2):
        toks = [t for t in range(128 * i, min(128 * (i + 1), lay.n_pad)) if lay.valid[t]]
        np.testing.assert_allclose(got[i], np.mean([q[t] for t in toks], axis=0), rtol=1e-13)


@pytest.mark.parametrize("lat", [(5, 6, 7), (4, 4, 12)])
def test_fine_stage_with_block_lists_equals_token_masked_sdpa(lat):
    lay, q, k, v = _case(lat, 8, 3)
    T = lay.n_cubes
    lists128, pbar = Bq.route_head_bq128(q, k, lay.valid, 2, 0.6)
    assert pbar.shape == ((T + 1) // 2, T)
    o, _ = O.attention_forward_head(q, k, v, Bq.cube_lists(lists128, T), lay.valid)
    mask = np.zeros((lay.n_pad, lay.n_pad), bool)
    for t in range(lay.n_pad):
        for j in lists128[t // 128]:
            mask[t, j * 64:(j + 1) * 64] = True
    mask &= lay.valid[None, :]
    mask[~lay.valid] = True                               # padding rows: any finite row, compared nowhere
    tt = lambda a: torch.from_numpy(a)[None, None]
    ref = F.scaled_dot_product_attention(tt(q), tt(k), tt(v), attn_mask=torch.from_numpy(mask)[None, None],
                                         scale=1 / math.sqrt(8))[0, 0].numpy()
    np.testing.assert_allclose(o[lay.valid], ref[lay.valid], rtol=1e-12, atol=1e-12)


def test_recall_three_ways():
    lay, q, k, v = _case((5, 8, 8), 8, 4)                 # T = 8, the second t-layer of cubes partial
    T = lay.n_cubes
    lists = O.route_head(q, k, lay.valid, 2, 0.5).lists
    tau = Bq.selected_mass(q, k, lists, lay.valid)
    np.testing.assert_allclose(tau, Bq.lse_recall(q, k, v, lists, lay.valid), rtol=1e-12, atol=1e-15)
    # direct sum of the token probabilities over the kept keys
    s = (q @ k.T) / math.sqrt(8)
    s[:, ~lay.valid] = -np.inf
    P = np.exp(s - s.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    t = 64 * 5 + 3
    assert abs(tau[t] - sum(P[t, j * 64:(j + 1) * 64].sum() for j in lists[5])) < 1e-13
    assert np.all(tau[~lay.valid] == 0) and np.all((tau[lay.valid] > 0) & (tau[lay.valid] <= 1 + 1e-15))
    # every block kept: all the mass
    full = Bq.selected_mass(q, k, [np.arange(T)] * T, lay.valid)
    np.testing.assert_allclose(full[lay.valid], 1.0, rtol=1e-13)
    # cube recall is the P_oracle mass of the kept blocks; the best set of the same size does at least as well
    recall, best = Bq.cube_recall(q, k, lists, lay.valid)
    Po = O.vsa2_router.oracle_block_scores(q, k, lay.valid)
    np.testing.assert_allclose(recall, [Po[i, lists[i]].sum() for i in range(T)], rtol=1e-12)
    assert np.all(best >= recall - 1e-12)
