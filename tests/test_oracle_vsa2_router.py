"""Pins for the oracle's VSA2 fine-grained router, per-sequence Top-K and oracle block
scores (CPU only).

Independent checks: R = one whole cube reproduces the cube-level router's P-bar (pooling,
scores and row softmax of the already pinned router); R = one token reproduces the
token-level softmax of dense attention (pinned against torch SDPA) aggregated per cube
pair; inputs constant over each group make every R agree with the token level; the
per-sequence selection is checked against a plain enumeration of all entries.
"""
import itertools
import math

import numpy as np
import pytest

import oracle as O
from oracle import vsa2_router as V


def _case(lat, D, seed):
    rng = np.random.default_rng(seed)
    lay = O.cube_layout(lat)
    q, k = (rng.standard_normal((lay.n_pad, D)) for _ in range(2))
    q[~lay.valid] = 0.0
    k[~lay.valid] = 0.0
    return lay, q, k


def test_group_layout():
    for R in itertools.product((1, 2, 4), repeat=3):
        gid, G = V.group_ids(R)
        assert G == 64 // (R[0] * R[1] * R[2])
        counts = np.bincount(gid, minlength=G)
        assert np.all(counts == 64 // G)                  # equal groups tile the cube
        # a group is one R_t x R_h x R_w box of the cube's (t, h, w) offsets
        s = np.arange(64)
        for g in range(G):
            a, b, d = s[gid == g] >> 4, (s[gid == g] >> 2) & 3, s[gid == g] & 3
            assert np.ptp(a) == R[0] - 1 and np.ptp(b) == R[1] - 1 and np.ptp(d) == R[2] - 1


@pytest.mark.parametrize("lat", [(4, 8, 8), (5, 6, 7)])
def test_whole_cube_groups_are_the_cube_router(lat):
    lay, q, k = _case(lat, 8, 1)
    Pr, _ = V.fine_grained_scores(q, k, lay.valid, R=(4, 4, 4))
    pbar = O.row_softmax(O.block_scores(O.pool_cubes(q, lay.valid), O.pool_cubes(k, lay.valid), 1 / math.sqrt(8)))
    np.testing.assert_allclose(Pr, pbar, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("lat", [(4, 8, 8), (5, 6, 7)])
def test_single_token_groups_are_the_token_softmax(lat):
    lay, q, k = _case(lat, 8, 2)
    Pr, _ = V.fine_grained_scores(q, k, lay.valid, R=(1, 1, 1))
    Po = V.oracle_block_scores(q, k, lay.valid)
    np.testing.assert_allclose(Pr, Po, rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(Po.sum(axis=1), 1.0, rtol=1e-12)
    # P_oracle by brute force on one cube pair: token probabilities of full attention
    s = (q @ k.T) / math.sqrt(8)
    s[:, ~lay.valid] = -np.inf
    P = np.exp(s - s.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    rows = [t for t in range(64, 128) if lay.valid[t]]
    assert abs(Po[1, 0] - np.mean([P[t, 0:64].sum() for t in rows])) < 1e-12


@pytest.mark.parametrize("R", [(2, 2, 2), (1, 2, 2), (4, 2, 1)])
def test_group_constant_inputs_match_the_token_level(R):
    # every token of a group carries its group's vectors; no padding, so every group has R
    # tokens and the token-level softmax splits each group's weight evenly among them
    lay = O.cube_layout((8, 8, 8))
    gid, G = V.group_ids(R)
    rng = np.random.default_rng(3)
    T = lay.n_cubes
    qg, kg = rng.standard_normal((T, G, 8)), rng.standard_normal((T, G, 8))
    q = qg[:, gid].reshape(-1, 8)
    k = kg[:, gid].reshape(-1, 8)
    Pr, Ph = V.fine_grained_scores(q, k, lay.valid, R=R)
    np.testing.assert_allclose(Pr, V.oracle_block_scores(q, k, lay.valid), rtol=1e-11)
    np.testing.assert_allclose(Ph.sum(axis=1), 1.0, rtol=1e-12)


def test_padding_groups_take_no_part():
    lay, q, k = _case((5, 6, 7), 8, 4)          # every axis ragged: some groups of edge cubes are empty
    Pr, Ph = V.fine_grained_scores(q, k, lay.valid, R=(2, 2, 2))
    _, cnt = V.pool_groups(q, lay.valid, R=(2, 2, 2))
    empty = cnt.reshape(-1) == 0
    assert empty.any()
    assert np.all(Ph[empty] == 0) and np.all(Ph[:, empty] == 0)
    np.testing.assert_allclose(Ph[~empty].sum(axis=1), 1.0, rtol=1e-12)
    np.testing.assert_allclose(Pr.sum(axis=1), 1.0, rtol=1e-12)
    # garbage in padding slots changes nothing
    q2, k2 = q.copy(), k.copy()
    q2[~lay.valid] = 7.0
    k2[~lay.valid] = -3.0
    assert np.array_equal(V.fine_grained_scores(q2, k2, lay.valid, R=(2, 2, 2))[0], Pr)


def test_per_sequence_topk_by_enumeration():
    rng = np.random.default_rng(5)
    N = 7
    P = rng.random((N, N))
    P[2, 3] = P[4, 1] = P[0, 6]                      # ties: broken by row-major index
    for K in range(0, N + 2):
        lists = V.per_sequence_topk(P, K)
        budget = min(K * N, N * N)
        assert sum(len(l) for l in lists) == budget
        chosen = {(i, int(j)) for i, l in enumerate(lists) for j in l}
        ranked = sorted(((P[i, j], -(i * N + j)), (i, j)) for i in range(N) for j in range(N))[::-1]
        assert chosen == {ij for _, ij in ranked[:budget]}
        for l in lists:
            assert np.all(np.diff(l) > 0)
    # a single dominant row takes several blocks, another row may take none
    P = np.full((4, 4), 0.01)
    P[0] = [0.97, 0.96, 0.95, 0.94]
    lists = V.per_sequence_topk(P, 1)
    assert [len(l) for l in lists] == [4, 0, 0, 0]
