"""Pins for the oracle's layout and router (CPU only).

Each test checks the oracle against something other than itself: numbers printed
on the pages (tests/golden/selection_examples.json), hand-worked layouts,
closed forms and brute force over every subset of small rows.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle as O

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "selection_examples.json")))


# ---------------------------------------------------------------------------- pages' numbers

@pytest.mark.parametrize("case", GOLD["selection"], ids=lambda c: c["name"])
def test_selection_worked_examples(case):
    if "weights_uniform_n" in case:
        w = np.ones(case["weights_uniform_n"])
    else:
        w = np.array(case["weights"], dtype=np.float64)
    k = case.get("k")
    if k is None:
        k = O.topk_from_fraction(case["k_frac"], len(w))
    got = O.hybrid_ids(w, k, case["p"])
    if "expect" in case:
        assert list(got) == case["expect"]
    if "expect_count" in case:
        assert len(got) == case["expect_count"]
    if "expect_mass" in case:
        assert math.isclose(w[got].sum() / w.sum(), case["expect_mass"], rel_tol=1e-12)


def test_top_p_reaches_or_exceeds():
    # 0.6 >= 0.6 must stop after the sink; a strict '>' would take two blocks.
    w = np.array([12.0, 4, 2, 1, 1])
    assert O.topp_count(w, 0.6) == 1
    assert O.topp_count(w, 0.6 + 1e-9) == 2


def test_topk_fraction_pin():
    for c in GOLD["topk_fraction"]:
        assert O.topk_from_fraction(c["frac"], c["T"]) == c["k"]
    # the build's own workloads: 3% of 624 and 1440 cubes, 1.5% of 1440
    assert O.topk_from_fraction(0.03, 624) == 19
    assert O.topk_from_fraction(0.03, 1440) == 44
    assert O.topk_from_fraction(0.015, 1440) == 22


def test_dropped_mass_pin():
    V = np.eye(3)
    for c in GOLD["dropped_mass"]:
        p, m = np.array(c["p"]), np.array(c["m"], dtype=np.float64)
        dropped, _, tau = O.eq8_error_terms(p, m, V)
        assert math.isclose(1.0 - tau, c["dropped"], rel_tol=1e-12)
        assert math.isclose(dropped.sum(), c["dropped"], rel_tol=1e-12)


def test_vsa_sparsity_and_shape_pins():
    for c in GOLD["vsa_sparsity"]:
        assert math.isclose(O.vsa_sparsity(c["K"], c["B"], c["L"]), c["sparsity"], rel_tol=1e-12)
    for c in GOLD["pbar_shape"]:
        assert list(O.block_grid_shape(c["N"], c["bq"], c["bkv"])) == c["shape"]


# ---------------------------------------------------------------------------- layout

def test_cube_index_hand_examples():
    lay = O.cube_layout((8, 8, 8))
    # token (t=5, h=2, w=7): cube (1, 0, 1) -> id 1*2*2 + 0*2 + 1 = 5; in-cube (1, 2, 3) -> 16 + 8 + 3
    lat_index = 5 * 64 + 2 * 8 + 7
    slot = int(np.nonzero(lay.src == lat_index)[0][0])
    assert slot == 5 * 64 + 27
    # every cube occupies 64 consecutive slots holding one 4x4x4 block of the latent
    for c in range(lay.n_cubes):
        src = lay.src[c * 64:(c + 1) * 64]
        t, h, w = src // 64, (src // 8) % 8, src % 8
        assert len(set(t // 4)) == len(set(h // 4)) == len(set(w // 4)) == 1
        assert sorted(zip(t % 4, h % 4, w % 4)) == sorted(itertools.product(range(4), repeat=3))


def test_layout_padding_and_bijection():
    lay = O.cube_layout((5, 6, 7))
    assert lay.grid == (2, 2, 2) and lay.n_pad == 8 * 64
    L = 5 * 6 * 7
    assert lay.valid.sum() == L
    assert sorted(lay.src[lay.valid].tolist()) == list(range(L))
    # the corner cube (1,1,1) keeps t in {4}, h in {4,5}, w in {4,5,6}: 1*2*3 = 6 valid tokens
    assert lay.valid[7 * 64:8 * 64].sum() == 6
    x = np.random.default_rng(0).standard_normal((2, L, 3))
    y = O.tile(x, lay)
    assert np.all(y[:, ~lay.valid] == 0)
    np.testing.assert_array_equal(O.untile(y, lay), x)


def test_wan_720p_cube_counts():
    lay = O.cube_layout((21, 45, 80))
    assert lay.grid == (6, 12, 20) and lay.n_pad == 92160 and lay.n_cubes == 1440
    n_valid = lay.valid.reshape(1440, 64).sum(axis=1)
    assert (n_valid == 64).sum() == 1100
    assert (n_valid == 16).sum() == 320
    assert (n_valid == 4).sum() == 20


# ---------------------------------------------------------------------------- pooling, scores

def test_pool_constant_partial_and_linear():
    lay = O.cube_layout((5, 4, 4))          # cube 1 holds one valid time slice (16 tokens)
    rng = np.random.default_rng(1)
    x = np.full((lay.n_pad, 3), 2.5)
    x[~lay.valid] = 99.0                     # padding values must not leak into the mean
    np.testing.assert_allclose(O.pool_cubes(x, lay.valid), 2.5, rtol=0, atol=0)
    y = rng.standard_normal((lay.n_pad, 3))
    manual = y[64:128][lay.valid[64:128]].mean(axis=0)
    np.testing.assert_allclose(O.pool_cubes(y, lay.valid)[1], manual, rtol=1e-15)
    assert lay.valid[64:128].sum() == 16
    z = rng.standard_normal((lay.n_pad, 3))
    np.testing.assert_allclose(O.pool_cubes(2 * y - 3 * z, lay.valid),
                               2 * O.pool_cubes(y, lay.valid) - 3 * O.pool_cubes(z, lay.valid),
                               rtol=1e-13, atol=1e-13)


def test_block_softmax_closed_form():
    s = O.block_scores(np.array([[1.0, 0.0]]), np.array([[1.0, 0.0], [0.0, 1.0]]), 1.0)
    p = O.row_softmax(s)
    e = math.e
    np.testing.assert_allclose(p[0], [e / (e + 1), 1 / (e + 1)], rtol=1e-15)
    q = np.array([[2.0, 1.0]]); k = np.array([[1.0, 1.0], [3.0, 0.0]])
    np.testing.assert_allclose(O.block_scores(q, k, 0.5), [[1.5, 3.0]], rtol=1e-15)


# ---------------------------------------------------------------------------- brute force

def _brute_topk(w, k):
    best = max(itertools.combinations(range(len(w)), k), key=lambda c: w[list(c)].sum())
    return set(best)


def _brute_topp(w, p):
    target = p * w.sum()
    for n in range(0, len(w) + 1):
        cands = [c for c in itertools.combinations(range(len(w)), n) if w[list(c)].sum() >= target]
        if cands:
            return n, set(max(cands, key=lambda c: w[list(c)].sum()))
    raise AssertionError


@pytest.mark.parametrize("seed", range(40))
def test_selection_brute_force(seed):
    rng = np.random.default_rng(seed)
    T = int(rng.integers(1, 11))
    w = rng.dirichlet(np.full(T, 0.5))
    k = int(rng.integers(0, T + 1))
    p = float(rng.uniform(0.05, 0.99))
    assert set(O.topk_ids(w, k).tolist()) == _brute_topk(w, k)
    n_p, best = _brute_topp(w, p)
    got = O.topp_ids(w, p)
    assert len(got) == n_p
    assert set(got.tolist()) == best
    # minimality: one block fewer never reaches the target
    srt = np.sort(w)[::-1]
    if n_p > 0:
        assert srt[:n_p].sum() >= p * w.sum() and srt[:n_p - 1].sum() < p * w.sum()
    hyb = set(O.hybrid_ids(w, k, p).tolist())
    union = _brute_topk(w, k) | best
    assert hyb == (union if union else {int(np.argmax(w))})


def test_selection_edge_cases():
    w = np.array([0.1, 0.4, 0.4, 0.1])
    assert list(O.hybrid_ids(w, 0, 0.0)) == [1]            # at least one block: arg-max, lower id on ties
    assert list(O.hybrid_ids(w, 4, 0.0)) == [0, 1, 2, 3]   # k = T keeps all
    assert list(O.hybrid_ids(w, 0, 1.0)) == [0, 1, 2, 3]   # p = 1 keeps all
    assert list(O.hybrid_ids(w, 99, 0.5)) == [0, 1, 2, 3]  # k beyond T is clamped
    assert list(O.topk_ids(w, 1)) == [1]
    assert list(O.hybrid_ids(w, 1, 0.5)) == [1, 2]         # 0.4 < 0.5 <= 0.8


def test_route_head_on_synthetic_tiny():
    import synth
    cfg = synth.get_config("tiny")
    x = synth.make_inputs(cfg, 0, names=("q", "k"))
    lay = O.cube_layout(cfg.lat)
    for h in range(cfg.H):
        q = O.tile(x["q"][0, h].double().numpy(), lay)
        k = O.tile(x["k"][0, h].double().numpy(), lay)
        tr = O.route_head(q, k, lay.valid, cfg.top_k, cfg.top_p)
        np.testing.assert_allclose(tr.pbar.sum(axis=1), 1.0, rtol=1e-12)
        for i, ids in enumerate(tr.lists):
            assert np.all(np.diff(ids) > 0) and ids[0] >= 0 and ids[-1] < lay.n_cubes
            assert len(ids) == max(tr.n_k[i], tr.n_p[i], 1)
        full = O.route_head(q, k, lay.valid, lay.n_cubes, 0.0)
        assert all(len(ids) == lay.n_cubes for ids in full.lists)
