"""Pins for the oracle's coarse branch and gated combination (CPU only).

Independent checks: token-level dense attention (torch float64 SDPA) on inputs that are
constant over each cube, the one-cube and equal-key closed forms, central finite
differences of L = <dO, O>, and torch float64 autograd of the same expression written
another way (pooling as a matrix, the fine branch as SDPA with an additive mask).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O


def _case(lat, D, seed, nsel=2):
    rng = np.random.default_rng(seed)
    lay = O.cube_layout(lat)
    q, k, v, do = (rng.standard_normal((lay.n_pad, D)) for _ in range(4))
    for x in (q, k, v, do):
        x[~lay.valid] = 0.0
    gate = rng.standard_normal(lay.n_pad)
    T = lay.n_cubes
    lists = [np.sort(rng.choice(T, size=min(T, int(rng.integers(1, nsel + 1))), replace=False))
             for _ in range(T)]
    return lay, q, k, v, do, gate, lists


@pytest.mark.parametrize("lat,D", [((4, 8, 8), 8), ((8, 4, 12), 16)])
def test_cube_constant_inputs_equal_token_dense_attention(lat, D):
    # every token of cube i carries (q_i, k_i, v_i): token-level softmax gives each cube's 64
    # equal keys the same weight, so full attention equals the cube-level attention repeated
    rng = np.random.default_rng(1)
    lay = O.cube_layout(lat)
    T = lay.n_cubes
    qc, kc, vc = (rng.standard_normal((T, D)) for _ in range(3))
    q, k, v = (np.repeat(x, 64, axis=0) for x in (qc, kc, vc))
    scale = 1 / math.sqrt(D)
    qbar, kbar, vbar, oc, lse, P = O.coarse_forward_head(q, k, v, lay.valid)
    np.testing.assert_allclose(qbar, qc, rtol=1e-14)
    np.testing.assert_allclose(vbar, vc, rtol=1e-14)
    t = lambda a: torch.from_numpy(a)[None, None]
    ref = F.scaled_dot_product_attention(t(q), t(k), t(v), scale=scale)[0, 0].numpy()
    np.testing.assert_allclose(O.repeat_cubes(oc, lay.valid), ref, rtol=1e-12, atol=1e-12)
    s = (q @ k.T) * scale
    tok_lse = np.log(np.exp(s).sum(axis=1))
    np.testing.assert_allclose(np.repeat(lse, 64) + math.log(64), tok_lse, rtol=1e-12)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=1e-14)


def test_one_cube_closed_form():
    lay, q, k, v, _, _, _ = _case((3, 4, 4), 8, 2)       # one cube, 48 valid tokens
    assert lay.n_cubes == 1 and lay.valid.sum() == 48
    qbar, kbar, vbar, oc, lse, P = O.coarse_forward_head(q, k, v, lay.valid)
    np.testing.assert_allclose(oc[0], v[lay.valid].mean(axis=0), rtol=1e-13)
    np.testing.assert_allclose(lse[0], q[lay.valid].mean(0) @ k[lay.valid].mean(0) / math.sqrt(8), rtol=1e-13)
    assert P[0, 0] == 1.0


def test_equal_keys_give_uniform_weights_over_cubes():
    lay, q, k, v, _, _, _ = _case((5, 6, 7), 8, 3)       # 2 x 2 x 2 cubes, all partial but one
    rng = np.random.default_rng(4)
    k = np.tile(rng.standard_normal(8), (lay.n_pad, 1))
    k[~lay.valid] = 0.0
    qbar, kbar, vbar, oc, lse, P = O.coarse_forward_head(q, k, v, lay.valid)
    T = lay.n_cubes
    np.testing.assert_allclose(P, 1.0 / T, rtol=1e-13)
    # V is averaged over the valid tokens of each cube, then uniformly over cubes
    cube_means = [v[c * 64:(c + 1) * 64][lay.valid[c * 64:(c + 1) * 64]].mean(axis=0) for c in range(T)]
    np.testing.assert_allclose(oc, np.tile(np.mean(cube_means, axis=0), (T, 1)), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, qbar @ k[0] / math.sqrt(8) + math.log(T), rtol=1e-12)


def _loss(q, k, v, gate, do, lists, valid):
    o, _, _, _ = O.gated_forward_head(q, k, v, gate, lists, valid)
    return float((o * do).sum())


def test_gated_backward_central_differences():
    lay, q, k, v, do, gate, lists = _case((5, 4, 8), 4, 5)   # T = 4 cubes, the last two partial
    dq, dk, dv, dg = O.gated_backward_head(q, k, v, do, gate, lists, lay.valid)
    h = 1e-6
    rng = np.random.default_rng(6)
    idx = np.nonzero(lay.valid)[0]
    args = {"q": q, "k": k, "v": v, "gate": gate}
    grads = {"q": dq, "k": dk, "v": dv}
    for name in ("q", "k", "v"):
        for r in rng.choice(idx, 10, replace=False):
            for c in range(4):
                ap, am = dict(args), dict(args)
                ap[name] = args[name].copy(); ap[name][r, c] += h
                am[name] = args[name].copy(); am[name][r, c] -= h
                fd = (_loss(**ap, do=do, lists=lists, valid=lay.valid)
                      - _loss(**am, do=do, lists=lists, valid=lay.valid)) / (2 * h)
                g = grads[name][r, c]
                assert abs(fd - g) <= 1e-6 * max(1.0, abs(g)), (name, r, c, fd, g)
    for r in rng.choice(idx, 16, replace=False):
        gp, gm = gate.copy(), gate.copy()
        gp[r] += h
        gm[r] -= h
        fd = (_loss(q, k, v, gp, do, lists, lay.valid) - _loss(q, k, v, gm, do, lists, lay.valid)) / (2 * h)
        assert abs(fd - dg[r]) <= 1e-6 * max(1.0, abs(dg[r])), (r, fd, dg[r])
    # padding inputs do not reach the output: zero gradients, and the loss ignores them
    for g in (dq, dk, dv):
        assert np.all(g[~lay.valid] == 0)
    assert np.all(dg[~lay.valid] == 0)
    g2 = gate.copy()
    g2[~lay.valid] += 5.0
    assert _loss(q, k, v, g2, do, lists, lay.valid) == _loss(q, k, v, gate, do, lists, lay.valid)
    # dO on padding rows is ignored (the output there is 0 whatever the inputs)
    do2 = do.copy()
    do2[~lay.valid] = np.random.default_rng(9).standard_normal(((~lay.valid).sum(), 4))
    for a, b in zip((dq, dk, dv, dg), O.gated_backward_head(q, k, v, do2, gate, lists, lay.valid)):
        assert np.array_equal(a, b)


def test_gated_backward_matches_autograd_of_matrix_form():
    lay, q, k, v, do, gate, lists = _case((6, 8, 8), 8, 7, nsel=3)  # T = 8, half the cubes partial
    dq, dk, dv, dg = O.gated_backward_head(q, k, v, do, gate, lists, lay.valid)
    o, _, _, _ = O.gated_forward_head(q, k, v, gate, lists, lay.valid)
    T, n = lay.n_cubes, lay.n_pad
    valid = torch.from_numpy(lay.valid)
    # pooling matrix A [T, n]: 1/n_i on the valid slots of cube i; its transpose repeats
    A = torch.zeros(T, n, dtype=torch.float64)
    for c in range(T):
        sl = slice(c * 64, (c + 1) * 64)
        A[c, sl] = valid[sl].double() / valid[sl].sum()
    R = (A > 0).double().T                                      # Repeat_B on valid slots
    allowed = torch.zeros(n, n, dtype=torch.bool)
    for i, sel in enumerate(lists):
        for j in sel:
            allowed[i * 64:(i + 1) * 64, j * 64:(j + 1) * 64] = True
    allowed &= valid[None, :]
    allowed[~valid] = True                                      # padding rows: any finite row, zeroed below
    tq, tk, tv, tg = (torch.tensor(a, requires_grad=True) for a in (q, k, v, gate))
    fine = F.scaled_dot_product_attention(tq[None, None], tk[None, None], tv[None, None], attn_mask=allowed,
                                          scale=1 / math.sqrt(8))[0, 0] * valid[:, None]
    Pc = torch.softmax((A @ tq) @ (A @ tk).T / math.sqrt(8), dim=1)
    out = tg[:, None] * (R @ (Pc @ (A @ tv))) + fine
    np.testing.assert_allclose(out.detach().numpy(), o, rtol=1e-12, atol=1e-12)
    (out * torch.from_numpy(do)).sum().backward()
    for mine, ref in ((dq, tq.grad), (dk, tk.grad), (dv, tv.grad), (dg, tg.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-11)


def test_zero_gate_is_the_fine_branch_alone():
    lay, q, k, v, do, _, lists = _case((5, 6, 7), 8, 8)
    zero = np.zeros(lay.n_pad)
    o, o_f, lse, coarse = O.gated_forward_head(q, k, v, zero, lists, lay.valid)
    ref, ref_lse = O.attention_forward_head(q, k, v, lists, lay.valid)
    assert np.array_equal(o, ref) and np.array_equal(o_f, ref) and np.array_equal(lse, ref_lse)
    dq, dk, dv, dg = O.gated_backward_head(q, k, v, do, zero, lists, lay.valid)
    for a, b in zip((dq, dk, dv), O.attention_backward_head(q, k, v, do, lists, lay.valid)):
        np.testing.assert_allclose(a, b, rtol=0, atol=0)
    np.testing.assert_allclose(dg, (do * O.repeat_cubes(coarse[3], lay.valid)).sum(axis=1), rtol=1e-14)
