"""Pins for the oracle's masked attention, its backward and the e4m3 decoder (CPU only).

Independent checks: torch's float64 scaled_dot_product_attention and autograd as a
library routine, central finite differences, equation 8 of the SpargeAttention2
page as an identity, closed-form invariants, and torch's float8_e4m3fn decoder.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O


def _rand_case(lat, D, seed, nsel=None, block=64):
    rng = np.random.default_rng(seed)
    lay = O.cube_layout(lat)
    n = lay.n_pad
    q, k, v, do = (rng.standard_normal((n, D)) for _ in range(4))
    for x in (q, k, v, do):
        x[~lay.valid] = 0.0
    T = lay.n_cubes
    lists = []
    for i in range(T):
        m = T if nsel is None else int(rng.integers(1, nsel + 1))
        lists.append(np.sort(rng.choice(T, size=min(m, T), replace=False)))
    return lay, q, k, v, do, lists


def _sdpa(q, k, v, valid, scale):
    t = lambda a: torch.from_numpy(a)[None, None]
    mask = torch.from_numpy(valid)[None, None, None, :].expand(1, 1, len(valid), len(valid))
    return F.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=mask, scale=scale)[0, 0].numpy()


@pytest.mark.parametrize("lat,D", [((4, 8, 8), 16), ((5, 6, 7), 8), ((8, 8, 4), 32)])
def test_all_blocks_equals_dense_sdpa(lat, D):
    lay, q, k, v, _, lists = _rand_case(lat, D, 0)
    scale = 1 / math.sqrt(D)
    o, lse = O.attention_forward_head(q, k, v, lists, lay.valid)
    ref = _sdpa(q, k, v, lay.valid, scale)
    np.testing.assert_allclose(o[lay.valid], ref[lay.valid], rtol=1e-12, atol=1e-12)
    assert np.all(o[~lay.valid] == 0) and np.all(lse[~lay.valid] == 0)
    s = (q @ k.T) * scale
    s[:, ~lay.valid] = -np.inf
    ref_lse = np.log(np.exp(s).sum(axis=1))
    np.testing.assert_allclose(lse[lay.valid], ref_lse[lay.valid], rtol=1e-12)
    od, _ = O.dense_attention_head(q, k, v, lay.valid)
    np.testing.assert_allclose(od[lay.valid], ref[lay.valid], rtol=1e-12, atol=1e-12)


def test_single_block_rows_equal_dense_on_that_block():
    lay, q, k, v, _, _ = _rand_case((4, 8, 8), 16, 1)
    T = lay.n_cubes
    lists = [np.array([(i + 1) % T]) for i in range(T)]
    o, _ = O.attention_forward_head(q, k, v, lists, lay.valid)
    for i in range(T):
        j = (i + 1) % T
        rows, cols = slice(i * 64, (i + 1) * 64), slice(j * 64, (j + 1) * 64)
        ref = _sdpa(q[rows], k[cols], v[cols], lay.valid[cols], 0.25)
        np.testing.assert_allclose(o[rows], ref, rtol=1e-12, atol=1e-12)


def test_eq8_error_decomposition_identity():
    lay, q, k, v, _, lists = _rand_case((4, 8, 12), 8, 2, nsel=3)
    o_s, _ = O.attention_forward_head(q, k, v, lists, lay.valid)
    o, P = O.dense_attention_head(q, k, v, lay.valid)
    for r in np.nonzero(lay.valid)[0][::7]:
        i = r // 64
        m = np.zeros(lay.n_pad)
        for j in lists[i]:
            m[j * 64:(j + 1) * 64] = 1.0
        m *= lay.valid
        dropped, renorm, tau = O.eq8_error_terms(P[r], m, v)
        assert 0 < tau <= 1
        np.testing.assert_allclose(o[r] - o_s[r], dropped + renorm, rtol=1e-10, atol=1e-12)


def test_constant_v_and_shift_invariance():
    lay, q, k, v, _, lists = _rand_case((4, 8, 8), 8, 3, nsel=2)
    c = np.random.default_rng(9).standard_normal(8)
    vc = np.tile(c, (lay.n_pad, 1))
    o, _ = O.attention_forward_head(q, k, vc, lists, lay.valid)
    np.testing.assert_allclose(o[lay.valid], np.tile(c, (lay.valid.sum(), 1)), rtol=1e-13, atol=1e-13)
    o1, lse1 = O.attention_forward_head(q, k, v, lists, lay.valid)
    u = np.random.default_rng(10).standard_normal(8)
    o2, lse2 = O.attention_forward_head(q, k + u, v, lists, lay.valid)   # scores shift by q.u per row
    np.testing.assert_allclose(o2, o1, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse2[lay.valid] - lse1[lay.valid], (q @ u)[lay.valid] / math.sqrt(8),
                               rtol=1e-10, atol=1e-11)


def _loss(q, k, v, g, lists, valid):
    o, _ = O.attention_forward_head(q, k, v, lists, valid)
    return float((o * g).sum())


def test_backward_central_differences():
    lay, q, k, v, do, lists = _rand_case((4, 4, 12), 4, 4, nsel=2)   # 3 cubes, 192 tokens
    dq, dk, dv = O.attention_backward_head(q, k, v, do, lists, lay.valid)
    h = 1e-6
    rng = np.random.default_rng(5)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        idx = np.nonzero(lay.valid)[0]
        for r in rng.choice(idx, 12, replace=False):
            for c in range(4):
                xp, xm = x.copy(), x.copy()
                xp[r, c] += h
                xm[r, c] -= h
                args_p = {"q": q, "k": k, "v": v}; args_p[name] = xp
                args_m = {"q": q, "k": k, "v": v}; args_m[name] = xm
                fd = (_loss(args_p["q"], args_p["k"], args_p["v"], do, lists, lay.valid)
                      - _loss(args_m["q"], args_m["k"], args_m["v"], do, lists, lay.valid)) / (2 * h)
                assert abs(fd - g[r, c]) <= 1e-6 * max(1.0, abs(g[r, c])), (name, r, c, fd, g[r, c])
    for g in (dq, dk, dv):
        assert np.all(g[~lay.valid] == 0)


def test_backward_invariants_and_dense_autograd():
    lay, q, k, v, do, lists = _rand_case((4, 8, 8), 16, 6, nsel=3)
    dq, dk, dv = O.attention_backward_head(q, k, v, do, lists, lay.valid)
    np.testing.assert_allclose(dk.sum(axis=0), 0.0, atol=1e-11)
    np.testing.assert_allclose(dv.sum(axis=0), do[lay.valid].sum(axis=0), rtol=1e-11, atol=1e-11)
    # all blocks: equal to the autograd gradient of dense SDPA in float64
    _, q, k, v, do, full = _rand_case((4, 8, 8), 16, 7)
    dq, dk, dv = O.attention_backward_head(q, k, v, do, full, lay.valid)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (q, k, v))
    mask = torch.from_numpy(lay.valid)[None, None, None, :].expand(1, 1, lay.n_pad, lay.n_pad)
    out = F.scaled_dot_product_attention(tq[None, None], tk[None, None], tv[None, None], attn_mask=mask, scale=0.25)
    g = torch.from_numpy(do * lay.valid[:, None])
    (out[0, 0] * g).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-10, atol=1e-11)


def test_partial_rows_restriction_matches_full():
    lay, q, k, v, do, lists = _rand_case((5, 8, 8), 8, 8, nsel=3)
    o, lse = O.attention_forward_head(q, k, v, lists, lay.valid)
    o2, lse2 = O.attention_forward_head(q, k, v, lists, lay.valid, q_blocks=[1, 3])
    for i in (1, 3):
        np.testing.assert_array_equal(o2[i * 64:(i + 1) * 64], o[i * 64:(i + 1) * 64])
    dq, dk, dv = O.attention_backward_head(q, k, v, do, lists, lay.valid)
    dq2, dk2, dv2 = O.attention_backward_head(q, k, v, do, lists, lay.valid, q_blocks=[2], kv_blocks=[0, 5])
    np.testing.assert_allclose(dq2[128:192], dq[128:192], rtol=1e-13, atol=1e-14)
    for j in (0, 5):
        sl = slice(j * 64, (j + 1) * 64)
        np.testing.assert_allclose(dk2[sl], dk[sl], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(dv2[sl], dv[sl], rtol=1e-12, atol=1e-13)


def test_e4m3_decode_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[ok], ref[ok])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x38] == 1.0
