"""Pins for the oracle's 3-D RoPE with the cube-major permutation (CPU only).

Checked against: a hand-rotated example, RoPE's defining property (the dot product of a
rotated query and a rotated key depends only on their relative position), pair norms, the
tables written out from RoFormer's frequency formula, and slots rotated one by one from their
own (t, h, w) with math.cos / math.sin.  Planted mistakes (a flipped sine, swapped axes) fail.
"""
import math

import numpy as np
import pytest

import oracle as O
from oracle import rope as R


def test_hand_rotation():
    # D = 2, one axis (t) of 3 positions, theta_0 = 1: token t is rotated by t radians
    cos, sin = np.cos(np.arange(3.0)), np.sin(np.arange(3.0))
    x = np.array([[1.0, 0.0], [1.0, 0.0], [0.0, 1.0]])
    y = R.rope_3d(x, (3, 1, 1), (2, 0, 0), cos, sin)
    assert np.allclose(y[0], [1.0, 0.0], atol=0)
    assert np.allclose(y[1], [math.cos(1.0), math.sin(1.0)], rtol=0, atol=1e-15)
    assert np.allclose(y[2], [-math.sin(2.0), math.cos(2.0)], rtol=0, atol=1e-15)


def test_tables_follow_roformer_frequencies():
    lat, sec = (5, 6, 7), (4, 6, 6)
    cos, sin = R.rope_tables(lat, sec, base=100.0)
    assert len(cos) == 5 * 2 + 6 * 3 + 7 * 3
    # axis h block starts after 5 * 2 entries; pair i = 2 at position m = 4: angle 4 * 100^(-4/6)
    assert math.isclose(cos[10 + 4 * 3 + 2], math.cos(4 * 100.0 ** (-4 / 6)), rel_tol=1e-15)
    # axis w block starts after 10 + 18 entries; pair 1 at position 6: angle 6 * 100^(-2/6)
    assert math.isclose(sin[28 + 6 * 3 + 1], math.sin(6 * 100.0 ** (-2 / 6)), rel_tol=1e-15)


def _check_relative(rope_fn, lat=(6, 5, 7), sec=(4, 6, 6)) -> bool:
    rng = np.random.default_rng(3)
    D = sum(sec)
    cos, sin = R.rope_tables(lat, sec, base=50.0)
    L = lat[0] * lat[1] * lat[2]
    q, k = rng.standard_normal(D), rng.standard_normal(D)
    x = np.tile(q, (L, 1))
    y = np.tile(k, (L, 1))
    rq, rk = rope_fn(x, lat, sec, cos, sin), rope_fn(y, lat, sec, cos, sin)
    idx = lambda t, h, w: (t * lat[1] + h) * lat[2] + w
    dots = []
    for (a, b) in (((0, 0, 0), (1, 2, 3)), ((2, 1, 1), (3, 3, 4)), ((4, 2, 3), (5, 4, 6))):   # same offset (1, 2, 3)
        dots.append(rq[idx(*a)] @ rk[idx(*b)])
    other = rq[idx(0, 0, 0)] @ rk[idx(1, 2, 4)]
    return bool(np.allclose(dots, dots[0], rtol=0, atol=1e-12) and abs(other - dots[0]) > 1e-6)


def test_relative_position_property():
    assert _check_relative(R.rope_3d)


def test_norms_and_identity_at_origin():
    rng = np.random.default_rng(0)
    lat, sec = (4, 4, 5), (4, 2, 2)
    cos, sin = R.rope_tables(lat, sec)
    x = rng.standard_normal((80, 8))
    y = R.rope_3d(x, lat, sec, cos, sin)
    assert np.allclose(y[0], x[0], rtol=0, atol=0)                     # position (0, 0, 0)
    assert np.allclose(np.hypot(y[:, 0::2], y[:, 1::2]), np.hypot(x[:, 0::2], x[:, 1::2]), rtol=1e-14)


def _check_slots() -> bool:
    rng = np.random.default_rng(1)
    lat, sec = (5, 6, 7), (4, 6, 6)
    D = sum(sec)
    lay = O.cube_layout(lat)
    x = rng.standard_normal((lat[0] * lat[1] * lat[2], D))
    cos, sin = R.rope_tables(lat, sec, base=30.0)
    y = R.tile_rope(x, lay, sec, cos, sin)
    if not np.all(y[~lay.valid] == 0):
        return False
    for slot in (0, 63, 64 + 17, lay.n_pad - 1 - 20, int(np.nonzero(lay.valid)[0][-1])):
        if not lay.valid[slot]:
            continue
        src = lay.src[slot]
        pos = (src // (lat[1] * lat[2]), (src // lat[2]) % lat[1], src % lat[2])
        want = x[src].copy()
        col = 0
        for axis, d in enumerate(sec):
            for i in range(d // 2):
                ang = pos[axis] * 30.0 ** (-2 * i / d)
                a, b = x[src, col + 2 * i], x[src, col + 2 * i + 1]
                want[col + 2 * i] = a * math.cos(ang) - b * math.sin(ang)
                want[col + 2 * i + 1] = a * math.sin(ang) + b * math.cos(ang)
            col += d
        if not np.allclose(y[slot], want, rtol=0, atol=1e-13):
            return False
    return True


def test_tile_rope_slots_rotated_from_their_own_position():
    assert _check_slots()


@pytest.mark.parametrize("variant", ["sine_flipped", "axes_swapped"])
def test_planted_mistakes_fail(variant, monkeypatch):
    real = R.rope_3d

    def wrong(x, lat, sec, cos, sin):
        if variant == "sine_flipped":
            return real(x, lat, sec, cos, -sin)
        # h and w positions exchanged: rotate the transposed grid with the same tables, transpose back
        lt, lh, lw = lat
        xt = x.reshape(lt, lh, lw, -1).transpose(0, 2, 1, 3).reshape(lt * lw * lh, -1)
        secs = (sec[0], sec[2], sec[1])
        y = real(xt, (lt, lw, lh), secs, *R.rope_tables((lt, lw, lh), secs, base=30.0))
        return y.reshape(lt, lw, lh, -1).transpose(0, 2, 1, 3).reshape(lt * lh * lw, -1)
    monkeypatch.setattr(R, "rope_3d", wrong)
    assert not _check_slots()


def test_untile_rope_inverts_tile_rope():
    rng = np.random.default_rng(2)
    lat, sec = (5, 6, 7), (4, 6, 6)
    lay = O.cube_layout(lat)
    x = rng.standard_normal((lat[0] * lat[1] * lat[2], sum(sec)))
    cos, sin = R.rope_tables(lat, sec, base=30.0)
    assert np.allclose(R.untile_rope(R.tile_rope(x, lay, sec, cos, sin), lay, sec, cos, sin), x, rtol=0, atol=1e-13)
