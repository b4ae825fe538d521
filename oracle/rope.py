"""3-D rotary position embedding applied together with the cube-major permutation, float64
(TEST INFRASTRUCTURE ONLY, like the rest of this package).

What it restates: VSA2 page, section 2.2 "Permutation": the tokens are permuted into
cube-major order once, at the start of the transformer, with a matching permutation of the
RoPE embeddings (RoFormer, Su et al.), since attention is the only operation that depends on
token order.  RoPE itself (the RoFormer reference the page cites): each consecutive pair of
channels (x_2i, x_2i+1) of a token at position m is rotated by the angle m * theta_i.

Readings where the pages are silent:

r1. The video's RoPE is 3-D: the head dimension splits into three contiguous sections of
    even sizes (d_t, d_h, d_w), d_t + d_h + d_w = D, rotated by the token's t, h and w
    position respectively.
r2. The angles come from caller-given tables, cos and sin of (position * theta_i) per axis:
    rows 0..lat_t-1 of width d_t/2 for t, then lat_h rows of width d_h/2 for h, then lat_w
    rows of width d_w/2 for w (RoFormer's theta_i = base^(-2i/d) is one way to fill them).
r3. A pair (a, b) rotated by an angle with cosine c and sine s becomes (a c - b s, a s + b c).
r4. The fused helper returns the rotated token at its cube-major slot; padding slots are 0.
"""
from __future__ import annotations

import numpy as np

from .attention import CubeLayout, tile, untile


def rope_tables(lat, sections, base: float = 10000.0):
    """(cos, sin) tables in the layout of reading r2 from RoFormer's frequencies
    theta_i = base^(-2i/d) of each section (d = that section's size)."""
    cos, sin = [], []
    for n, d in zip(lat, sections):
        if d == 0:
            continue
        theta = base ** (-np.arange(0, d, 2) / d)
        ang = np.arange(n)[:, None] * theta[None, :]
        cos.append(np.cos(ang).reshape(-1))
        sin.append(np.sin(ang).reshape(-1))
    return np.concatenate(cos), np.concatenate(sin)


def _axis_rows(lat, sections):
    """Offsets of each axis' block of rows in the tables (reading r2)."""
    offs, o = [], 0
    for n, d in zip(lat, sections):
        offs.append(o)
        o += n * (d // 2)
    return offs


def rope_3d(x: np.ndarray, lat, sections, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate every token of ``x [L, D]`` (latent order, row-major t, h, w) by its 3-D position."""
    lt, lh, lw = lat
    L, D = x.shape
    assert L == lt * lh * lw and sum(sections) == D and all(d % 2 == 0 for d in sections)
    offs = _axis_rows(lat, sections)
    out = x.astype(np.float64).copy()
    pos = np.stack(np.meshgrid(np.arange(lt), np.arange(lh), np.arange(lw), indexing="ij"), -1).reshape(L, 3)
    col = 0
    for axis, d in enumerate(sections):
        half = d // 2
        for i in range(half):
            rows = offs[axis] + pos[:, axis] * half + i
            c, s = cos[rows], sin[rows]
            a, b = x[:, col + 2 * i].astype(np.float64), x[:, col + 2 * i + 1].astype(np.float64)
            out[:, col + 2 * i] = a * c - b * s
            out[:, col + 2 * i + 1] = a * s + b * c
        col += d
    return out


def tile_rope(x: np.ndarray, lay: CubeLayout, sections, cos, sin) -> np.ndarray:
    """Reading r4: the cube-major tensor of the rotated tokens ``[n_pad, D]``."""
    return tile(rope_3d(x, lay.lat, sections, cos, sin), lay)


def untile_rope(y: np.ndarray, lay: CubeLayout, sections, cos, sin) -> np.ndarray:
    """The inverse: latent order ``[L, D]``, each token rotated back (the angle negated)."""
    return rope_3d(untile(y, lay), lay.lat, sections, cos, -sin)
