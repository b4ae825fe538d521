"""VSA2's fine-grained router, per-sequence Top-K and the oracle block scores, float64
(TEST INFRASTRUCTURE ONLY, like the rest of this package).

What it restates (VSA2 page, section 2.2 and its router equations; "Gradient-Free Router
Design" in section 3.3):

* Q_r, K_r = MeanPool_R([Q, K]): each cube is split into G = 64 / R groups of R = R_t x R_h x
  R_w tokens, and each group is pooled;
* P^_r = Softmax(Q_r K_r^T / sqrt(D)) over all key groups of the sequence, one row per query
  group;
* P_r = the G x G aggregation of P^_r into one score per (query cube, key cube);
* per-sequence Top-K: one budget of N * K blocks for the whole N x N score matrix of a head,
  allocated across query cubes by score instead of K per row;
* P_oracle = MeanPool_{B x B}(P) of the true token-level softmax P, the reference the router
  approximates (R = 1 is that case).

Readings where the pages are silent:

v1. Group layout: slot (a, b, d) of a cube (t, h, w offsets) belongs to group
    ((a // R_t) * (4 // R_h) + b // R_h) * (4 // R_w) + d // R_w; each R_x divides 4.
v2. A group is pooled over its valid tokens; a group without any takes no part (no query
    row, zero probability as a key).
v3. Aggregation: P_r[i, j] is the mass a query group of cube i puts on the key groups of
    cube j, averaged over the valid query groups of cube i.  Each row sums to 1; without
    padding this is G times MeanPool_{G x G}, a constant factor that no Top-K sees.
v4. Per-sequence Top-K keeps the min(K N, N^2) largest entries of P_r per (batch, head),
    ordered by (score descending, row-major index ascending); a query cube may get none
    (the fine branch then contributes 0 for it and the coarse branch still covers it).
v5. The oracle scores use the same aggregation at token level (R = 1).

Pins (tests/test_oracle_vsa2_router.py): R = (4, 4, 4) gives the cube-level router's P-bar,
R = (1, 1, 1) the token-level P_oracle from dense attention, inputs constant over each group
give P_oracle at any R, and per-sequence Top-K is checked by enumeration.
"""
from __future__ import annotations

import math

import numpy as np

from .attention import dense_attention_head


def group_ids(R=(2, 2, 2)) -> tuple:
    """(group id of each of the 64 slots of a cube, G) for group shape R (reading v1)."""
    rt, rh, rw = R
    assert all(4 % r == 0 for r in R), R
    nh, nw = 4 // rh, 4 // rw
    s = np.arange(64)
    a, b, d = s >> 4, (s >> 2) & 3, s & 3
    gid = ((a // rt) * nh + b // rh) * nw + d // rw
    return gid, (4 // rt) * nh * nw


def pool_groups(x: np.ndarray, valid: np.ndarray, R=(2, 2, 2)):
    """MeanPool_R: ``x [n_pad, D]`` -> (means [T, G, D], valid-token counts [T, G])."""
    gid, G = group_ids(R)
    n_pad, D = x.shape
    T = n_pad // 64
    xs = x.reshape(T, 64, D)
    vs = valid.reshape(T, 64)
    means = np.zeros((T, G, D))
    counts = np.zeros((T, G), np.int64)
    for c in range(T):
        for g in range(G):
            rows = xs[c][(gid == g) & vs[c]]
            counts[c, g] = len(rows)
            if len(rows):
                means[c, g] = rows.sum(axis=0) / len(rows)
    return means, counts


def fine_grained_scores(q, k, valid, R=(2, 2, 2), scale=None):
    """P_r [T, T] (rows sum to 1) and the group-level softmax P^_r [T*G, T*G] (rows of
    query groups without valid tokens, and columns of such key groups, are 0)."""
    D = q.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    qr, qn = pool_groups(q, valid, R)
    kr, kn = pool_groups(k, valid, R)
    T, G, _ = qr.shape
    qv, kv = qn.reshape(-1) > 0, kn.reshape(-1) > 0
    s = (qr.reshape(T * G, D) @ kr.reshape(T * G, D).T) * scale
    s[:, ~kv] = -np.inf
    s[~qv] = 0.0                                       # rows without a query: any finite row, zeroed below
    e = np.exp(s - s.max(axis=1, keepdims=True))
    Ph = e / e.sum(axis=1, keepdims=True)
    Ph[~qv] = 0.0
    mass = Ph.reshape(T, G, T, G).sum(axis=3)          # [query cube, query group, key cube]
    Pr = mass.sum(axis=1) / qv.reshape(T, G).sum(axis=1)[:, None]
    return Pr, Ph


def oracle_block_scores(q, k, valid, scale=None):
    """P_oracle: the token-level softmax P aggregated per (query cube, key cube) as in
    reading v3 (mass on cube j averaged over the valid query tokens of cube i)."""
    n_pad = q.shape[0]
    T = n_pad // 64
    _, P = dense_attention_head(q, k, np.zeros_like(q), valid, scale)
    P = P.copy()
    P[~valid] = 0.0
    mass = P.reshape(T, 64, T, 64).sum(axis=3)
    return mass.sum(axis=1) / valid.reshape(T, 64).sum(axis=1)[:, None]


def per_sequence_topk(P: np.ndarray, K: int):
    """Reading v4: the min(K*N, N*N) largest entries of ``P [N, N]`` as ascending per-row lists."""
    N = P.shape[0]
    budget = min(K * N, N * N)
    flat = P.reshape(-1)
    order = np.lexsort((np.arange(N * N), -flat))      # score descending, then index ascending
    keep = np.zeros(N * N, bool)
    keep[order[:budget]] = True
    keep = keep.reshape(N, N)
    return [np.nonzero(keep[i])[0] for i in range(N)]
