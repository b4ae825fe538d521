"""SpargeAttention2's asymmetric blocks (b_q = 128 query tokens, b_kv = 64 key tokens) on the
cube layout, and the router recall diagnostic, float64 (TEST INFRASTRUCTURE ONLY, like the
rest of this package).

What it restates:

* asymmetric blocks .... SpargeAttention2 page, "Block-Pooled Attention for Efficient Mask
                         Construction" step 1 (T_m = N / b_q query blocks, T_n = N / b_kv key
                         blocks, b_q = 128 and b_kv = 64 in all experiments) with steps 2-4 and
                         equation 9 unchanged: pooling, scores, row softmax and the hybrid
                         Top-k / Top-p union, now over a T_m x T_n matrix
* recall ............... SpargeAttention2 page, equation 8: tau = sum_j p_j m_j, the share of a
                         query's true attention mass inside its kept blocks; VSA2 page, section
                         2.2: P_oracle = MeanPool_{B x B}(P), against which a selection of n
                         blocks per query cube can be measured (VSA page, "Kernel Implementation":
                         Top-32 captures 50-90% of the mass)

Readings where the pages are silent:

s1. On the cube-major layout a 128-token query block is the two consecutive cubes 2i and
    2i + 1; with an odd cube count the last block is one cube.
s2. A query block is pooled over the valid tokens of both its cubes; keys stay per cube.
s3. Every query token of block i attends the key cubes block i selected (both cubes of the
    block share one list).
s4. Recall of a query cube: the mean over its valid rows of tau; the best recall with n blocks
    is the sum of the n largest entries of that cube's P_oracle row.

Pins (tests/test_oracle_blocks128.py): pair-duplicated queries give the 64-token router's
lists, scores against token loops, the fine stage against SDPA with a token mask built from
the block lists; recall against equation 8's tau, against exp(lse_selected - lse_all), and
the identity with P_oracle.
"""
from __future__ import annotations

import math

import numpy as np

from .attention import (attention_forward_head, block_scores, dense_attention_head, eq8_error_terms,
                        hybrid_ids, pool_cubes, row_softmax)
from .vsa2_router import oracle_block_scores


def pool_query_pairs(q: np.ndarray, valid: np.ndarray) -> np.ndarray:
    """Reading s1-s2: mean of the valid tokens of each 128-token query block, ``[ceil(T/2), D]``."""
    n_pad, D = q.shape
    if (n_pad // 64) % 2:
        q = np.concatenate([q, np.zeros((64, D))])
        valid = np.concatenate([valid, np.zeros(64, bool)])
    return pool_cubes(q, valid, block=128)


def route_head_bq128(q, k, valid, top_k: int, top_p: float, scale=None):
    """Router with 128-token query blocks: (lists per query block, P-bar [ceil(T/2), T])."""
    D = q.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    pbar = row_softmax(block_scores(pool_query_pairs(q, valid), pool_cubes(k, valid), scale))
    return [hybrid_ids(row, top_k, top_p) for row in pbar], pbar


def cube_lists(block_lists, T: int):
    """Reading s3: the list of query block i for both of its cubes (T per-cube lists)."""
    return [block_lists[c // 2] for c in range(T)]


def selected_mass(q, k, lists, valid, scale=None):
    """tau per query token (0 on padding rows): true softmax mass inside the selected cubes."""
    n_pad = q.shape[0]
    _, P = dense_attention_head(q, k, np.zeros_like(q), valid, scale)
    tau = np.zeros(n_pad)
    for i, sel in enumerate(lists):
        rows = np.arange(i * 64, (i + 1) * 64)
        rows = rows[valid[rows]]
        if len(rows) == 0:
            continue
        m = np.zeros(n_pad)
        for j in sel:
            m[j * 64:(j + 1) * 64] = 1.0
        for t in rows:
            tau[t] = eq8_error_terms(P[t], m, np.zeros((n_pad, 1)))[2]
    return tau


def cube_recall(q, k, lists, valid, scale=None):
    """Reading s4: (recall of each query cube, best recall with the same block counts)."""
    T = q.shape[0] // 64
    tau = selected_mass(q, k, lists, valid, scale)
    vb = valid.reshape(T, 64)
    recall = np.array([tau[i * 64:(i + 1) * 64][vb[i]].mean() for i in range(T)])
    Po = oracle_block_scores(q, k, valid, scale)
    best = np.array([np.sort(Po[i])[::-1][:len(lists[i])].sum() for i in range(T)])
    return recall, best


def lse_recall(q, k, v, lists, valid, scale=None):
    """tau per token as exp(lse over the selected keys - lse over all keys) (0 on padding)."""
    T = q.shape[0] // 64
    _, lse_sel = attention_forward_head(q, k, v, lists, valid, scale)
    _, lse_all = attention_forward_head(q, k, v, [np.arange(T)] * T, valid, scale)
    return np.where(valid, np.exp(lse_sel - lse_all), 0.0)
