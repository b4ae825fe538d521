"""Coarse branch and gated combination, float64 (TEST INFRASTRUCTURE ONLY, like the rest of
this package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it).

What it restates:

* coarse branch ........ VSA page, "Big-Picture Architecture" item 2 and "What the coarse
                         attention output O_c provides"; VSA2 page section 2.2, "Coarse
                         Branch": the mean-pooled Q_c, K_c, V_c, the dense cube-level softmax
                         P_c = Softmax(Q_c K_c^T / sqrt(D)), O^_c = P_c V_c, and
                         O_c = Repeat_B(O^_c) back on the tokens of each cube
* gated combination .... VSA2 page section 2.2, the gate equation: O = G (.) O_c + O_f with
                         G = tanh(X W_g), one scalar per token (and head); VSA page, "Gated
                         Combination" (the fine gate removed, i.e. G_f = 1, in its sparse
                         adaptation)
* backward ............. textbook derivative of the expression above: the mask M of the fine
                         branch is held constant (VSA2 page section 2.1), everything else
                         (pooling, the cube-level softmax, the gate) carries gradient

Readings where the pages are silent:

c1. The operation takes the gate values G (after the tanh); the projection X W_g and its
    tanh are linear-layer work outside attention, like the Q, K, V projections, so the
    backward returns dL/dG.
c2. V is pooled like Q and K: the mean of the valid tokens of each cube.  Repeat_B writes
    O^_c only to valid slots; padding rows of O stay 0 and the gate at a padding slot has
    no effect (its gradient is 0).
c3. The cube-level softmax runs over all T cubes (every cube holds a valid token), with
    the fine stage's scale (1/sqrt(D) unless given).
c4. The adjoint of the mean over the n_i valid tokens of cube i hands dX_i / n_i to each
    of them.

Parity pins (tests/test_oracle_coarse.py): token-level dense attention on cube-constant
inputs, the one-cube and equal-key closed forms, and central finite differences of
L = <dO, O> with respect to q, k, v and G.
"""
from __future__ import annotations

import math

import numpy as np

from .attention import attention_backward_head, attention_forward_head, block_scores, pool_cubes, row_softmax


def coarse_forward_head(q, k, v, valid, scale=None, block=64):
    """Cube-level dense attention for one head.

    Returns (qbar, kbar, vbar [T, D], oc_hat [T, D], lse_c [T], P_c [T, T]); lse_c is the
    natural log of each row's normaliser of the scaled scores.
    """
    D = q.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    qbar, kbar, vbar = (pool_cubes(x, valid, block) for x in (q, k, v))
    s = block_scores(qbar, kbar, scale)
    P = row_softmax(s)
    m = s.max(axis=1)
    lse = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
    return qbar, kbar, vbar, P @ vbar, lse, P


def repeat_cubes(xc, valid, block=64):
    """Repeat_B: row i of ``xc [T, D]`` on every valid slot of cube i; padding slots 0."""
    out = np.repeat(np.asarray(xc, np.float64), block, axis=0)
    out[~valid] = 0.0
    return out


def gated_forward_head(q, k, v, gate, lists, valid, scale=None, block=64, q_blocks=None):
    """O = G (.) Repeat_B(O^_c) + BlockSparseAttn(Q, K, V; M) for one head.

    ``gate`` is ``[n_pad]`` (one scalar per token).  Returns (o, o_f, lse, coarse) where
    ``coarse`` is the tuple of :func:`coarse_forward_head`.  ``q_blocks`` restricts the
    fine branch to some query blocks (as in :func:`attention_forward_head`); rows outside
    them are then meaningful only through the coarse term.
    """
    o_f, lse = attention_forward_head(q, k, v, lists, valid, scale, block, q_blocks)
    coarse = coarse_forward_head(q, k, v, valid, scale, block)
    o = np.asarray(gate, np.float64)[:, None] * repeat_cubes(coarse[3], valid, block) + o_f
    return o, o_f, lse, coarse


def gated_backward_head(q, k, v, do, gate, lists, valid, scale=None, block=64, q_blocks=None, kv_blocks=None,
                        visit=None):
    """dQ, dK, dV (fine plus coarse) and dG of L = <dO, O>, O as in :func:`gated_forward_head`.

    Fine branch: its output enters O with weight 1, so it takes dO as is.
    Coarse branch, per cube i with valid tokens t and n_i of them:
        dG_t = dO_t . O^_c[i];       dO^_c[i] = sum_t G_t dO_t
        dV_c = P_c^T dO^_c;          dP_c = dO^_c V_c^T
        dS_c = P_c (.) (dP_c - rowsum(P_c (.) dP_c))
        dQ_c = scale dS_c K_c;       dK_c = scale dS_c^T Q_c
    and each valid token of cube i receives dX_c[i] / n_i.  ``q_blocks`` / ``kv_blocks`` /
    ``visit`` restrict the fine branch's dQ rows / dK, dV rows / visited query blocks as in
    :func:`attention_backward_head` (the cube-level part is always complete).
    """
    n_pad, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    T = n_pad // block
    dq, dk, dv = attention_backward_head(q, k, v, do, lists, valid, scale, block, q_blocks, kv_blocks, visit)
    qbar, kbar, vbar, oc_hat, _, P = coarse_forward_head(q, k, v, valid, scale, block)
    g = np.asarray(gate, np.float64) * valid
    dgate = (do * repeat_cubes(oc_hat, valid, block)).sum(axis=1)
    doc = (g[:, None] * do).reshape(T, block, D).sum(axis=1)
    dvbar = P.T @ doc
    dP = doc @ vbar.T
    dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
    dqbar = scale * (dS @ kbar)
    dkbar = scale * (dS.T @ qbar)
    n = valid.reshape(T, block).sum(axis=1).astype(np.float64)
    for grad, gbar in ((dq, dqbar), (dk, dkbar), (dv, dvbar)):
        grad += repeat_cubes(gbar / n[:, None], valid, block)
    return dq, dk, dv, dgate
