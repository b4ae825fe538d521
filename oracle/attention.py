"""The oracle proper: cube layout, router and masked softmax attention in float64.

Test infrastructure only (see the package docstring).  Each function cites the
passage of the pages it restates.  Readings taken where the pages are silent:

1. Query and key blocks are both one 4x4x4 cube of 64 tokens (VSA page, "Cube
   Partitioning"; VSA2 page section 2.2).  SpargeAttention2's b_q = 128 is a
   different configuration.
2. Pooling over a cube that holds padding averages the valid tokens only.
3. Top-k takes an absolute block count k (the caller converts k% with
   ``topk_from_fraction`` = ceil(k% * T)); k is clamped to T.
4. Top-p keeps the shortest prefix of the descending order whose sum reaches
   (>=) p times the row sum; p >= 1 keeps every block, p <= 0 contributes none.
5. Ties in the descending order are broken by the smaller block index first.
6. Every row keeps at least one block.
7. The softmax scale is 1/sqrt(D) in both stages unless given; lse is the natural
   log of the row's normaliser of the scaled scores.
8. Index lists are written in ascending block order.
9. Padding query rows get O = 0 and lse = 0 and zero gradients; padding keys get
   probability 0 and zero gradients.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


# ----------------------------------------------------------------------------------
# layout (VSA page, "Cube Partitioning and Token Re-Indexing"; VSA2 page 2.2, padding)

@dataclass
class CubeLayout:
    lat: tuple            # valid latent grid (T, H, W)
    cube: tuple           # cube shape, (4, 4, 4)
    grid: tuple           # number of cubes per axis (N_t, N_h, N_w)
    n_pad: int            # padded token count = 64 * N_t * N_h * N_w
    n_cubes: int          # T_n (= T_m): number of cubes
    src: np.ndarray       # [n_pad] latent index of each cube-major slot, -1 for padding
    valid: np.ndarray     # [n_pad] bool


def cube_layout(lat, cube=(4, 4, 4)) -> CubeLayout:
    """Cube-major order of a (T, H, W) latent padded up to multiples of the cube shape.

    Token (t, h, w) goes to slot ``cube_id * B + (t % Ct) * Ch * Cw + (h % Ch) * Cw + (w % Cw)``
    with ``cube_id = (t // Ct) * N_h * N_w + (h // Ch) * N_w + (w // Cw)`` and B = Ct*Ch*Cw.
    The VSA page states this two-term form in words (cube index times B plus the
    position inside the cube); the within-cube order is row-major (t, h, w).
    """
    lt, lh, lw = lat
    ct, ch, cw = cube
    nt, nh, nw = -(-lt // ct), -(-lh // ch), -(-lw // cw)
    bsz = ct * ch * cw
    n_pad = nt * nh * nw * bsz
    src = np.full(n_pad, -1, dtype=np.int64)
    for t in range(nt * ct):
        for h in range(nh * ch):
            for w in range(nw * cw):
                cube_id = (t // ct) * nh * nw + (h // ch) * nw + (w // cw)
                slot = cube_id * bsz + (t % ct) * ch * cw + (h % ch) * cw + (w % cw)
                if t < lt and h < lh and w < lw:
                    src[slot] = t * lh * lw + h * lw + w
    return CubeLayout(tuple(lat), tuple(cube), (nt, nh, nw), n_pad, nt * nh * nw, src, src >= 0)


def tile(x: np.ndarray, lay: CubeLayout) -> np.ndarray:
    """Latent-order ``[..., L, D]`` -> cube-major ``[..., n_pad, D]``; padding slots are zero."""
    out = np.zeros(x.shape[:-2] + (lay.n_pad, x.shape[-1]), dtype=x.dtype)
    out[..., lay.valid, :] = x[..., lay.src[lay.valid], :]
    return out


def untile(y: np.ndarray, lay: CubeLayout) -> np.ndarray:
    """Inverse of :func:`tile` (padding slots are dropped)."""
    L = lay.lat[0] * lay.lat[1] * lay.lat[2]
    out = np.zeros(y.shape[:-2] + (L, y.shape[-1]), dtype=y.dtype)
    out[..., lay.src[lay.valid], :] = y[..., lay.valid, :]
    return out


# ----------------------------------------------------------------------------------
# router (SpargeAttention2 page, "Block-Pooled Attention for Efficient Mask Construction")

def pool_cubes(x: np.ndarray, valid: np.ndarray, block: int = 64) -> np.ndarray:
    """Step 2: mean of the valid tokens of each 64-token block.  ``x`` is ``[n_pad, D]``."""
    n_pad, D = x.shape
    T = n_pad // block
    xb = x.reshape(T, block, D)
    vb = valid.reshape(T, block)
    out = np.zeros((T, D), dtype=np.float64)
    for c in range(T):
        rows = xb[c][vb[c]]
        if len(rows):
            out[c] = rows.sum(axis=0) / len(rows)
    return out


def block_scores(qbar: np.ndarray, kbar: np.ndarray, scale: float) -> np.ndarray:
    """Step 3: S-bar = Q-bar K-bar^T * scale (scale = 1/sqrt(d) on the page)."""
    return (qbar @ kbar.T) * scale


def row_softmax(s: np.ndarray) -> np.ndarray:
    """Step 3: P-bar = Softmax(S-bar) along each row."""
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def descending_order(row: np.ndarray) -> np.ndarray:
    """Block ids sorted by weight, largest first; equal weights: smaller id first (reading 5)."""
    ids = np.arange(len(row))
    return np.lexsort((ids, -row))


def topk_ids(row: np.ndarray, k: int) -> np.ndarray:
    """Top-k selector: the ``k`` largest entries of the row (k clamped to the row length)."""
    k = max(0, min(int(k), len(row)))
    return descending_order(row)[:k]


def topp_count(row: np.ndarray, p: float) -> int:
    """Length of the Top-p prefix: smallest m with sum of the m largest >= p * row sum."""
    T = len(row)
    if p >= 1.0:
        return T
    if p <= 0.0:
        return 0
    target = p * row.sum()
    csum = np.cumsum(row[descending_order(row)])
    reached = np.nonzero(csum >= target)[0]
    return int(reached[0]) + 1 if len(reached) else T


def topp_ids(row: np.ndarray, p: float) -> np.ndarray:
    """Top-p selector: the shortest descending prefix whose cumulative sum reaches p of the total."""
    return descending_order(row)[:topp_count(row, p)]


def hybrid_ids(row: np.ndarray, k: int, p: float) -> np.ndarray:
    """Equation 9: the union of the Top-k and Top-p sets, at least one block, ascending ids."""
    sel = np.union1d(topk_ids(row, k), topp_ids(row, p))
    if len(sel) == 0:
        sel = descending_order(row)[:1]
    return np.sort(sel).astype(np.int64)


@dataclass
class RouterTrace:
    """Everything the parity tests need to check one (b, h) slice of the router."""
    pbar: np.ndarray      # [T, T] fp64 block probabilities
    lists: list           # T arrays of ascending kv block ids
    n_k: np.ndarray       # [T] Top-k size
    n_p: np.ndarray       # [T] Top-p prefix length
    qbar: np.ndarray
    kbar: np.ndarray


def route_head(q: np.ndarray, k: np.ndarray, valid: np.ndarray, top_k: int, top_p: float,
               scale: float | None = None, block: int = 64) -> RouterTrace:
    """The whole router for one head: pool, score, softmax, hybrid select, index lists.

    ``q`` and ``k`` are cube-major ``[n_pad, D]`` float64 (exact copies of the inputs).
    """
    D = q.shape[-1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    qbar = pool_cubes(q, valid, block)
    kbar = pool_cubes(k, valid, block)
    pbar = row_softmax(block_scores(qbar, kbar, scale))
    T = pbar.shape[0]
    lists, nk, npp = [], np.zeros(T, np.int64), np.zeros(T, np.int64)
    for i in range(T):
        row = pbar[i]
        lists.append(hybrid_ids(row, top_k, top_p))
        nk[i] = min(max(top_k, 0), T)
        npp[i] = topp_count(row, top_p)
    return RouterTrace(pbar, lists, nk, npp, qbar, kbar)


def topk_from_fraction(frac: float, T: int) -> int:
    """SpargeAttention2's k% -> block count: ceil(k% * T_n)."""
    return int(math.ceil(frac * T - 1e-12))


def block_grid_shape(N: int, bq: int, bkv: int) -> tuple:
    """Shape of P-bar for N tokens with query blocks of bq and key blocks of bkv (whole blocks)."""
    return (N // bq, N // bkv)


def vsa_sparsity(K: int, B: int, L: int) -> float:
    """VSA's fine-stage sparsity 1 - K*B/L (fraction of the L x L entries that are blocked)."""
    return 1.0 - K * B / L


# ----------------------------------------------------------------------------------
# fine stage: masked softmax attention (SpargeAttention2 page, "Kernel Implementation of
# the Hybrid-Masked Block-Sparse Attention"; VSA2 page 2.1: O = softmax(QK^T/sqrt(D) + M) V)

def _keys_of(lists_i, valid, block):
    cols = np.concatenate([np.arange(j * block, (j + 1) * block) for j in lists_i])
    return cols[valid[cols]]


def attention_forward_head(q, k, v, lists, valid, scale=None, block=64, q_blocks=None):
    """O and lse for one head.  ``lists[i]`` are the key blocks of query block i.

    Two-pass softmax over exactly the valid keys of the selected blocks.
    Returns (o [n_pad, D] fp64, lse [n_pad] fp64); padding rows are 0.
    ``q_blocks`` restricts the work to some query blocks (other rows stay 0).
    """
    n_pad, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = np.zeros((n_pad, v.shape[1]), np.float64)
    lse = np.zeros(n_pad, np.float64)
    T = n_pad // block
    for i in (range(T) if q_blocks is None else q_blocks):
        rows = np.arange(i * block, (i + 1) * block)
        rows = rows[valid[rows]]
        if len(rows) == 0:
            continue
        cols = _keys_of(lists[i], valid, block)
        s = (q[rows] @ k[cols].T) * scale
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        o[rows] = (e / l) @ v[cols]
        lse[rows] = (m + np.log(l))[:, 0]
    return o, lse


def attention_backward_head(q, k, v, do, lists, valid, scale=None, block=64,
                            q_blocks=None, kv_blocks=None, visit=None):
    """dQ, dK, dV of O = softmax(scale*QK^T + M) V with M fixed, for one head.

    dV_c = sum_r P_rc dO_r ; dP_rc = dO_r . v_c ; Delta_r = sum_c P_rc dP_rc ;
    dS = P * (dP - Delta) ; dQ_r = scale sum_c dS_rc k_c ; dK_c = scale sum_r dS_rc q_r.
    ``q_blocks`` limits which dQ rows are produced; ``kv_blocks`` limits which dK/dV
    rows are produced (all query blocks that attend them are still visited).
    ``visit`` limits the query blocks whose contributions are computed at all (a sample
    of the work, used for timing); by default every query block is visited.
    """
    n_pad, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    T = n_pad // block
    dq = np.zeros_like(q, dtype=np.float64)
    dk = np.zeros_like(k, dtype=np.float64)
    dv = np.zeros_like(v, dtype=np.float64)
    want_kv = None if kv_blocks is None else set(int(j) for j in kv_blocks)
    want_q = None if q_blocks is None else set(int(i) for i in q_blocks)
    for i in (range(T) if visit is None else visit):
        sel = lists[i]
        need_q = want_q is None or i in want_q
        need_kv = want_kv is None or any(int(j) in want_kv for j in sel)
        if not (need_q or need_kv):
            continue
        rows = np.arange(i * block, (i + 1) * block)
        rows = rows[valid[rows]]
        if len(rows) == 0:
            continue
        cols = _keys_of(sel, valid, block)
        s = (q[rows] @ k[cols].T) * scale
        e = np.exp(s - s.max(axis=1, keepdims=True))
        P = e / e.sum(axis=1, keepdims=True)
        dP = do[rows] @ v[cols].T
        delta = (P * dP).sum(axis=1, keepdims=True)
        dS = P * (dP - delta)
        if need_q:
            dq[rows] = scale * (dS @ k[cols])
        if need_kv:
            dk[cols] += scale * (dS.T @ q[rows])
            dv[cols] += P.T @ do[rows]
    return dq, dk, dv


def dense_attention_head(q, k, v, valid, scale=None):
    """Plain dense softmax attention over the valid keys (the all-blocks special case)."""
    D = q.shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    s = (q @ k.T) * scale
    s[:, ~valid] = -np.inf
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    P = e / e.sum(axis=1, keepdims=True)
    o = P @ v
    o[~valid] = 0.0
    return o, P


def eq8_error_terms(p: np.ndarray, m: np.ndarray, V: np.ndarray):
    """Equation 8: e = o - o_s = (p*(1-m) + (1 - 1/tau) (p*m)) V, tau = sum_j p_j m_j.

    Returns (dropped term, renormalisation term, tau) for one query row ``p``.
    """
    tau = float((p * m).sum())
    dropped = (p * (1.0 - m)) @ V
    renorm = ((1.0 - 1.0 / tau) * (p * m)) @ V
    return dropped, renorm, tau


# ----------------------------------------------------------------------------------
# fp8 e4m3 inputs (SparkDiffusion page, section 4.3 uses E4M3; the format itself:
# 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities,
# S.1111.111 is NaN)

def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    c = codes.astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & ((c & 7) == 7), np.nan, val)
    return s * val


def dequantize_rows(codes: np.ndarray, scales: np.ndarray, rows: int = 64) -> np.ndarray:
    """``codes [n_pad, D]`` e4m3 bytes with one scale per ``rows`` rows -> float64."""
    x = e4m3_decode(codes)
    return x * np.repeat(scales.astype(np.float64), rows)[:, None]
