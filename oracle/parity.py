"""The parity rule for index lists (test infrastructure, like the rest of the oracle).

A row of the CUDA router matches when its set equals the oracle's.  Selection is an
integer decision taken from floating point, so a differing row is still accepted as a
*tie row* when every block of the symmetric difference has an oracle probability within
``tie_rel`` (1e-6) relative of the oracle's boundary value, or the oracle's cumulative mass
at the Top-p crossing lies within ``tie_rel`` of p times the row sum (SpargeAttention2 page,
equation 9 and "Definition of the two component selectors": the boundary of the Top-k and
Top-p sets is where equal or nearly equal block probabilities make several sets valid).
Tie rows are counted and reported; any other difference is a mismatch.
"""
from __future__ import annotations

import numpy as np

from .attention import RouterTrace, descending_order

TIE_REL = 1e-6


def classify_router_rows(tr: RouterTrace, got_lists, top_p: float, tie_rel: float = TIE_REL):
    """Returns (mismatch rows, tie rows, indices of the mismatching rows)."""
    mismatch, ties, bad_rows = 0, 0, []
    for i, (ref, got) in enumerate(zip(tr.lists, got_lists)):
        if len(ref) == len(got) and np.array_equal(ref, got):
            continue
        row = tr.pbar[i]
        order = descending_order(row)
        n = len(ref)
        bval = row[order[n - 1]]
        sym = np.setxor1d(ref, got)
        tie_a = len(sym) > 0 and bool(np.all(np.abs(row[sym] - bval) <= tie_rel * bval))
        tie_b = False
        if 0 < top_p < 1:
            csum = np.cumsum(row[order])
            target = top_p * row.sum()
            for m in (tr.n_p[i] - 1, tr.n_p[i]):
                if 1 <= m <= len(row) and abs(csum[m - 1] - target) <= tie_rel * target:
                    tie_b = True
        if tie_a or tie_b:
            ties += 1
        else:
            mismatch += 1
            bad_rows.append(i)
    return mismatch, ties, bad_rows
