"""Pins for two oracle functions that are compositions of pinned parts (CPU only):
``dequantize_rows`` (e4m3 codes times one scale per 64-token cube) and ``route_head``
(pool Q and K, score at the default 1/sqrt(D), softmax, hybrid selection).

Both are checked against values worked out by hand in the comments below, not against
the oracle's own parts.  Each check is also run on deliberately wrong variants (a scale
grouped per token or shifted by one cube; keys pooled from Q, the scale dropped, padding
averaged in) planted in the oracle on the CPU, and must reject every one of them.

Pages: SparkDiffusion page section 4.3 (E4M3 inputs); SpargeAttention2 page,
"Block-Pooled Attention for Efficient Mask Construction", steps 2-3 (mean pooling,
S = Qbar Kbar^T / sqrt(d), row softmax) and "The Hybrid Top-k+Top-p Masking Rule"
(equation 9).
"""
import math

import numpy as np
import pytest

import oracle as O
import oracle.attention as OA

# ------------------------------------------------------------------------------ e4m3
# Codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits) and their values, by hand:
#   0x38 = 0.0111.000 -> 2^0 * 1.000  = 1.0
#   0x39 = 0.0111.001 -> 2^0 * 1.125  = 1.125
#   0x3A = 0.0111.010 -> 2^0 * 1.25   = 1.25
#   0x30 = 0.0110.000 -> 2^-1         = 0.5
#   0x01 = 0.0000.001 -> subnormal 1/8 * 2^-6 = 2^-9
#   0xB8 = 1.0111.000 -> -1.0
#   0x7E = 0.1111.110 -> 2^8 * 1.75   = 448 (largest finite)
#   0x00 -> 0
_CODES = [0x38, 0x39, 0x3A, 0x30, 0x01, 0xB8, 0x7E, 0x00]
_VALUES = [1.0, 1.125, 1.25, 0.5, 2.0 ** -9, -1.0, 448.0, 0.0]
# two cubes of 64 rows, two columns: row r holds code r % 8 in column 0 and code
# (r + 3) % 8 in column 1; cube 0 has scale 0.5, cube 1 scale 3.0
_SCALES = np.array([0.5, 3.0], dtype=np.float32)


def _codes_2cubes():
    c = np.zeros((128, 2), dtype=np.uint8)
    for r in range(128):
        c[r, 0] = _CODES[r % 8]
        c[r, 1] = _CODES[(r + 3) % 8]
    return c


def _expected_2cubes():
    # written out per row from the table above: value(code) * scale(cube of the row)
    e = np.zeros((128, 2))
    for r in range(128):
        s = 0.5 if r < 64 else 3.0
        e[r, 0] = _VALUES[r % 8] * s
        e[r, 1] = _VALUES[(r + 3) % 8] * s
    return e


def _dequant_ok(fn) -> bool:
    try:
        got = fn(_codes_2cubes(), _SCALES)
    except Exception:
        return False
    exp = _expected_2cubes()
    if got.shape != exp.shape or not np.array_equal(got, exp):
        return False
    # the cube boundary, spelled out: row 63 is the last of cube 0 (scale 0.5), row 64 the
    # first of cube 1 (scale 3): row 63 holds codes 0x00 (63 % 8 = 7) and 0x3A (66 % 8 = 2),
    # row 64 codes 0x38 and 0x30, row 65 codes 0x39 and 0x01
    return (got[63, 0] == 0.0 and got[63, 1] == 0.625 and got[64, 0] == 3.0 and got[64, 1] == 1.5
            and got[65, 0] == 3.375 and got[65, 1] == 3.0 * 2.0 ** -9 and got[62, 0] == 224.0)


def test_dequantize_rows_hand_values():
    assert _dequant_ok(O.dequantize_rows)
    assert O.dequantize_rows(_codes_2cubes(), _SCALES)[127, 1] == 3.75   # code 0x3A (130 % 8 = 2) * 3


@pytest.mark.parametrize("variant", ["per_token", "shift_one_row", "shift_one_cube", "groups_of_32"])
def test_dequantize_rows_rejects_planted_mistakes(variant):
    def wrong(codes, scales, rows=64):
        x = O.e4m3_decode(codes)
        s = np.repeat(scales.astype(np.float64), rows)
        if variant == "per_token":                 # one scale per token, cycling
            s = np.resize(scales.astype(np.float64), len(x))
        elif variant == "shift_one_row":           # off by one row at the cube edge
            s = np.roll(s, 1)
        elif variant == "shift_one_cube":          # cube c takes the scale of cube c + 1
            s = np.repeat(np.roll(scales.astype(np.float64), -1), rows)
        elif variant == "groups_of_32":
            s = np.resize(np.repeat(scales.astype(np.float64), 32), len(x))
        return x * s[:, None]
    assert not _dequant_ok(wrong)


# ------------------------------------------------------------------------------ route_head
# Three 64-token cubes, D = 4, so the default scale is 1/sqrt(4) = 0.5.  Token rows:
#   cube 0 (64 valid):   q = (4,0,0,0) on even slots, 0 on odd          -> qbar0 = (2,0,0,0)
#                        k = (1, +0.5,0,0) even, (1, -0.5,0,0) odd        -> kbar0 = (1,0,0,0)
#   cube 1 (16 valid: slots 0..15; slots 16..63 are padding holding 1000 in every entry)
#                        q = (0,2,0,0)                                    -> qbar1 = (0,2,0,0)
#                        k = (0,1,+3,0) even, (0,1,-3,0) odd               -> kbar1 = (0,1,0,0)
#   cube 2 (64 valid):   q = (0,0,+1,+1) even, (0,0,-1,-1) odd             -> qbar2 = 0
#                        k = (1,1,0,0)                                    -> kbar2 = (1,1,0,0)
# Sbar = 0.5 * qbar kbar^T:
#   row 0: (1, 0, 1)   row 1: (0, 1, 1)   row 2: (0, 0, 0)
# Pbar, with E = e = exp(1): row 0 = (E, 1, E) / (2E + 1), row 1 = (1, E, E) / (2E + 1),
# row 2 = (1, 1, 1) / 3.
# Selection with k = 1, p = 0.5 (order: probability descending, then id ascending):
#   row 0: order (0, 2, 1); Top-1 {0}; E/(2E+1) = 0.4223 < 0.5, 2E/(2E+1) = 0.8446 >= 0.5
#          -> n_p = 2, Top-p {0, 2}; hybrid {0, 2}
#   row 1: order (1, 2, 0); hybrid {1, 2} (n_p = 2)
#   row 2: order (0, 1, 2); 1/3 < 0.5, 2/3 >= 0.5 -> n_p = 2; hybrid {0, 1}
def _route_case():
    n_pad, D = 192, 4
    q = np.zeros((n_pad, D))
    k = np.zeros((n_pad, D))
    valid = np.ones(n_pad, bool)
    for s in range(64):
        r = s
        q[r] = (4, 0, 0, 0) if s % 2 == 0 else (0, 0, 0, 0)
        k[r] = (1, 0.5, 0, 0) if s % 2 == 0 else (1, -0.5, 0, 0)
        r = 64 + s
        if s < 16:
            q[r] = (0, 2, 0, 0)
            k[r] = (0, 1, 3, 0) if s % 2 == 0 else (0, 1, -3, 0)
        else:
            valid[r] = False
            q[r] = k[r] = 1000.0
        r = 128 + s
        q[r] = (0, 0, 1, 1) if s % 2 == 0 else (0, 0, -1, -1)
        k[r] = (1, 1, 0, 0)
    return q, k, valid


def _route_ok(route=None) -> bool:
    route = route or O.route_head
    q, k, valid = _route_case()
    tr = route(q, k, valid, 1, 0.5)
    E = math.e
    exp_q = np.array([[2, 0, 0, 0], [0, 2, 0, 0], [0, 0, 0, 0]], float)
    exp_k = np.array([[1, 0, 0, 0], [0, 1, 0, 0], [1, 1, 0, 0]], float)
    exp_p = np.array([[E, 1, E], [1, E, E], [1, 1, 1]], float)
    exp_p /= exp_p.sum(axis=1, keepdims=True)
    return (np.array_equal(tr.qbar, exp_q) and np.array_equal(tr.kbar, exp_k)
            and np.allclose(tr.pbar, exp_p, rtol=1e-14, atol=0)
            and [list(x) for x in tr.lists] == [[0, 2], [1, 2], [0, 1]]
            and list(tr.n_k) == [1, 1, 1] and list(tr.n_p) == [2, 2, 2])


def test_route_head_hand_case():
    assert _route_ok()


def test_route_head_hand_case_probabilities_spelled_out():
    q, k, valid = _route_case()
    tr = O.route_head(q, k, valid, 1, 0.5)
    assert abs(tr.pbar[0, 0] - 0.42231879825152) < 1e-13     # e / (2e + 1), e = 2.718281828459045
    assert abs(tr.pbar[0, 1] - 0.15536240349696) < 1e-13     # 1 / (2e + 1)
    assert abs(tr.pbar[2, 2] - 1.0 / 3.0) < 1e-15


@pytest.mark.parametrize("variant", ["scale_dropped", "scale_one_over_d", "keys_pooled_from_q", "padding_averaged",
                                     "zero_padded_mean"])
def test_route_head_rejects_planted_mistakes(variant, monkeypatch):
    real_scores, real_pool = OA.block_scores, OA.pool_cubes
    if variant == "scale_dropped":
        monkeypatch.setattr(OA, "block_scores", lambda qb, kb, scale: real_scores(qb, kb, 1.0))
    elif variant == "scale_one_over_d":
        monkeypatch.setattr(OA, "block_scores", lambda qb, kb, scale: real_scores(qb, kb, scale * scale))
    elif variant == "keys_pooled_from_q":
        monkeypatch.setattr(OA, "block_scores", lambda qb, kb, scale: real_scores(qb, qb, scale))
    elif variant == "padding_averaged":
        monkeypatch.setattr(OA, "pool_cubes", lambda x, valid, block=64: real_pool(x, np.ones_like(valid), block))
    elif variant == "zero_padded_mean":
        def zero_pad(x, valid, block=64):
            xz = np.where(valid[:, None], x, 0.0)
            return xz.reshape(-1, block, x.shape[1]).sum(axis=1) / block
        monkeypatch.setattr(OA, "pool_cubes", zero_pad)
    assert not _route_ok(OA.route_head)
