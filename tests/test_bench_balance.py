"""Host-side load-balance model of bench.py --sweep (CPU only)."""
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_selection_masks_from_lists():
    idx = torch.tensor([[[[0, 2, 9], [1, 9, 9], [0, 1, 2]]]], dtype=torch.int32)   # B=1, H=1, T=3, cap=3
    cnt = torch.tensor([[[2, 1, 3]]], dtype=torch.int32)
    (M,) = bench.selection_masks(idx, cnt)
    assert M.tolist() == [[True, False, True], [False, True, False], [True, True, True]]


def test_cta_balance_by_hand():
    # T = 3 -> pairs (0,1) and (2, -).  Rows: {0,2}, {1}, {0,1,2}; columns: {0,2}, {1,2}, {0,2}.
    M = np.array([[1, 0, 1], [0, 1, 0], [1, 1, 1]], bool)
    r = bench.cta_balance([M, M], sms=3)
    # query pairs: unions {0,1,2} (3 entries -> 2 steps, 3 tiles) and {0,1,2} (2 steps, 3 tiles);
    # items 0..3 over 3 CTAs: CTA 0 gets items 0 and 3
    f = r["forward_dq"]
    assert f["ctas"] == 3 and f["steps_per_cta_max"] == 4
    assert abs(f["steps_max_over_mean"] - 4 / (8 / 3)) < 1e-3
    # key pairs: columns 0,1 -> {0,1,2} (2 steps, 4 tiles); column 2 -> {0,2} (1 step, 2 tiles)
    k = r["dkdv"]
    assert k["steps_per_cta_max"] == 3 and abs(k["tiles_max_over_mean"] - 6 / 4) < 1e-3
    assert abs(r["union_entries_per_tile"] - 12 / 12) < 1e-9
