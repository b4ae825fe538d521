"""Dynamic work distribution of the attention kernels and their per-CTA clock records
(SA_DEBUG_CTA_CLOCKS), through the C ABI.

The forward, dQ and dK/dV kernels take their work items (pairs of cubes) in order from a
per-launch counter.  The records must account for every item and pipeline step exactly once,
and turning them on must not change a single output bit."""
import numpy as np
import pytest
import torch

import block_sparse_attention_cubes_b200 as sa
import synth
from parity import gpu_inputs, gpu_lists

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    from block_sparse_attention_cubes_b200 import build
    build.build()
    yield


def _pair_steps(lists, T):
    """Pipeline steps of the pair items: ceil(|union of the two cubes' lists| / 2) per pair."""
    steps = 0
    for i in range(0, T, 2):
        u = set(lists[i].tolist()) | (set(lists[i + 1].tolist()) if i + 1 < T else set())
        steps += (len(u) + 1) // 2
    return steps


def _transpose(lists, T):
    cols = [[] for _ in range(T)]
    for i, l in enumerate(lists):
        for j in l:
            cols[int(j)].append(i)
    return [np.array(c, dtype=np.int64) for c in cols]


@pytest.mark.parametrize("lat,k", [((8, 8, 12), 3), ((21, 9, 13), 5)])
def test_cta_records_cover_every_item_once(lat, k):
    cfg = synth.small_config("bal", 2, 3, 128, lat, k, 0.9)
    x, p, t = gpu_inputs(cfg)
    idx, cnt = sa.plan(t["q"], t["k"], p)
    ref = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p, with_f32=True)
    gref = sa.backward(t["q"], t["k"], t["v"], ref[0], ref[1], t["do"], idx, cnt, p, out_f32=ref[2])
    pc = sa.make_params(p.B, p.H, p.D, (p.lat_t, p.lat_h, p.lat_w), p.top_k, p.top_p,
                        debug_flags=sa.DEBUG_CTA_CLOCKS)
    wf, wb = sa.new_workspace(pc, sa.OP_FORWARD), sa.new_workspace(pc, sa.OP_BACKWARD)
    out, lse, o32 = sa.forward(t["q"], t["k"], t["v"], idx, cnt, pc, ws=wf, with_f32=True)
    g = sa.backward(t["q"], t["k"], t["v"], out, lse, t["do"], idx, cnt, pc, ws=wb, out_f32=o32)
    torch.cuda.synchronize()
    for a_, b_ in zip((out, lse, o32) + tuple(g), tuple(ref) + tuple(gref)):
        assert torch.equal(a_, b_)
    T = cnt.shape[-1]
    n_items = cfg.B * cfg.H * ((T + 1) // 2)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    fsteps = bsteps = 0
    for b in range(cfg.B):
        for h in range(cfg.H):
            lists = gpu_lists(idx, cnt, b, h)
            fsteps += _pair_steps(lists, T)
            bsteps += _pair_steps(_transpose(lists, T), T)
    for kernel, ws, steps in ((0, wf, fsteps), (1, wb, fsteps), (2, wb, bsteps)):
        rec = sa.cta_clocks(ws, kernel)
        assert rec.shape == (min(n_items, sms), 4), kernel
        assert int(rec[:, 2].sum()) == n_items, kernel
        assert int(rec[:, 3].sum()) == steps, kernel
        assert np.all(rec[:, 1] >= rec[:, 0]) and np.all(rec[:, 0] > 0)
    # without the flag nothing is recorded
    plain = sa.new_workspace(p, sa.OP_FORWARD)
    sa.forward(t["q"], t["k"], t["v"], idx, cnt, p, ws=plain)
    assert sa.cta_clocks(plain, 0).shape == (0, 4)
