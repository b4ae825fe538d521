"""Device-side error reporting through the workspace status block (no GPU fault is
caused: bad entries are skipped by the kernels' own range checks, and the timeout
test uses the library's hook that makes a producer issue no loads, so the consumers'
bounded waits run out and the kernel returns)."""
import pytest
import torch

import block_sparse_attention_cubes_b200 as sa
import synth
from parity import gpu_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    from block_sparse_attention_cubes_b200 import build
    build.build()
    yield


def _case():
    cfg = synth.small_config("st", 1, 2, 128, (8, 8, 12), 3, 0.9)
    x, p, t = gpu_inputs(cfg)
    idx, cnt = sa.plan(t["q"], t["k"], p)
    return cfg, p, t, idx, cnt


def test_index_out_of_range_is_reported():
    cfg, p, t, idx, cnt = _case()
    bad = idx.clone()
    bad[0, 1, 3, 0] = cnt.shape[-1]          # == T, one past the last cube
    ws = sa.new_workspace(p, sa.OP_FORWARD)
    out, lse = sa.forward(t["q"], t["k"], t["v"], bad, cnt, p, ws=ws)
    assert sa.device_status(ws) == 8         # SA_ERR_DEVICE_INDEX
    assert torch.isfinite(out.float()).all()
    out2, _ = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p, ws=ws)
    assert sa.device_status(ws) == 0         # the next call starts from a clean status
    bad_cnt = cnt.clone()
    bad_cnt[0, 0, 0] = p.kv_capacity + 1
    sa.forward(t["q"], t["k"], t["v"], idx, bad_cnt, p, ws=ws)
    assert sa.device_status(ws) == 8


def test_capacity_clipping_is_reported():
    cfg = synth.small_config("cap", 1, 2, 128, (8, 8, 12), 6, 0.9)
    x, p0, t = gpu_inputs(cfg, names=("q", "k"))
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, 6, 0.9, kv_capacity=2)
    ws = sa.new_workspace(p, sa.OP_PLAN)
    idx, cnt = sa.plan(t["q"], t["k"], p, ws=ws)
    assert sa.device_status(ws) == 4         # SA_ERR_CAPACITY
    assert int(cnt.max()) == 2


def test_bounded_wait_times_out_and_context_survives():
    cfg, p, t, idx, cnt = _case()
    hooked = sa.make_params(p.B, p.H, p.D, (p.lat_t, p.lat_h, p.lat_w), p.top_k, p.top_p,
                            timeout_ms=200, debug_flags=sa.DEBUG_SKIP_LOADS)
    ws = sa.new_workspace(hooked, sa.OP_FORWARD)
    sa.forward(t["q"], t["k"], t["v"], idx, cnt, hooked, ws=ws)
    assert sa.device_status(ws) == 7         # SA_ERR_DEVICE_TIMEOUT
    out, lse = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p, ws=ws)
    assert sa.device_status(ws) == 0
    assert torch.isfinite(out.float()).all()


def test_host_errors_before_launch():
    import ctypes
    cfg, p, t, idx, cnt = _case()
    small = torch.empty(8, dtype=torch.uint8, device="cuda")
    with pytest.raises(sa.SAError) as e:
        sa.plan(t["q"], t["k"], p, ws=small)
    assert e.value.status == 5
    with pytest.raises(ValueError):
        sa.forward(t["q"][:, :, 1:], t["k"], t["v"], idx, cnt, p)       # wrong shape, caught by the binding
    # a pointer 2 bytes into a buffer is refused by the C ABI before any launch
    lib = sa.load_library()
    ws = sa.new_workspace(p, sa.OP_PLAN)
    st = lib.sa_plan(ctypes.c_void_p(t["q"].data_ptr() + 2), ctypes.c_void_p(t["k"].data_ptr()), None, None,
                     ctypes.byref(p), ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(cnt.data_ptr()),
                     ctypes.c_void_p(ws.data_ptr()), ws.numel(), None)
    assert st == 3
