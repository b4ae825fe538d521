"""sa_step_host (one step from and to host memory, copies overlapped with the work over chunks of
(batch, head) problems) against the device entry points run on the same data: tile, sa_plan,
sa_forward (fp32 output kept), sa_backward, untile.

Every (batch, head) problem is computed by the same kernels whatever the chunk it falls in,
so the host results must equal the device path's bit for bit (the fp16 single-product switch
of the backward is decided per call; these inputs take it in every chunk and in the whole).
The device path itself is held to the oracle by the parity tests.
"""
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


def _device_step(x, p, t):
    idx, cnt = sa.plan(t["q"], t["k"], p)
    out, lse, o32 = sa.forward(t["q"], t["k"], t["v"], idx, cnt, p, with_f32=True)
    dq, dk, dv = sa.backward(t["q"], t["k"], t["v"], out, lse, t["do"], idx, cnt, p, out_f32=o32)
    return [sa.untile(r, p).cpu() for r in (out, dq, dk, dv)]


@pytest.mark.parametrize("name,B,H,D,lat,k,pp,chunks", [
    ("sh_b2h3", 2, 3, 128, (5, 9, 13), 3, 0.9, (1, 4, 6, 100)),   # ragged grid; chunks of 1, 4 + 2, all
    ("sh_d64", 1, 5, 64, (8, 8, 12), 2, 0.8, (2, 3)),              # D = 64; 2 + 2 + 1, 3 + 2
])
def test_step_host_equals_device_path(name, B, H, D, lat, k, pp, chunks):
    cfg = synth.small_config(name, B, H, D, lat, k, pp)
    x, p, t = gpu_inputs(cfg)
    ref = _device_step(x, p, t)
    host = {n: x[n].contiguous().pin_memory() for n in ("q", "k", "v", "do")}
    for c in chunks:
        ws = torch.empty(sa.step_host_workspace_size(p, c), dtype=torch.uint8, device="cuda")
        got = sa.step_host(host["q"], host["k"], host["v"], host["do"], p, c, ws=ws)
        torch.cuda.synchronize()
        assert sa.device_status(ws) == 0
        for name_, g, r in zip(("out", "dq", "dk", "dv"), got, ref):
            assert g.dtype == r.dtype and g.shape == r.shape
            assert torch.equal(g, r), (c, name_, float((g.float() - r.float()).abs().max()))


def test_step_host_twice_and_on_a_side_stream():
    cfg = synth.small_config("sh_rep", 1, 4, 128, (8, 12, 8), 3, 0.9)
    x, p, t = gpu_inputs(cfg)
    ref = _device_step(x, p, t)
    host = {n: x[n].contiguous().pin_memory() for n in ("q", "k", "v", "do")}
    s = torch.cuda.Stream()
    ws = torch.empty(sa.step_host_workspace_size(p, 2), dtype=torch.uint8, device="cuda")
    outs = [torch.empty_like(r).pin_memory() for r in ref]
    for _ in range(2):  # the same buffers again: the second call starts after the first on the stream
        sa.step_host(host["q"], host["k"], host["v"], host["do"], p, 2, *outs, ws=ws, stream=s)
    s.synchronize()
    for g, r in zip(outs, ref):
        assert torch.equal(g, r)


def test_step_host_rejects_bad_host_tensors():
    cfg = synth.small_config("sh_bad", 1, 2, 64, (8, 8, 8), 2, 0.9)
    x, p, _ = gpu_inputs(cfg)
    q = x["q"].contiguous()
    with pytest.raises(ValueError):
        sa.step_host(q.cuda(), q, q, q, p, 1)                       # a device tensor
    with pytest.raises(ValueError):
        sa.step_host(q.float(), q, q, q, p, 1)                      # not bf16
    with pytest.raises(ValueError):
        sa.step_host(q[:, :1], q, q, q, p, 1)                       # wrong shape
