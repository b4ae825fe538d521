"""sa_plan_static, the router entry point that allocates nothing, against sa_plan.

Some callers cannot allocate device memory (a framework recording a CUDA graph, a
server confined to a pre-reserved arena, plain C callers without an allocator); for
them the library keeps its router scratch in a fixed 64 MiB device array.  This test
calls that entry point twice in a row through the C ABI and checks both results
against the workspace-based sa_plan: the outputs are block indices and counts, so
they must be identical.  It lives in its own file, collected last, and passes alone
or after the other tests.
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


@pytest.mark.parametrize("cfg", [synth.get_config("tiny"), synth.get_config("480p"),
                                 synth.small_config("pad", 2, 3, 128, (5, 9, 13), 3, 0.8)],
                         ids=["tiny", "480p", "padded-B2"])
def test_static_plan_matches_workspace_plan_twice(cfg):
    x, p, t = gpu_inputs(cfg, names=("q", "k"))
    ref_idx, ref_cnt = sa.plan(t["q"], t["k"], p)
    used = torch.arange(p.kv_capacity, device="cuda") < ref_cnt[..., None]
    for _ in range(2):
        idx = torch.full_like(ref_idx, -1)
        cnt = torch.full_like(ref_cnt, -1)
        sa.plan_static(t["q"], t["k"], p, idx, cnt)
        torch.cuda.synchronize()
        assert torch.equal(cnt, ref_cnt)
        assert torch.equal(idx[used], ref_idx[used])


def test_static_plan_rejects_too_large_and_clipping():
    cfg = synth.get_config("720p")
    p = sa.make_params(cfg.B, cfg.H, cfg.D, cfg.lat, cfg.top_k, cfg.top_p)
    assert sa.workspace_size(p, sa.OP_PLAN) > (64 << 20)
    q = torch.zeros((1, 40, 92160, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((1, 40, 1440, 1440), dtype=torch.int32, device="cuda")
    cnt = torch.empty((1, 40, 1440), dtype=torch.int32, device="cuda")
    with pytest.raises(sa.SAError) as e:
        sa.plan_static(q, q, p, idx, cnt)
    assert e.value.status == 5            # SA_ERR_WORKSPACE: beyond the fixed scratch
    small = sa.make_params(1, 2, 64, (16, 16, 16), 8, 0.9, kv_capacity=10)
    q2 = torch.zeros((1, 2, 4096, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sa.SAError) as e:
        sa.plan_static(q2, q2, small, torch.empty((1, 2, 64, 10), dtype=torch.int32, device="cuda"),
                       torch.empty((1, 2, 64), dtype=torch.int32, device="cuda"))
    assert e.value.status == 1            # kv_capacity must equal T
