"""sa_tile_rope / sa_untile_rope against the oracle's 3-D RoPE with the cube-major permutation
(GPU, through the C ABI).  Both sides take the same fp32 cosine and sine tables (RoFormer's
frequencies); the CUDA path rotates in fp32 and rounds to the element type, so bf16 outputs
are compared within half a bf16 ulp (at most 2^-8 of the value, just above a power of two)
plus the fp32 rotation's error, fp32 outputs within 1e-6 relative."""
import numpy as np
import pytest
import torch

import block_sparse_attention_cubes_b200 as sa
import oracle as O
from oracle import rope as R

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu(cuda_ok):
    from block_sparse_attention_cubes_b200 import build
    build.build()
    yield


CASES = [((5, 6, 7), 128, (32, 48, 48)), ((8, 8, 12), 64, (16, 24, 24)), ((21, 9, 13), 128, (64, 32, 32))]


@pytest.mark.parametrize("lat,D,sec", CASES)
def test_tile_rope_matches_oracle(lat, D, sec):
    B, H = 1, 3
    lay = O.cube_layout(lat)
    L = lat[0] * lat[1] * lat[2]
    g = torch.Generator().manual_seed(7)
    x32 = torch.randn((B, H, L, D), generator=g) * 3.0
    cos, sin = R.rope_tables(lat, sec, base=500.0)
    cs32, sn32 = torch.from_numpy(cos).float(), torch.from_numpy(sin).float()
    p = sa.make_params(B, H, D, lat, 1, 0.5)
    cs_d, sn_d = cs32.cuda(), sn32.cuda()
    for dtype, rel in ((torch.bfloat16, 2.0 ** -8 + 2.0 ** -20), (torch.float32, 1e-6)):
        x = x32.to(dtype)
        y = sa.tile_rope(x.cuda(), p, sec, cs_d, sn_d)
        torch.cuda.synchronize()
        for h in range(H):
            ref = R.tile_rope(x[0, h].double().numpy(), lay, sec, cs32.double().numpy(), sn32.double().numpy())
            got = y[0, h].double().cpu().numpy()
            assert np.all(got[~lay.valid] == 0)
            err = np.abs(got - ref)
            # per pair: the bound scales with the pair's magnitude
            mag = np.repeat(np.hypot(ref[:, 0::2], ref[:, 1::2]), 2, axis=1)
            assert np.all(err <= rel * mag + 1e-30), (dtype, h, float((err / (mag + 1e-30)).max()))
        back = sa.untile_rope(y, p, sec, cs_d, sn_d)
        torch.cuda.synchronize()
        if dtype == torch.float32:
            assert torch.allclose(back.cpu(), x, rtol=0, atol=1e-5 * float(x.abs().max()))


def test_rope_relative_position_on_the_gpu():
    # equal query and key vectors at every token: after rotation, dots depend on offsets only
    lat, D, sec = (6, 5, 7), 64, (16, 24, 24)
    p = sa.make_params(1, 1, D, lat, 1, 0.5)
    L = lat[0] * lat[1] * lat[2]
    g = torch.Generator().manual_seed(1)
    q, k = torch.randn(D, generator=g), torch.randn(D, generator=g)
    cos, sin = R.rope_tables(lat, sec, base=50.0)
    cs, sn = torch.from_numpy(cos).float().cuda(), torch.from_numpy(sin).float().cuda()
    xq = q.expand(1, 1, L, D).contiguous().cuda()
    xk = k.expand(1, 1, L, D).contiguous().cuda()
    lay = O.cube_layout(lat)
    slot = {int(s): i for i, s in enumerate(lay.src) if s >= 0}
    rq = sa.tile_rope(xq, p, sec, cs, sn)[0, 0].double().cpu()
    rk = sa.tile_rope(xk, p, sec, cs, sn)[0, 0].double().cpu()
    idx = lambda t, h, w: slot[(t * lat[1] + h) * lat[2] + w]
    dots = [float(rq[idx(*a)] @ rk[idx(*b)]) for a, b in (((0, 0, 0), (1, 2, 3)), ((2, 1, 1), (3, 3, 4)),
                                                           ((4, 2, 3), (5, 4, 6)))]
    assert max(dots) - min(dots) < 1e-4 * (1 + abs(dots[0]))


def test_rope_host_checks():
    p = sa.make_params(1, 1, 64, (4, 4, 4), 1, 0.5)
    x = torch.zeros((1, 1, 64, 64), dtype=torch.bfloat16, device="cuda")
    t = torch.zeros(4 * 8 + 4 * 8 + 4 * 16, dtype=torch.float32, device="cuda")
    with pytest.raises((ValueError, sa.SAError)):      # sections do not add up to D
        sa.tile_rope(x, p, (16, 16, 30), t, t)
    with pytest.raises((ValueError, sa.SAError)):      # odd section
        sa.tile_rope(x, p, (15, 17, 32), t, t)
