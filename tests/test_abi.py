"""The C ABI library loads and exports every symbol include/sa.h declares; host-side
validation answers without touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_cubes_b200 as sa
from block_sparse_attention_cubes_b200 import build as sa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    sa_build.build()
    return sa.load_library()


def test_header_declares_exactly_the_exports(lib):
    hdr = open(os.path.join(ROOT, "include", "sa.h")).read()
    declared = set(re.findall(r"SA_API\s+[\w\s\*]+?\b(sa_\w+)\s*\(", hdr))
    assert declared == set(sa.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_exported_dynamic_symbols(lib):
    out = os.popen(f"nm -D --defined-only {sa.LIB_PATH}").read()
    for name in sa.EXPORTS:
        assert re.search(rf"\bT {name}\b", out), name


def test_geometry_and_workspace(lib):
    p = sa.make_params(1, 40, 128, (21, 45, 80), 44, 0.9)
    assert sa.geometry(p) == (92160, 1440)
    assert lib.sa_topk_from_fraction(0.03, 1440) == 44
    assert lib.sa_topk_from_fraction(0.03, 1562) == 47
    T, BH = 1440, 40
    plan_ws = sa.workspace_size(p, sa.OP_PLAN)
    # pooled rows (fp64) + their 4 int8 limbs + per-row data + int32 keys
    assert plan_ws >= 256 + 2 * BH * T * 128 * 8 + 2 * BH * 4 * T * 128 + BH * T * T * 4
    # the routers that keep every fp64 score (coarse branch) need the full score matrix
    assert sa.workspace_size(p, sa.OP_PLAN_COARSE) >= 256 + 2 * BH * T * 128 * 8 + BH * T * T * 8
    assert sa.workspace_size(p, sa.OP_FORWARD) >= 256 + 1440 * 8 + 40 * 720 * min(2 * 1440, 1440) * 4  # masks + pair unions
    assert sa.workspace_size(p, sa.OP_BACKWARD) >= BH * 92160 * 4 + BH * T * T * 4


def test_host_validation_without_gpu(lib):
    p = sa.make_params(1, 2, 96, (8, 8, 8), 4, 0.5)          # D = 96 is not built
    assert sa.workspace_size(p, 0) == 0
    bad = ctypes.c_void_p(16)
    st = lib.sa_plan(bad, bad, None, None, ctypes.byref(p), bad, bad, bad, 1 << 20, None)
    assert st == 2  # SA_ERR_UNSUPPORTED, returned before any launch
    p = sa.make_params(1, 2, 64, (8, 8, 8), -1, 0.5)
    assert lib.sa_plan(bad, bad, None, None, ctypes.byref(p), bad, bad, bad, 1 << 20, None) == 1
    p = sa.make_params(1, 2, 64, (8, 8, 8), 4, float("nan"))
    assert lib.sa_plan(bad, bad, None, None, ctypes.byref(p), bad, bad, bad, 1 << 20, None) == 1
    p = sa.make_params(1, 2, 64, (8, 8, 8), 4, 0.5, kv_capacity=9)   # T = 8
    assert lib.sa_plan(bad, bad, None, None, ctypes.byref(p), bad, bad, bad, 1 << 20, None) == 1
    p = sa.make_params(1, 2, 64, (8, 8, 8), 4, 0.5)
    assert lib.sa_plan(None, bad, None, None, ctypes.byref(p), bad, bad, bad, 1 << 20, None) == 1
    odd = ctypes.c_void_p(24)                                    # 8 bytes off a 16-byte boundary
    assert lib.sa_plan(odd, bad, None, None, ctypes.byref(p), bad, bad, bad, 1 << 20, None) == 3
    assert lib.sa_plan(bad, bad, None, None, ctypes.byref(p), bad, bad, bad, 16, None) == 5
    fp8 = sa.make_params(1, 2, 128, (8, 8, 8), 4, 0.5, qk_dtype=sa.FP8_E4M3)
    assert lib.sa_plan(bad, bad, None, None, ctypes.byref(fp8), bad, bad, bad, 1 << 30, None) == 1
    assert lib.sa_status_string(7) == b"a bounded wait inside a kernel timed out"
    assert lib.sa_last_launch_count() == 0


def test_product_path_has_no_cpu_fallback():
    import torch
    if torch.cuda.is_available():
        pytest.skip("GPU present")
    p = sa.make_params(1, 1, 64, (4, 4, 4), 1, 0.5)
    with pytest.raises(RuntimeError):
        sa.plan(torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16), torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16), p)


def test_package_does_not_import_oracle():
    import ast
    pkg = os.path.join(ROOT, "block_sparse_attention_cubes_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            tree = ast.parse(open(os.path.join(pkg, fn)).read())
            for node in ast.walk(tree):
                if isinstance(node, (ast.Import, ast.ImportFrom)):
                    names = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
                    assert not any(n.split(".")[0] == "oracle" for n in names), fn


def test_coarse_entry_points_validate_on_the_host(lib):
    p = sa.make_params(2, 3, 64, (8, 8, 8), 4, 0.5)          # T = 8, B*H = 6
    T, BH, D, npad = 8, 6, 64, 512
    bwd = sa.workspace_size(p, sa.OP_BACKWARD)
    plan64 = 256 + 2 * BH * T * D * 8 + BH * T * T * 8      # status, fp64 Qbar, Kbar and every score
    # fp64 plan + Pc; backward + dOc^, three per-cube terms, delta_c, scores and dS (each 256-byte aligned)
    assert sa.workspace_size(p, sa.OP_PLAN_COARSE) >= plan64 + BH * T * T * 4
    assert sa.workspace_size(p, sa.OP_BACKWARD_GATED) >= bwd + 4 * BH * T * D * 4 + BH * T * 4 + 2 * BH * T * T * 4
    assert sa.workspace_size(p, sa.OP_BLOCK_MASS) == 256 + 256     # status block + cube masks
    assert sa.workspace_size(p, 7) == 0
    bad = ctypes.c_void_p(16)
    c = sa.CoarseC(16, 16, 16, 16, 16)
    cref = ctypes.byref(c)
    # every error below is returned before anything touches the device
    assert lib.sa_plan_coarse(bad, bad, bad, ctypes.byref(p), bad, bad, None, bad, 1 << 30, None) == 1
    assert lib.sa_plan_coarse(bad, bad, None, ctypes.byref(p), bad, bad, cref, bad, 1 << 30, None) == 1
    assert lib.sa_plan_coarse(bad, bad, bad, ctypes.byref(p), bad, bad, cref, bad, 16, None) == 5
    odd = sa.CoarseC(16, 16, 24, 16, 16)
    assert lib.sa_plan_coarse(bad, bad, bad, ctypes.byref(p), bad, bad, ctypes.byref(odd), bad, 1 << 30, None) == 3
    nul = sa.CoarseC(16, 16, 16, None, 16)
    assert lib.sa_plan_coarse(bad, bad, bad, ctypes.byref(p), bad, bad, ctypes.byref(nul), bad, 1 << 30, None) == 1
    fp8 = sa.make_params(2, 3, 128, (8, 8, 8), 4, 0.5, qk_dtype=sa.FP8_E4M3)
    assert lib.sa_plan_coarse(bad, bad, bad, ctypes.byref(fp8), bad, bad, cref, bad, 1 << 30, None) == 2
    # gated forward: gate required; the fine stage's checks follow
    assert lib.sa_forward_gated(bad, bad, bad, bad, bad, ctypes.byref(p), cref, None, bad, bad, None, bad, 1 << 30,
                                None) == 1
    assert lib.sa_forward_gated(bad, bad, bad, bad, bad, ctypes.byref(p), cref, bad, bad, bad, None, bad, 1 << 30,
                                None) == 1                      # out_f32 is required
    assert lib.sa_forward_gated(bad, bad, bad, bad, bad, ctypes.byref(p), cref, bad, bad, bad, bad, bad, 16,
                                None) == 5
    # gated backward: coarse, gate and dgate required, the gated workspace size enforced
    args = [bad] * 10
    assert lib.sa_backward_gated(*args, ctypes.byref(p), None, bad, bad, bad, bad, bad, 1 << 30, None) == 1
    args_nogate = [bad] * 7 + [None] + [bad] * 2
    assert lib.sa_backward_gated(*args_nogate, ctypes.byref(p), cref, bad, bad, bad, bad, bad, 1 << 30, None) == 1
    assert lib.sa_backward_gated(*args, ctypes.byref(p), cref, bad, bad, bad, bad, bad, bwd, None) == 5
    args_no32 = [bad] * 4 + [None] + [bad] * 5                  # out_f32 is required
    assert lib.sa_backward_gated(*args_no32, ctypes.byref(p), cref, bad, bad, bad, bad, bad, 1 << 30, None) == 1
    many = sa.make_params(1, 70000, 64, (4, 4, 4), 1, 0.5)      # B*H above one grid layer per head
    assert lib.sa_plan_coarse(bad, bad, bad, ctypes.byref(many), bad, bad, cref, bad, 1 << 40, None) == 2
    assert lib.sa_last_launch_count() == 0


def test_recall_validates_on_the_host(lib):
    p = sa.make_params(1, 2, 64, (8, 8, 8), 4, 0.5)
    bad = ctypes.c_void_p(16)
    assert lib.sa_recall(bad, bad, ctypes.byref(p), None, None, None) == 1      # no output
    assert lib.sa_recall(None, bad, ctypes.byref(p), bad, bad, None) == 1
    assert lib.sa_recall(bad, ctypes.c_void_p(18), ctypes.byref(p), bad, None, None) == 3
    assert lib.sa_last_launch_count() == 0


def test_plan_bq128_validates_on_the_host(lib):
    p = sa.make_params(1, 2, 64, (8, 8, 12), 4, 0.5)          # T = 12: 6 query blocks
    T, BH, M, D = 12, 2, 6, 64
    plan = 256 + 2 * BH * T * D * 8 + BH * T * T * 8          # status, fp64 Qbar, Kbar and every score
    # the fp64 plan's, then the block means (fp64) and the block lists and counts
    assert sa.workspace_size(p, sa.OP_PLAN_BQ128) >= plan + BH * M * D * 8 + BH * M * (T + 1) * 4
    bad = ctypes.c_void_p(16)
    assert lib.sa_plan_bq128(None, bad, ctypes.byref(p), bad, bad, bad, 1 << 30, None) == 1
    assert lib.sa_plan_bq128(bad, bad, ctypes.byref(p), bad, bad, bad, plan, None) == 5
    fp8 = sa.make_params(1, 2, 128, (8, 8, 12), 4, 0.5, qk_dtype=sa.FP8_E4M3)
    assert lib.sa_plan_bq128(bad, bad, ctypes.byref(fp8), bad, bad, bad, 1 << 30, None) == 2
    many = sa.make_params(1, 70000, 64, (4, 4, 4), 1, 0.5)
    assert lib.sa_plan_bq128(bad, bad, ctypes.byref(many), bad, bad, bad, 1 << 40, None) == 2
    assert lib.sa_last_launch_count() == 0


def test_fine_stage_layout_and_static_plan_validate_on_the_host(lib):
    """Error paths of sa_forward, sa_backward, sa_tile / sa_untile, sa_plan_static and
    sa_get_device_status that return before anything touches the device."""
    p = sa.make_params(1, 2, 64, (8, 8, 8), 4, 0.5)            # T = 8
    P = ctypes.byref(p)
    bad, odd = ctypes.c_void_p(16), ctypes.c_void_p(24)
    big = 1 << 30
    # sa_forward(q, k, v, q_scale, k_scale, kv_index, kv_count, p, out, lse, out_f32, ws, ws_bytes, stream)
    assert lib.sa_forward(bad, bad, None, None, None, bad, bad, P, bad, bad, None, bad, big, None) == 1
    assert lib.sa_forward(bad, bad, odd, None, None, bad, bad, P, bad, bad, None, bad, big, None) == 3
    assert lib.sa_forward(bad, bad, bad, None, None, bad, bad, P, bad, bad, odd, bad, big, None) == 3
    assert lib.sa_forward(bad, bad, bad, None, None, bad, bad, P, bad, bad, None, bad, 16, None) == 5
    f8 = sa.make_params(1, 2, 64, (8, 8, 8), 4, 0.5, qk_dtype=sa.FP8_E4M3)
    assert lib.sa_forward(bad, bad, bad, bad, bad, bad, bad, ctypes.byref(f8), bad, bad, None, bad, big, None) == 2
    f8d = sa.make_params(1, 2, 128, (8, 8, 8), 4, 0.5, qk_dtype=sa.FP8_E4M3)
    assert lib.sa_forward(bad, bad, bad, None, bad, bad, bad, ctypes.byref(f8d), bad, bad, None, bad, big, None) == 1
    # sa_backward(q, k, v, out, out_f32, lse, dout, kv_index, kv_count, p, dq, dk, dv, ws, ws_bytes, stream)
    assert lib.sa_backward(bad, bad, bad, bad, None, bad, bad, bad, bad, P, None, bad, bad, bad, big, None) == 1
    assert lib.sa_backward(bad, bad, bad, bad, None, bad, odd, bad, bad, P, bad, bad, bad, bad, big, None) == 3
    assert lib.sa_backward(bad, bad, bad, bad, None, bad, bad, bad, bad, P, bad, bad, bad, bad, 16, None) == 5
    assert lib.sa_backward(bad, bad, bad, bad, None, bad, bad, bad, bad, ctypes.byref(f8d), bad, bad, bad, bad,
                           big, None) == 2
    # sa_tile / sa_untile(src, dst, p, elem_bytes, stream)
    assert lib.sa_tile(bad, bad, P, 3, None) == 1                # element size not 1, 2 or 4
    assert lib.sa_tile(None, bad, P, 2, None) == 1
    p4 = sa.make_params(1, 2, 4, (8, 8, 8), 4, 0.5)             # 8-byte rows: not a multiple of 16
    assert lib.sa_untile(bad, bad, ctypes.byref(p4), 2, None) == 2
    assert lib.sa_untile(bad, odd, P, 2, None) == 3
    # sa_plan_static(q, k, q_scale, k_scale, p, kv_index, kv_count, stream)
    pc = sa.make_params(1, 2, 64, (8, 8, 8), 4, 0.5, kv_capacity=4)
    assert lib.sa_plan_static(bad, bad, None, None, ctypes.byref(pc), bad, bad, None) == 1   # capacity != T
    assert lib.sa_plan_static(odd, bad, None, None, P, bad, bad, None) == 3
    f8s = sa.make_params(1, 2, 128, (8, 8, 8), 4, 0.5, qk_dtype=sa.FP8_E4M3)
    odd4 = ctypes.c_void_p(18)                                   # fp32 scales must be 4-byte aligned
    assert lib.sa_plan_static(bad, bad, odd4, bad, ctypes.byref(f8s), bad, bad, None) == 3
    assert lib.sa_plan_static(bad, bad, None, bad, ctypes.byref(f8s), bad, bad, None) == 1   # scale missing
    huge = sa.make_params(1, 40, 128, (21, 45, 80), 44, 0.9)   # needs far more than the 64 MiB array
    assert lib.sa_plan_static(bad, bad, None, None, ctypes.byref(huge), bad, bad, None) == 5
    assert lib.sa_get_device_status(None, None) == 1
    assert lib.sa_last_launch_count() == 0


def test_cta_clocks_validate_on_the_host(lib):
    """sa_get_cta_clocks rejects bad arguments before touching the device, and forward and
    backward workspaces carry room for the records (three kernels x 1024 CTAs x 32 bytes)."""
    p = sa.make_params(1, 2, 64, (8, 8, 8), 2, 0.9)
    rec = 3 * 1024 * 32
    assert sa.workspace_size(p, sa.OP_FORWARD) >= 256 + rec
    assert sa.workspace_size(p, sa.OP_BACKWARD) >= 256 + rec
    out = (ctypes.c_ulonglong * 16)()
    n = ctypes.c_int(-1)
    fake = ctypes.c_void_p(16)
    for ws, size, kernel, o, np_ in ((None, 10 ** 6, 0, out, ctypes.byref(n)),      # null workspace
                                     (fake, 10 ** 6, 3, out, ctypes.byref(n)),      # kernel outside 0..2
                                     (fake, 10 ** 6, -1, out, ctypes.byref(n)),
                                     (fake, 256 + rec - 1, 0, out, ctypes.byref(n)),  # too small for the records
                                     (fake, 10 ** 6, 0, None, ctypes.byref(n)),     # null output
                                     (fake, 10 ** 6, 0, out, None)):                # null count
        assert lib.sa_get_cta_clocks(ws, size, kernel, o, 4, np_, None) == 1


def test_step_host_validates_on_the_host(lib):
    """sa_step_host_workspace_size and the error paths of sa_step_host that return before any
    stream, event or copy is made."""
    p = sa.make_params(2, 3, 64, (8, 8, 8), 4, 0.5)            # B*H = 6 problems, T = 8, L = 512
    P = ctypes.byref(p)
    npad, T, L, D = 512, 8, 512, 64
    w1, w2, w6 = (lib.sa_step_host_workspace_size(P, c) for c in (1, 2, 6))
    assert 0 < w1 < w2 < w6
    assert lib.sa_step_host_workspace_size(P, 100) == w6       # chunks never exceed B*H
    assert lib.sa_step_host_workspace_size(P, 0) == 0
    # per problem at least: two slots of latent inputs and outputs, the cube-major tensors, the lists
    per = 2 * 4 * L * D * 2 + 4 * npad * D * 2 + T * T * 4 + npad * D * (2 + 4 + 3 * 4) + 2 * L * D * (2 + 3 * 4)
    assert w2 >= 2 * per + sum(sa.workspace_size(sa.make_params(1, 2, 64, (8, 8, 8), 4, 0.5), op)
                               for op in (sa.OP_PLAN, sa.OP_FORWARD, sa.OP_BACKWARD))
    bad, odd = ctypes.c_void_p(16), ctypes.c_void_p(24)
    # sa_step_host(q, k, v, dout, p, chunk_heads, out, dq, dk, dv, ws, ws_bytes, stream)
    assert lib.sa_step_host(bad, bad, bad, None, P, 2, bad, bad, bad, bad, bad, w2, None) == 1
    assert lib.sa_step_host(bad, bad, bad, bad, P, 0, bad, bad, bad, bad, bad, w2, None) == 1
    assert lib.sa_step_host(bad, bad, bad, bad, P, 2, bad, bad, bad, bad, None, w2, None) == 5
    assert lib.sa_step_host(bad, bad, bad, bad, P, 2, bad, bad, bad, bad, bad, w2 - 1, None) == 5
    assert lib.sa_step_host(bad, bad, bad, bad, P, 2, bad, bad, bad, bad, odd, w2, None) == 3
    f8 = sa.make_params(1, 2, 128, (8, 8, 8), 4, 0.5, qk_dtype=sa.FP8_E4M3)
    assert lib.sa_step_host(bad, bad, bad, bad, ctypes.byref(f8), 1, bad, bad, bad, bad, bad, 1 << 30, None) == 2
    d96 = sa.make_params(1, 2, 96, (8, 8, 8), 4, 0.5)
    assert lib.sa_step_host_workspace_size(ctypes.byref(d96), 1) == 0
    assert lib.sa_step_host(bad, bad, bad, bad, ctypes.byref(d96), 1, bad, bad, bad, bad, bad, 1 << 30, None) == 2
    assert lib.sa_last_launch_count() == 0
