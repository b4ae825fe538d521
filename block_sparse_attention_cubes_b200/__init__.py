"""Cube-routed block-sparse attention for B200 (sm_100a): thin Python binding of libsa.

Every step of the path runs in the CUDA kernels of ``libsa.so``; this module only
marshals arguments (device pointers, sizes, the current CUDA stream) and allocates
outputs and workspaces with torch.  There is no CPU fallback: importing works without
a GPU, but every compute call needs the built library and a CUDA device.

Entry points mirror the C ABI in ``include/sa.h``:

* :func:`plan`      router -> ``kv_index [B,H,T,cap]``, ``kv_count [B,H,T]``
* :func:`forward`   fine stage -> ``out [B,H,Npad,D]`` bf16, ``lse [B,H,Npad]`` fp32
* :func:`backward`  -> ``dq, dk, dv`` fp32
* :func:`tile` / :func:`untile`  latent order <-> cube-major padded order
* :func:`plan_coarse`     router + coarse branch -> lists and a :class:`Coarse`
* :func:`forward_gated`   fine stage, then ``O = G * Repeat(Oc) + O_f``
* :func:`backward_gated`  -> ``dq, dk, dv`` (fine + coarse) and ``dgate``
* :func:`recall`          router recall diagnostic from two forward lse's
* :func:`plan_bq128`      router with 128-token query blocks (cube pairs)
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsa.so")

SA_OK = 0
STATUS_NAMES = {0: "SA_OK", 1: "SA_ERR_INVALID_ARG", 2: "SA_ERR_UNSUPPORTED", 3: "SA_ERR_ALIGNMENT",
                4: "SA_ERR_CAPACITY", 5: "SA_ERR_WORKSPACE", 6: "SA_ERR_LAUNCH", 7: "SA_ERR_DEVICE_TIMEOUT",
                8: "SA_ERR_DEVICE_INDEX"}
OP_PLAN, OP_FORWARD, OP_BACKWARD, OP_PLAN_COARSE, OP_BACKWARD_GATED, OP_PLAN_BQ128, OP_BLOCK_MASS = 0, 1, 2, 3, 4, 5, 6
BF16, FP8_E4M3 = 0, 1
DEBUG_SKIP_LOADS = 1
DEBUG_ROUTER_FALLBACK = 2
DEBUG_CTA_CLOCKS = 4
DEBUG_STATIC_ITEMS = 8

# every symbol include/sa.h declares
EXPORTS = ("sa_padded_tokens", "sa_num_cubes", "sa_topk_from_fraction", "sa_workspace_size", "sa_tile",
           "sa_untile", "sa_plan", "sa_forward", "sa_backward", "sa_get_device_status", "sa_status_string",
           "sa_last_launch_count", "sa_plan_static", "sa_plan_coarse", "sa_forward_gated", "sa_backward_gated", "sa_recall", "sa_plan_bq128",
           "sa_plan_fallback_rows", "sa_tile_rope", "sa_untile_rope", "sa_block_mass", "sa_best_recall",
           "sa_plan_fine_workspace_size", "sa_plan_fine", "sa_get_cta_clocks", "sa_step_host_workspace_size",
           "sa_step_host")


class SAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("D", ctypes.c_int),
                ("lat_t", ctypes.c_int), ("lat_h", ctypes.c_int), ("lat_w", ctypes.c_int),
                ("top_k", ctypes.c_int), ("top_p", ctypes.c_float), ("kv_capacity", ctypes.c_int),
                ("qk_dtype", ctypes.c_int), ("softmax_scale", ctypes.c_float),
                ("timeout_ms", ctypes.c_uint), ("debug_flags", ctypes.c_uint)]


class CoarseC(ctypes.Structure):
    _fields_ = [("qbar", ctypes.c_void_p), ("kbar", ctypes.c_void_p), ("vbar", ctypes.c_void_p),
                ("oc", ctypes.c_void_p), ("lse", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libsa.so and declare its signatures.  Raises when the library is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libsa.so not built at {path}; run `python -m block_sparse_attention_cubes_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(Params)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    sig = {
        "sa_padded_tokens": (i32, [P]),
        "sa_num_cubes": (i32, [P]),
        "sa_topk_from_fraction": (i32, [ctypes.c_double, i32]),
        "sa_workspace_size": (sz, [P, i32]),
        "sa_tile": (i32, [vp, vp, P, i32, vp]),
        "sa_untile": (i32, [vp, vp, P, i32, vp]),
        "sa_plan": (i32, [vp, vp, vp, vp, P, vp, vp, vp, sz, vp]),
        "sa_forward": (i32, [vp, vp, vp, vp, vp, vp, vp, P, vp, vp, vp, vp, sz, vp]),
        "sa_backward": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, vp, P, vp, vp, vp, vp, sz, vp]),
        "sa_get_device_status": (i32, [vp, vp]),
        "sa_status_string": (ctypes.c_char_p, [i32]),
        "sa_last_launch_count": (i32, []),
        "sa_plan_static": (i32, [vp, vp, vp, vp, P, vp, vp, vp]),
        "sa_plan_coarse": (i32, [vp, vp, vp, P, vp, vp, ctypes.POINTER(CoarseC), vp, sz, vp]),
        "sa_forward_gated": (i32, [vp, vp, vp, vp, vp, P, ctypes.POINTER(CoarseC), vp, vp, vp, vp, vp, sz, vp]),
        "sa_backward_gated": (i32, [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, P, ctypes.POINTER(CoarseC), vp, vp, vp,
                                    vp, vp, sz, vp]),
        "sa_recall": (i32, [vp, vp, P, vp, vp, vp]),
        "sa_plan_bq128": (i32, [vp, vp, P, vp, vp, vp, sz, vp]),
        "sa_plan_fallback_rows": (i32, [vp, vp]),
        "sa_tile_rope": (i32, [vp, vp, P, i32, i32, i32, i32, vp, vp, vp]),
        "sa_untile_rope": (i32, [vp, vp, P, i32, i32, i32, i32, vp, vp, vp]),
        "sa_block_mass": (i32, [vp, vp, vp, P, vp, vp, sz, vp]),
        "sa_best_recall": (i32, [vp, vp, P, vp, vp]),
        "sa_plan_fine_workspace_size": (sz, [P, i32, i32, i32]),
        "sa_plan_fine": (i32, [vp, vp, P, i32, i32, i32, vp, vp, vp, vp, sz, vp]),
        "sa_get_cta_clocks": (i32, [vp, sz, i32, vp, i32, ctypes.POINTER(ctypes.c_int), vp]),
        "sa_step_host_workspace_size": (sz, [P, i32]),
        "sa_step_host": (i32, [vp, vp, vp, vp, P, i32, vp, vp, vp, vp, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    _lib = lib
    return lib


def make_params(B: int, H: int, D: int, lat, top_k: int, top_p: float, kv_capacity: int | None = None,
                qk_dtype: int = BF16, softmax_scale: float = 0.0, timeout_ms: int = 0, debug_flags: int = 0) -> Params:
    lt, lh, lw = lat
    T = math.ceil(lt / 4) * math.ceil(lh / 4) * math.ceil(lw / 4)
    cap = T if kv_capacity is None else kv_capacity
    return Params(B, H, D, lt, lh, lw, top_k, top_p, cap, qk_dtype, softmax_scale, timeout_ms, debug_flags)


def geometry(p: Params):
    """(Npad, T) for the parameters."""
    lib = load_library()
    return lib.sa_padded_tokens(ctypes.byref(p)), lib.sa_num_cubes(ctypes.byref(p))


def workspace_size(p: Params, op: int) -> int:
    return int(load_library().sa_workspace_size(ctypes.byref(p), op))


def last_launch_count() -> int:
    return int(load_library().sa_last_launch_count())


def _torch():
    import torch
    if not torch.cuda.is_available():
        raise RuntimeError("libsa needs a CUDA device; there is no CPU path")
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != SA_OK:
        raise SAError(status, what)


def _contig(t, name, dtype=None, device=None):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return t


def _shape(t, shape, name):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _token_tensor(t, p: Params, name, elem_bytes):
    npad, _ = geometry(p)
    _contig(t, name)
    _shape(t, (p.B, p.H, npad, p.D), name)
    if t.element_size() != elem_bytes:
        raise TypeError(f"{name} must have {elem_bytes}-byte elements")


def new_workspace(p: Params, op: int, device=None):
    torch = _torch()
    return torch.empty(max(workspace_size(p, op), 256), dtype=torch.uint8, device=device or "cuda")


def device_status(ws, stream=None) -> int:
    """Synchronise the stream and return the status recorded in the workspace (0 = SA_OK)."""
    return int(load_library().sa_get_device_status(_ptr(ws), _stream(stream)))


def cta_clocks(ws, kernel: int, stream=None):
    """Per-CTA records ``[n, 4]`` uint64 (start ns, end ns, items, steps) of attention kernel
    ``kernel`` (0 forward, 1 dQ, 2 dK/dV) from the last call on workspace ``ws`` made with
    ``DEBUG_CTA_CLOCKS``; synchronises the stream."""
    import numpy as np
    out = np.zeros((1024, 4), dtype=np.uint64)
    n = ctypes.c_int(0)
    _check(load_library().sa_get_cta_clocks(_ptr(ws), ws.numel(), int(kernel), out.ctypes.data, 1024,
                                            ctypes.byref(n), _stream(stream)), "sa_get_cta_clocks")
    return out[:n.value].copy()


def plan_fallback_rows(ws, stream=None) -> int:
    """Synchronise the stream and return how many rows the last :func:`plan` on workspace
    ``ws`` decided on its fp64 path (rows whose tensor-core decision was within the error
    bounds of changing)."""
    n = int(load_library().sa_plan_fallback_rows(_ptr(ws), _stream(stream)))
    if n < 0:
        raise SAError(6, "sa_plan_fallback_rows")
    return n


def tile(x, p: Params, out=None, stream=None):
    """Latent ``[B,H,L,D]`` -> cube-major ``[B,H,Npad,D]`` (same dtype, padding zero)."""
    torch = _torch()
    _contig(x, "x")
    npad, _ = geometry(p)
    if out is None:
        out = torch.empty((p.B, p.H, npad, x.shape[-1]), dtype=x.dtype, device=x.device)
    q = Params.from_buffer_copy(p)
    q.D = x.shape[-1]
    _check(load_library().sa_tile(_ptr(x), _ptr(out), ctypes.byref(q), x.element_size(), _stream(stream)), "sa_tile")
    return out


def _rope_tables(p: Params, sections, rope_cos, rope_sin, device):
    torch = _torch()
    dt, dh, dw = sections
    n = p.lat_t * (dt // 2) + p.lat_h * (dh // 2) + p.lat_w * (dw // 2)
    for t, name in ((rope_cos, "rope_cos"), (rope_sin, "rope_sin")):
        _contig(t, name, torch.float32)
        if t.numel() != n or t.device != device:
            raise ValueError(f"{name} must hold {n} fp32 values on {device}")


def tile_rope(x, p: Params, sections, rope_cos, rope_sin, out=None, stream=None):
    """Latent ``[B,H,L,D]`` -> cube-major ``[B,H,Npad,D]`` with each token rotated by its 3-D
    RoPE angles (``sections`` = (d_t, d_h, d_w); tables as in ``sa_tile_rope``)."""
    torch = _torch()
    _contig(x, "x")
    npad, _ = geometry(p)
    _rope_tables(p, sections, rope_cos, rope_sin, x.device)
    if out is None:
        out = torch.empty((p.B, p.H, npad, x.shape[-1]), dtype=x.dtype, device=x.device)
    q = Params.from_buffer_copy(p)
    q.D = x.shape[-1]
    _check(load_library().sa_tile_rope(_ptr(x), _ptr(out), ctypes.byref(q), x.element_size(), *sections,
                                       _ptr(rope_cos), _ptr(rope_sin), _stream(stream)), "sa_tile_rope")
    return out


def untile_rope(y, p: Params, sections, rope_cos, rope_sin, out=None, stream=None):
    """Inverse of :func:`tile_rope`: cube-major -> latent order with the inverse rotation."""
    torch = _torch()
    _contig(y, "y")
    L = p.lat_t * p.lat_h * p.lat_w
    _rope_tables(p, sections, rope_cos, rope_sin, y.device)
    if out is None:
        out = torch.empty((p.B, p.H, L, y.shape[-1]), dtype=y.dtype, device=y.device)
    q = Params.from_buffer_copy(p)
    q.D = y.shape[-1]
    _check(load_library().sa_untile_rope(_ptr(y), _ptr(out), ctypes.byref(q), y.element_size(), *sections,
                                         _ptr(rope_cos), _ptr(rope_sin), _stream(stream)), "sa_untile_rope")
    return out


def untile(y, p: Params, out=None, stream=None):
    torch = _torch()
    _contig(y, "y")
    L = p.lat_t * p.lat_h * p.lat_w
    if out is None:
        out = torch.empty((p.B, p.H, L, y.shape[-1]), dtype=y.dtype, device=y.device)
    q = Params.from_buffer_copy(p)
    q.D = y.shape[-1]
    _check(load_library().sa_untile(_ptr(y), _ptr(out), ctypes.byref(q), y.element_size(), _stream(stream)),
           "sa_untile")
    return out


def _router_args(q, k, p: Params, q_scale, k_scale, kv_index, kv_count):
    """Checks shared by the routers before anything reaches the library: token tensors,
    caller-given output buffers (int32, contiguous, [B,H,T,cap] / [B,H,T], on q's device)
    and, for e4m3 Q/K, the per-cube fp32 scales [B,H,T] on q's device."""
    torch = _torch()
    eb = 1 if p.qk_dtype == FP8_E4M3 else 2
    _token_tensor(q, p, "q", eb)
    _token_tensor(k, p, "k", eb)
    _, T = geometry(p)
    dev = q.device
    if k.device != dev:
        raise ValueError("q and k must be on the same device")
    for t, name, shape in ((kv_index, "kv_index", (p.B, p.H, T, p.kv_capacity)), (kv_count, "kv_count", (p.B, p.H, T))):
        if t is None:
            continue
        _contig(t, name, torch.int32)
        _shape(t, shape, name)
        if t.device != dev:
            raise ValueError(f"{name} must be on {dev}")
    if p.qk_dtype == FP8_E4M3:
        for t, name in ((q_scale, "q_scale"), (k_scale, "k_scale")):
            if t is None:
                raise ValueError(f"{name} is required for e4m3 Q/K")
            _contig(t, name, torch.float32)
            _shape(t, (p.B, p.H, T), name)
            if t.device != dev:
                raise ValueError(f"{name} must be on {dev}")
    return T, dev


def plan(q, k, p: Params, q_scale=None, k_scale=None, kv_index=None, kv_count=None, ws=None, stream=None):
    """Router: returns (kv_index [B,H,T,cap] int32, kv_count [B,H,T] int32)."""
    torch = _torch()
    T, dev = _router_args(q, k, p, q_scale, k_scale, kv_index, kv_count)
    if kv_index is None:
        kv_index = torch.empty((p.B, p.H, T, p.kv_capacity), dtype=torch.int32, device=dev)
    if kv_count is None:
        kv_count = torch.empty((p.B, p.H, T), dtype=torch.int32, device=dev)
    if ws is None:
        ws = new_workspace(p, OP_PLAN, dev)
    st = load_library().sa_plan(_ptr(q), _ptr(k), _ptr(q_scale), _ptr(k_scale), ctypes.byref(p), _ptr(kv_index),
                                _ptr(kv_count), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "sa_plan")
    return kv_index, kv_count


def plan_static(q, k, p: Params, kv_index, kv_count, q_scale=None, k_scale=None, stream=None):
    """Router with the library's fixed 64 MiB scratch instead of a workspace (see
    ``sa_plan_static`` in include/sa.h).  Outputs are caller-provided; nothing is allocated."""
    if kv_index is None or kv_count is None:
        raise ValueError("plan_static writes into caller-given kv_index and kv_count")
    _router_args(q, k, p, q_scale, k_scale, kv_index, kv_count)
    st = load_library().sa_plan_static(_ptr(q), _ptr(k), _ptr(q_scale), _ptr(k_scale), ctypes.byref(p),
                                       _ptr(kv_index), _ptr(kv_count), _stream(stream))
    _check(st, "sa_plan_static")
    return kv_index, kv_count


def forward(q, k, v, kv_index, kv_count, p: Params, q_scale=None, k_scale=None, out=None, lse=None, ws=None,
            stream=None, with_f32: bool = False, out_f32=None):
    """Fine stage forward: returns (out [B,H,Npad,D] bf16, lse [B,H,Npad] fp32), plus the
    fp32 copy of out as a third element when ``with_f32`` is set (for an exact backward)."""
    torch = _torch()
    npad, T = geometry(p)
    eb = 1 if p.qk_dtype == FP8_E4M3 else 2
    _token_tensor(q, p, "q", eb)
    _token_tensor(k, p, "k", eb)
    _token_tensor(v, p, "v", 2)
    _contig(kv_index, "kv_index", torch.int32)
    _contig(kv_count, "kv_count", torch.int32)
    _shape(kv_index, (p.B, p.H, T, p.kv_capacity), "kv_index")
    _shape(kv_count, (p.B, p.H, T), "kv_count")
    dev = q.device
    if out is None:
        out = torch.empty((p.B, p.H, npad, p.D), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((p.B, p.H, npad), dtype=torch.float32, device=dev)
    if with_f32 and out_f32 is None:
        out_f32 = torch.empty((p.B, p.H, npad, p.D), dtype=torch.float32, device=dev)
    if ws is None:
        ws = new_workspace(p, OP_FORWARD, dev)
    st = load_library().sa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(q_scale), _ptr(k_scale), _ptr(kv_index),
                                   _ptr(kv_count), ctypes.byref(p), _ptr(out), _ptr(lse), _ptr(out_f32), _ptr(ws),
                                   ws.numel(), _stream(stream))
    _check(st, "sa_forward")
    return (out, lse, out_f32) if with_f32 else (out, lse)


def backward(q, k, v, out, lse, dout, kv_index, kv_count, p: Params, dq=None, dk=None, dv=None, ws=None,
             stream=None, out_f32=None):
    """Fine stage backward: returns (dq, dk, dv), each [B,H,Npad,D] fp32.  Pass the
    forward's ``out_f32`` to take Delta = rowsum(dO * O) from the unrounded output."""
    torch = _torch()
    npad, T = geometry(p)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _token_tensor(t, p, n, 2)
    if out_f32 is not None:
        _token_tensor(out_f32, p, "out_f32", 4)
    _contig(lse, "lse", torch.float32)
    _shape(lse, (p.B, p.H, npad), "lse")
    _contig(kv_index, "kv_index", torch.int32)
    _contig(kv_count, "kv_count", torch.int32)
    _shape(kv_index, (p.B, p.H, T, p.kv_capacity), "kv_index")
    _shape(kv_count, (p.B, p.H, T), "kv_count")
    dev = q.device
    shape = tuple(q.shape)
    dq = torch.empty(shape, dtype=torch.float32, device=dev) if dq is None else dq
    dk = torch.empty(shape, dtype=torch.float32, device=dev) if dk is None else dk
    dv = torch.empty(shape, dtype=torch.float32, device=dev) if dv is None else dv
    if ws is None:
        ws = new_workspace(p, OP_BACKWARD, dev)
    st = load_library().sa_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(out_f32), _ptr(lse), _ptr(dout),
                                    _ptr(kv_index),
                                    _ptr(kv_count), ctypes.byref(p), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                                    ws.numel(), _stream(stream))
    _check(st, "sa_backward")
    return dq, dk, dv


@dataclass
class Coarse:
    """Cube-level tensors of the coarse branch, fp32: qbar, kbar, vbar, oc ``[B,H,T,D]`` and
    lse ``[B,H,T]`` (written by :func:`plan_coarse`, read by the gated backward)."""
    qbar: object
    kbar: object
    vbar: object
    oc: object
    lse: object

    @classmethod
    def empty(cls, p: Params, device=None):
        torch = _torch()
        _, T = geometry(p)
        f = lambda *shape: torch.empty(shape, dtype=torch.float32, device=device or "cuda")
        return cls(f(p.B, p.H, T, p.D), f(p.B, p.H, T, p.D), f(p.B, p.H, T, p.D), f(p.B, p.H, T, p.D),
                   f(p.B, p.H, T))

    def c_struct(self, p: Params) -> CoarseC:
        torch = _torch()
        _, T = geometry(p)
        for n in ("qbar", "kbar", "vbar", "oc"):
            t = getattr(self, n)
            _contig(t, n, torch.float32)
            _shape(t, (p.B, p.H, T, p.D), n)
        _contig(self.lse, "lse", torch.float32)
        _shape(self.lse, (p.B, p.H, T), "lse")
        return CoarseC(*(t.data_ptr() for t in (self.qbar, self.kbar, self.vbar, self.oc, self.lse)))


def _gate_tensor(gate, p: Params, name="gate"):
    torch = _torch()
    npad, _ = geometry(p)
    _contig(gate, name, torch.float32)
    _shape(gate, (p.B, p.H, npad), name)


def plan_coarse(q, k, v, p: Params, kv_index=None, kv_count=None, coarse=None, ws=None, stream=None):
    """Router and coarse branch in one call: returns (kv_index, kv_count, :class:`Coarse`)."""
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _token_tensor(t, p, n, 2)
    _, T = geometry(p)
    dev = q.device
    if kv_index is None:
        kv_index = torch.empty((p.B, p.H, T, p.kv_capacity), dtype=torch.int32, device=dev)
    if kv_count is None:
        kv_count = torch.empty((p.B, p.H, T), dtype=torch.int32, device=dev)
    if coarse is None:
        coarse = Coarse.empty(p, dev)
    if ws is None:
        ws = new_workspace(p, OP_PLAN_COARSE, dev)
    cs = coarse.c_struct(p)
    st = load_library().sa_plan_coarse(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(p), _ptr(kv_index), _ptr(kv_count),
                                       ctypes.byref(cs), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "sa_plan_coarse")
    return kv_index, kv_count, coarse


def forward_gated(q, k, v, kv_index, kv_count, p: Params, coarse: Coarse, gate, out=None, lse=None, ws=None,
                  stream=None, out_f32=None):
    """Fine stage then ``O = G * Repeat(Oc) + O_f``; returns (out, lse, out_f32).  The fp32
    copy is always produced (the library forms the sum in fp32)."""
    torch = _torch()
    npad, T = geometry(p)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _token_tensor(t, p, n, 2)
    _gate_tensor(gate, p)
    _contig(kv_index, "kv_index", torch.int32)
    _contig(kv_count, "kv_count", torch.int32)
    _shape(kv_index, (p.B, p.H, T, p.kv_capacity), "kv_index")
    _shape(kv_count, (p.B, p.H, T), "kv_count")
    dev = q.device
    if out is None:
        out = torch.empty((p.B, p.H, npad, p.D), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((p.B, p.H, npad), dtype=torch.float32, device=dev)
    if out_f32 is None:
        out_f32 = torch.empty((p.B, p.H, npad, p.D), dtype=torch.float32, device=dev)
    if ws is None:
        ws = new_workspace(p, OP_FORWARD, dev)
    cs = coarse.c_struct(p)
    st = load_library().sa_forward_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_index), _ptr(kv_count), ctypes.byref(p),
                                         ctypes.byref(cs), _ptr(gate), _ptr(out), _ptr(lse), _ptr(out_f32), _ptr(ws),
                                         ws.numel(), _stream(stream))
    _check(st, "sa_forward_gated")
    return out, lse, out_f32


def backward_gated(q, k, v, out, lse, dout, gate, kv_index, kv_count, p: Params, coarse: Coarse, dq=None, dk=None,
                   dv=None, dgate=None, ws=None, stream=None, out_f32=None):
    """Gradients of the gated output: returns (dq, dk, dv, dgate), fp32.  ``out_f32`` (the fp32
    copy from :func:`forward_gated` with ``with_f32=True``) is required by the library."""
    torch = _torch()
    npad, T = geometry(p)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _token_tensor(t, p, n, 2)
    if out_f32 is not None:
        _token_tensor(out_f32, p, "out_f32", 4)
    _gate_tensor(gate, p)
    _contig(lse, "lse", torch.float32)
    _shape(lse, (p.B, p.H, npad), "lse")
    _contig(kv_index, "kv_index", torch.int32)
    _contig(kv_count, "kv_count", torch.int32)
    _shape(kv_index, (p.B, p.H, T, p.kv_capacity), "kv_index")
    _shape(kv_count, (p.B, p.H, T), "kv_count")
    dev = q.device
    shape = tuple(q.shape)
    dq = torch.empty(shape, dtype=torch.float32, device=dev) if dq is None else dq
    dk = torch.empty(shape, dtype=torch.float32, device=dev) if dk is None else dk
    dv = torch.empty(shape, dtype=torch.float32, device=dev) if dv is None else dv
    dgate = torch.empty((p.B, p.H, npad), dtype=torch.float32, device=dev) if dgate is None else dgate
    if ws is None:
        ws = new_workspace(p, OP_BACKWARD_GATED, dev)
    cs = coarse.c_struct(p)
    st = load_library().sa_backward_gated(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(out_f32), _ptr(lse), _ptr(dout),
                                          _ptr(gate), _ptr(kv_index), _ptr(kv_count), ctypes.byref(p),
                                          ctypes.byref(cs), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dgate), _ptr(ws),
                                          ws.numel(), _stream(stream))
    _check(st, "sa_backward_gated")
    return dq, dk, dv, dgate


def plan_bq128(q, k, p: Params, kv_index=None, kv_count=None, ws=None, stream=None):
    """Router with 128-token query blocks (cube pairs): per-cube lists like :func:`plan`, both
    cubes of a block holding the block's list."""
    torch = _torch()
    _token_tensor(q, p, "q", 2)
    _token_tensor(k, p, "k", 2)
    _, T = geometry(p)
    dev = q.device
    if kv_index is None:
        kv_index = torch.empty((p.B, p.H, T, p.kv_capacity), dtype=torch.int32, device=dev)
    if kv_count is None:
        kv_count = torch.empty((p.B, p.H, T), dtype=torch.int32, device=dev)
    if ws is None:
        ws = new_workspace(p, OP_PLAN_BQ128, dev)
    st = load_library().sa_plan_bq128(_ptr(q), _ptr(k), ctypes.byref(p), _ptr(kv_index), _ptr(kv_count), _ptr(ws),
                                      ws.numel(), _stream(stream))
    _check(st, "sa_plan_bq128")
    return kv_index, kv_count


def recall(lse_kept, lse_all, p: Params, stream=None):
    """Router recall: (tau per token [B,H,Npad], its mean per query cube [B,H,T]), fp32, with
    tau = exp(lse_kept - lse_all) (lse of :func:`forward` on the router's lists and on lists
    holding every block)."""
    torch = _torch()
    npad, T = geometry(p)
    for t, n in ((lse_kept, "lse_kept"), (lse_all, "lse_all")):
        _contig(t, n, torch.float32)
        _shape(t, (p.B, p.H, npad), n)
    tau = torch.empty((p.B, p.H, npad), dtype=torch.float32, device=lse_kept.device)
    cube = torch.empty((p.B, p.H, T), dtype=torch.float32, device=lse_kept.device)
    st = load_library().sa_recall(_ptr(lse_kept), _ptr(lse_all), ctypes.byref(p), _ptr(tau), _ptr(cube),
                                  _stream(stream))
    _check(st, "sa_recall")
    return tau, cube


def plan_fine(q, k, p: Params, R=(2, 2, 2), kv_index=None, kv_count=None, with_scores: bool = False, ws=None,
              stream=None):
    """VSA2's fine-grained router with per-sequence Top-K (``p.top_k`` blocks per query cube on
    average): returns (kv_index, kv_count), plus P_r ``[B,H,T,T]`` fp32 when ``with_scores``."""
    torch = _torch()
    T, dev = _router_args(q, k, p, None, None, kv_index, kv_count)
    if kv_index is None:
        kv_index = torch.empty((p.B, p.H, T, p.kv_capacity), dtype=torch.int32, device=dev)
    if kv_count is None:
        kv_count = torch.empty((p.B, p.H, T), dtype=torch.int32, device=dev)
    pr = torch.empty((p.B, p.H, T, T), dtype=torch.float32, device=dev) if with_scores else None
    lib = load_library()
    if ws is None:
        n = int(lib.sa_plan_fine_workspace_size(ctypes.byref(p), *R))
        if n == 0:
            raise SAError(2, "sa_plan_fine_workspace_size")
        ws = torch.empty(n, dtype=torch.uint8, device=dev)
    _check(lib.sa_plan_fine(_ptr(q), _ptr(k), ctypes.byref(p), *R, _ptr(kv_index), _ptr(kv_count), _ptr(pr),
                            _ptr(ws), ws.numel(), _stream(stream)), "sa_plan_fine")
    return (kv_index, kv_count, pr) if with_scores else (kv_index, kv_count)


def block_mass(q, k, lse_all, p: Params, ws=None, stream=None):
    """P_oracle ``[B,H,T,T]`` fp32: the token-level softmax mass per (query cube, key cube),
    averaged over the query cube's valid tokens (``lse_all``: lse of :func:`forward` on lists
    holding every block)."""
    torch = _torch()
    npad, T = geometry(p)
    _token_tensor(q, p, "q", 2)
    _token_tensor(k, p, "k", 2)
    _contig(lse_all, "lse_all", torch.float32)
    _shape(lse_all, (p.B, p.H, npad), "lse_all")
    out = torch.empty((p.B, p.H, T, T), dtype=torch.float32, device=q.device)
    if ws is None:
        ws = new_workspace(p, OP_BLOCK_MASS, q.device)
    _check(load_library().sa_block_mass(_ptr(q), _ptr(k), _ptr(lse_all), ctypes.byref(p), _ptr(out), _ptr(ws),
                                        ws.numel(), _stream(stream)), "sa_block_mass")
    return out


def best_recall(pblock, kv_count, p: Params, stream=None):
    """``[B,H,T]`` fp32: the sum of the kv_count largest entries of each row of ``pblock``."""
    torch = _torch()
    _, T = geometry(p)
    _contig(pblock, "pblock", torch.float32)
    _shape(pblock, (p.B, p.H, T, T), "pblock")
    _contig(kv_count, "kv_count", torch.int32)
    _shape(kv_count, (p.B, p.H, T), "kv_count")
    out = torch.empty((p.B, p.H, T), dtype=torch.float32, device=pblock.device)
    _check(load_library().sa_best_recall(_ptr(pblock), _ptr(kv_count), ctypes.byref(p), _ptr(out), _stream(stream)),
           "sa_best_recall")
    return out


def step_host_workspace_size(p: Params, chunk_heads: int) -> int:
    return int(load_library().sa_step_host_workspace_size(ctypes.byref(p), int(chunk_heads)))


def step_host(q, k, v, dout, p: Params, chunk_heads: int, out=None, dq=None, dk=None, dv=None, ws=None,
              stream=None):
    """One step (layout, router, forward, backward, layout back) from and to HOST memory with
    the copies overlapped with the work, ``chunk_heads`` (batch, head) problems at a time
    (``sa_step_host``).  q, k, v, dout: CPU ``[B,H,L,D]`` bf16 in latent order, best pinned;
    returns CPU ``(out bf16, dq, dk, dv fp32)``, each ``[B,H,L,D]``.  The results are final
    once ``stream`` (default: the current one) has been synchronised."""
    torch = _torch()
    L = p.lat_t * p.lat_h * p.lat_w
    shape = (p.B, p.H, L, p.D)
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (dout, "dout")):
        if t.is_cuda or not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be a contiguous CPU bf16 tensor")
        _shape(t, shape, name)
    def host_out(t, name, dtype):
        if t is None:
            return torch.empty(shape, dtype=dtype).pin_memory()
        if t.is_cuda or not t.is_contiguous() or t.dtype != dtype:
            raise ValueError(f"{name} must be a contiguous CPU {dtype} tensor")
        _shape(t, shape, name)
        return t
    out = host_out(out, "out", torch.bfloat16)
    dq, dk, dv = (host_out(t, n, torch.float32) for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")))
    need = step_host_workspace_size(p, chunk_heads)
    if need == 0:
        raise SAError(1, "sa_step_host_workspace_size")
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        if stream is not None:  # the allocator hands this memory out again only after `stream`'s work
            ws.record_stream(stream)
    _contig(ws, "ws", torch.uint8)
    _check(load_library().sa_step_host(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), ctypes.byref(p), int(chunk_heads),
                                       _ptr(out), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                                       _stream(stream)), "sa_step_host")
    return out, dq, dk, dv


@dataclass
class Attention:
    """Router + fine stage with buffers kept between calls (one layer's worth)."""
    params: Params

    def __post_init__(self):
        self._ws = {}

    def _w(self, op, dev):
        if op not in self._ws:
            self._ws[op] = new_workspace(self.params, op, dev)
        return self._ws[op]

    def plan(self, q, k, q_scale=None, k_scale=None):
        return plan(q, k, self.params, q_scale, k_scale, ws=self._w(OP_PLAN, q.device))

    def forward(self, q, k, v, kv_index, kv_count, q_scale=None, k_scale=None, with_f32=True):
        """Returns (out, lse, out_f32) (out_f32 is None when ``with_f32`` is False)."""
        r = forward(q, k, v, kv_index, kv_count, self.params, q_scale, k_scale, ws=self._w(OP_FORWARD, q.device),
                    with_f32=with_f32)
        return r if with_f32 else (r[0], r[1], None)

    def backward(self, q, k, v, out, lse, dout, kv_index, kv_count, out_f32=None):
        return backward(q, k, v, out, lse, dout, kv_index, kv_count, self.params, ws=self._w(OP_BACKWARD, q.device),
                        out_f32=out_f32)
