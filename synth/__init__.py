"""Seeded synthetic inputs shaped like Wan2.1 video-DiT attention activations.

This module holds no step of the attention method: it only draws numbers.  It is
shared by the tests, the oracle harness and ``bench.py`` so that every side sees
the same bf16 bits.  Tensors come out in *latent* (row-major t, h, w) token
order, shape ``[B, H, L, D]`` with ``L = lat_t * lat_h * lat_w``; moving them
to cube-major order is a step of the method and each side does it itself.

Recipe (per batch b, head h, tensor X in {q, k, v, do}):

* ``noise = N(0, 1)`` drawn from a Philox counter generator keyed by
  ``SeedSequence([seed, tensor_id, b, h])``.
* A smooth positional term ``phi_c(t,h,w) = sqrt(2) * sin(2*pi*(f_c . (t/T, h/H, w/W)) + theta_c)``
  with one integer frequency vector ``f_c in {0,1,2}^3 \\ {0}`` and one phase
  ``theta_c ~ U[0, 2*pi)`` per channel c, drawn from ``SeedSequence([seed, 100, b, h])``.
  The same phi is used for q, k and v of a head, so pooled q and k of nearby
  cubes correlate and the block scores peak near the diagonal.
* ``q = noise + alpha * phi``, ``k = kscale * (noise + alpha * phi)``,
  ``v = noise + 0.5 * alpha * phi``, ``do = noise``.
* Sink heads multiply the key of latent token 0 by ``sink`` (8 by default).
* Values are rounded fp64 -> fp32 -> bf16, each step round-to-nearest-even.
* Gates of the gated combination (``make_gate``): ``tanh(N(0, 1))`` per cube-major token
  slot, fp32, keyed by ``SeedSequence([seed, 4, b, h])``.

``alpha`` is set per head type ("uniform" or "sink"); for the configurations
with a sparsity target it was calibrated once against the fp64 oracle router
(see ``calibration.json``), so the achieved sparsity is reported, not assumed.
"""
from __future__ import annotations

import json
import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np
import torch

TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "do": 3}
_HERE = os.path.dirname(os.path.abspath(__file__))


@dataclass(frozen=True)
class HeadType:
    name: str          # "uniform" or "sink"
    alpha: float       # amplitude of the positional term
    kscale: float = 1.0
    sink: float = 1.0  # factor on the key of latent token 0


@dataclass(frozen=True)
class Config:
    name: str
    B: int
    H: int
    D: int
    lat: tuple          # (lat_t, lat_h, lat_w)
    top_k: int
    top_p: float
    head_types: tuple   # one HeadType per head
    passes: str         # "fwd" or "fwd+bwd"
    qk_dtype: str = "bf16"   # "bf16" or "fp8_e4m3"
    target_density: float | None = None
    note: str = ""

    @property
    def L(self) -> int:
        return self.lat[0] * self.lat[1] * self.lat[2]


def _calibrated_alpha(cfg_name: str, head_type: str, default: float) -> float:
    path = os.path.join(_HERE, "calibration.json")
    if not os.path.exists(path):
        return default
    with open(path) as f:
        table = json.load(f)
    return float(table.get(cfg_name, {}).get(head_type, default))


def _split_heads(H: int, cfg_name: str, a_uniform: float, a_sink: float):
    au = _calibrated_alpha(cfg_name, "uniform", a_uniform)
    as_ = _calibrated_alpha(cfg_name, "sink", a_sink)
    half = H // 2
    return tuple([HeadType("uniform", au)] * half + [HeadType("sink", as_, sink=8.0)] * (H - half))


def get_config(name: str) -> Config:
    """The five workloads: tiny, 480p, 720p, 720p-fp8, and the 720p sweep point(s)."""
    if name == "tiny":
        return Config("tiny", 1, 2, 64, (16, 16, 16), 8, 0.9,
                      (HeadType("uniform", 1.0, kscale=0.1), HeadType("sink", 1.0, sink=8.0)),
                      "fwd", note="correctness case; no sparsity target")
    if name == "480p":
        return Config("480p", 1, 12, 128, (21, 30, 52), math.ceil(0.03 * 624), 0.9,
                      _split_heads(12, "480p", 1.0, 1.0), "fwd", target_density=0.10)
    if name == "720p":
        return Config("720p", 1, 40, 128, (21, 45, 80), math.ceil(0.03 * 1440), 0.9,
                      _split_heads(40, "720p", 1.0, 1.0), "fwd+bwd", target_density=0.05)
    if name == "720p_fp8":
        return Config("720p_fp8", 1, 40, 128, (21, 45, 80), math.ceil(0.015 * 1440), 0.9,
                      _split_heads(40, "720p_fp8", 1.0, 1.0), "fwd", qk_dtype="fp8_e4m3",
                      target_density=0.03)
    if name.startswith("sweep"):
        # sweep_<p>_<density%>, e.g. sweep_0.9_95 -> p=0.9, alpha calibrated for 95 % sparsity
        _, p, sp = name.split("_")
        dens = 1.0 - float(sp) / 100.0
        return Config(name, 1, 40, 128, (21, 45, 80), 4, float(p),
                      _split_heads(40, f"sweep_{sp}", 1.0, 1.0), "fwd+bwd",
                      target_density=dens)
    raise KeyError(name)


def small_config(name: str, B: int, H: int, D: int, lat, top_k: int, top_p: float,
                 alpha: float = 1.0, qk_dtype: str = "bf16") -> Config:
    """An ad-hoc small workload for parity tests (half uniform, half sink heads)."""
    half = max(H // 2, 0)
    hts = tuple([HeadType("uniform", alpha)] * half + [HeadType("sink", alpha, sink=8.0)] * (H - half))
    return Config(name, B, H, D, tuple(lat), top_k, top_p, hts, "fwd+bwd", qk_dtype=qk_dtype)


def with_alpha(cfg: Config, alpha_uniform: float, alpha_sink: float) -> Config:
    hts = tuple(replace(h, alpha=(alpha_uniform if h.name == "uniform" else alpha_sink))
                for h in cfg.head_types)
    return replace(cfg, head_types=hts)


# ----------------------------------------------------------------------------------
# drawing

def _phi(cfg: Config, seed: int, b: int, h: int) -> np.ndarray:
    rng = np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, 100, b, h])))
    freqs = np.array([(a, bb, c) for a in range(3) for bb in range(3) for c in range(3)
                      if (a, bb, c) != (0, 0, 0)], dtype=np.float64)
    f = freqs[rng.integers(0, len(freqs), size=cfg.D)]            # [D, 3]
    theta = rng.uniform(0.0, 2.0 * math.pi, size=cfg.D)           # [D]
    lt, lh, lw = cfg.lat
    t = np.arange(lt, dtype=np.float64) / lt
    hh = np.arange(lh, dtype=np.float64) / lh
    w = np.arange(lw, dtype=np.float64) / lw
    # phase per token and channel, latent row-major order
    ph = (f[:, 0][None, None, None, :] * t[:, None, None, None]
          + f[:, 1][None, None, None, :] * hh[None, :, None, None]
          + f[:, 2][None, None, None, :] * w[None, None, :, None])
    return (math.sqrt(2.0) * np.sin(2.0 * math.pi * ph + theta)).reshape(cfg.L, cfg.D)


def _to_bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)


def components(cfg: Config, seed: int, name: str, b: int, h: int):
    """The two draws behind one head of one tensor: (noise, phi), both fp64 [L, D]
    (phi is None for do)."""
    rng = np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, TENSOR_IDS[name], b, h])))
    noise = rng.standard_normal((cfg.L, cfg.D))
    return noise, (None if name == "do" else _phi(cfg, seed, b, h))


def combine(name: str, noise: np.ndarray, phi, ht: HeadType) -> torch.Tensor:
    """Assemble one head from its draws with the head type's amplitude, scale and sink."""
    x = noise.copy()
    if name != "do":
        x += ht.alpha * (0.5 if name == "v" else 1.0) * phi
        if name == "k":
            x *= ht.kscale
            x[0] *= ht.sink
    return _to_bf16(x)


def _one_head(cfg: Config, seed: int, name: str, b: int, h: int) -> torch.Tensor:
    noise, phi = components(cfg, seed, name, b, h)
    return combine(name, noise, phi, cfg.head_types[h])


def make_inputs(cfg: Config, seed: int = 0, names=("q", "k", "v", "do"), heads=None,
                threads: int | None = None) -> dict:
    """Draw the named tensors as bf16 CPU tensors ``[B, len(heads), L, D]`` (latent order)."""
    heads = list(range(cfg.H)) if heads is None else list(heads)
    threads = threads or min(16, os.cpu_count() or 1)
    out = {}
    for name in names:
        jobs = [(b, h) for b in range(cfg.B) for h in heads]
        with ThreadPoolExecutor(threads) as ex:
            parts = list(ex.map(lambda bh: _one_head(cfg, seed, name, bh[0], bh[1]), jobs))
        t = torch.stack(parts).reshape(cfg.B, len(heads), cfg.L, cfg.D)
        out[name] = t
    return out


GATE_ID = 4


def make_gate(cfg: Config, seed: int = 0, heads=None) -> torch.Tensor:
    """Gate values of the gated combination, fp32 ``[B, len(heads), Npad]`` in cube-major slot
    order (one per token slot; the slot order does not matter to an i.i.d. draw):
    ``tanh(N(0, 1))`` from a Philox generator keyed by ``SeedSequence([seed, 4, b, h])``,
    i.e. values spread over the open range of a tanh gate.  Padding slots get values too;
    both sides must ignore them."""
    heads = list(range(cfg.H)) if heads is None else list(heads)
    npad = 64 * math.prod(-(-n // 4) for n in cfg.lat)
    parts = []
    for b in range(cfg.B):
        for h in heads:
            rng = np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, GATE_ID, b, h])))
            parts.append(np.tanh(rng.standard_normal(npad)).astype(np.float32))
    return torch.from_numpy(np.stack(parts).reshape(cfg.B, len(heads), npad))


def quantize_e4m3_rows(x: torch.Tensor, rows: int = 64):
    """Quantise ``x[..., N, D]`` to fp8 e4m3 with one fp32 scale per group of ``rows`` rows.

    scale = amax(|group|) / 448 (1 when the group is all zero); codes are
    round-to-nearest-even of x / scale, clamped to +-448.  Works on any device.
    Returns (codes as uint8 tensor, scales fp32 ``[..., N // rows]``).
    """
    *lead, N, D = x.shape
    assert N % rows == 0
    g = x.float().reshape(*lead, N // rows, rows * D)
    amax = g.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    y = (g / scale[..., None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    codes = y.view(torch.uint8).reshape(*lead, N, D)
    return codes, scale.float()
