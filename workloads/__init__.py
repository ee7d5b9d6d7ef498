"""Seeded synthetic long-context attention inputs.

This module only draws random numbers and shapes them into per-head Q, K, V tensors
with the structure of long-context attention (sink keys, local correlation, vertical
columns, diagonal "slash" offsets, video frames).  It holds none of the sparse-attention
method's arithmetic: both the CUDA path and the CPU oracle consume the same bf16 bytes
produced here.

Every tensor or feature has its own CPU ``torch.Generator`` seeded with
``seed * 1000 + k`` (k: Q=0, K=1, V=2, sink=3, vertical-pos=4, vertical-dir=5,
slash-offsets=6, slash-dirs=7, frames=8).  Values are generated in fp32 (the AR(1)
filter in fp64) and rounded to bf16 (round-to-nearest-even) once.

Layouts: ``Q`` is ``[H][L][d]``, ``K`` and ``V`` are ``[Hkv][L][d]``, batch 1,
contiguous bf16.  Query head ``h`` uses KV head ``h // (H // Hkv)``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "get", "generate", "kv_group"]

_K_Q, _K_K, _K_V, _K_SINK, _K_VPOS, _K_VDIR, _K_SLASH_OFF, _K_SLASH_DIR, _K_FRAMES = range(9)


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic attention layer: shapes, method parameters and input recipe."""

    name: str
    H: int
    Hkv: int
    L: int
    d: int
    S: int
    B: int
    tau: float
    recipe: str  # "ar_sinks" | "ar_sinks_vertical" | "slash" | "video" | "iid"
    n_vertical: int = 16
    n_slash: int = 8
    frame_len: int = 1024

    @property
    def Nb(self) -> int:
        return self.L // self.B

    @property
    def Ns(self) -> int:
        return self.L // self.S

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = [
    Workload("tiny-causal-h2-L2k-d64", H=2, Hkv=2, L=2048, d=64, S=8, B=64, tau=0.9,
             recipe="ar_sinks"),
    Workload("llama3-8b-layer-L32k", H=32, Hkv=8, L=32768, d=128, S=16, B=128, tau=0.9,
             recipe="ar_sinks_vertical"),
    Workload("llama3-8b-layer-L128k", H=32, Hkv=8, L=131072, d=128, S=16, B=128, tau=0.9,
             recipe="ar_sinks_vertical"),
    Workload("slash-stress-L64k", H=32, Hkv=8, L=65536, d=128, S=16, B=128, tau=0.9,
             recipe="slash"),
    Workload("video-vlm-layer-L96k", H=28, Hkv=4, L=98304, d=128, S=16, B=128, tau=0.9,
             recipe="video", frame_len=1024),
]


def get(which, **overrides) -> Workload:
    """Workload by index or name, with optional field overrides (e.g. a shorter L)."""
    if isinstance(which, Workload):
        w = which
    elif isinstance(which, int):
        w = WORKLOADS[which]
    else:
        w = next(x for x in WORKLOADS if x.name == which)
    return w.with_(**overrides) if overrides else w


def kv_group(h: int, H: int, Hkv: int) -> int:
    """KV head used by query head ``h`` (contiguous grouping, as in Llama-style GQA)."""
    return h // (H // Hkv)


def _gen(seed: int, k: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 1000 + k)
    return g


def _normal(g: torch.Generator, shape, std: float) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32).mul_(std)


def _unit(g: torch.Generator, *shape) -> torch.Tensor:
    v = torch.randn(*shape, generator=g, dtype=torch.float64)
    return (v / v.norm(dim=-1, keepdim=True)).to(torch.float32)


def _ar1(eps: torch.Tensor, phi: float = 0.8, gain: float = 0.6) -> torch.Tensor:
    """K_0 = e_0, K_t = phi*K_{t-1} + gain*e_t along dim 1 (stationary for gain^2+phi^2=1)."""
    from scipy.signal import lfilter

    x = eps.to(torch.float64).numpy()
    x[:, 0, :] /= gain
    y = lfilter([gain], [1.0, -phi], x, axis=1)
    return torch.from_numpy(np.ascontiguousarray(y)).to(torch.float32)


def _add_sinks(w: Workload, Q, K, seed: int, n_sink: int = 4):
    s0 = 0.5 * math.sqrt(w.d)
    u = _unit(_gen(seed, _K_SINK), w.Hkv, w.d)
    n = min(n_sink, w.L)
    K[:, :n, :] += 3.0 * s0 * u[:, None, :]
    G = w.H // w.Hkv
    Q += s0 * u.repeat_interleave(G, dim=0)[:, None, :]


def _add_verticals(w: Workload, Q, K, seed: int):
    s0 = 0.5 * math.sqrt(w.d)
    gp = _gen(seed, _K_VPOS)
    v = _unit(_gen(seed, _K_VDIR), w.H, w.d)
    lo = min(4, w.L - 1)
    for h in range(w.H):
        n = min(w.n_vertical, w.L - lo)
        cols = torch.randperm(w.L - lo, generator=gp)[:n] + lo
        K[kv_group(h, w.H, w.Hkv), cols, :] += 2.5 * s0 * v[h]
        Q[h] += s0 * v[h]


def _add_slashes(w: Workload, Q, K, seed: int):
    """Diagonal offsets: key s carries a per-position unit direction W_s (per KV head);
    query t of head h adds W_{t-delta} for each of its offsets, so q_t and k_{t-delta}
    share a direction of magnitude 2x the background row norm."""
    s0 = 0.5 * math.sqrt(w.d)
    go = _gen(seed, _K_SLASH_OFF)
    W = _unit(_gen(seed, _K_SLASH_DIR), w.Hkv, w.L, w.d)
    K += 2.0 * s0 * W
    half = max(1, w.L // 2)
    for h in range(w.H):
        g = kv_group(h, w.H, w.Hkv)
        deltas = torch.randperm(half, generator=go)[: w.n_slash] + 1
        for dl in deltas.tolist():
            if dl < w.L:
                Q[h, dl:, :] += 2.0 * s0 * W[g, : w.L - dl, :]


def generate(w: Workload, seed: int = 0) -> Dict[str, torch.Tensor]:
    """Q [H][L][d], K and V [Hkv][L][d] as contiguous bf16 CPU tensors."""
    H, Hkv, L, d = w.H, w.Hkv, w.L, w.d
    if H % Hkv:
        raise ValueError("H must be a multiple of Hkv")
    std = 0.5
    Q = _normal(_gen(seed, _K_Q), (H, L, d), std)
    V = _normal(_gen(seed, _K_V), (Hkv, L, d), std)
    eps = _normal(_gen(seed, _K_K), (Hkv, L, d), std)
    if w.recipe in ("ar_sinks", "ar_sinks_vertical"):
        K = _ar1(eps) if L > 0 else eps
        _add_sinks(w, Q, K, seed)
        if w.recipe == "ar_sinks_vertical":
            _add_verticals(w, Q, K, seed)
    elif w.recipe == "slash":
        K = eps
        _add_sinks(w, Q, K, seed)
        _add_slashes(w, Q, K, seed)
    elif w.recipe == "video":
        F = max(1, -(-L // w.frame_len))
        gf = _gen(seed, _K_FRAMES)
        m0 = _normal(gf, (Hkv, 1, d), std)
        steps = _normal(gf, (Hkv, max(F - 1, 0), d), 0.05)
        means = torch.cat([m0, m0 + steps.cumsum(dim=1)], dim=1)  # [Hkv][F][d]
        frame_of_t = torch.arange(L) // w.frame_len
        K = 0.9 * means[:, frame_of_t, :] + math.sqrt(0.19) * eps
    elif w.recipe == "iid":
        K = eps
    else:
        raise ValueError(f"unknown recipe {w.recipe}")
    return {
        "Q": Q.to(torch.bfloat16).contiguous(),
        "K": K.to(torch.bfloat16).contiguous(),
        "V": V.to(torch.bfloat16).contiguous(),
    }


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 bit patterns of a bf16 CPU tensor (a view, no copy)."""
    assert t.dtype == torch.bfloat16 and t.is_contiguous()
    return t.view(torch.int16).numpy().view(np.uint16)
