"""Seeded synthetic inputs and the workload table for block-sparse video attention.

This module is shared by the CUDA path's tests and benchmark and by the CPU oracle's
tests.  It holds no arithmetic of the attention method itself: only the shapes of the
workloads and a seeded generator of bf16 Q/K/V tensors.

Workload shapes follow the configurations shown for RainFusion2.0 ("RainFusion2.0:
Temporal-Spatial Awareness and Hardware-Efficient Block-wise Sparse Attention",
sciencestack page, Figure 2 caption: Wan2.2 / HunyuanVideo1.5 720p video at 80%
sparsity, Qwen-image-edit 1024x1024 at 60% sparsity).  No real activations or model
weights are used; the tensors stand in for them.

Generator (one tensor X of shape [B, N, heads, D], tokens in raster (t, h, w) order):

    X = 0.5 * F + eps,     eps ~ N(0, 1) i.i.d.
    F[t,h,w,head,c] = sum_{j=1..4} (1/sqrt 2) * sin(2*pi*(ft*t/T + fh*h/H + fw*w/W) + phi)

with (ft, fh, fw, phi) drawn per (head, c, j): ft ~ U[0.5, 2], fh, fw ~ U[0.5, 4],
phi ~ U[0, 2*pi).  Var F is about 1, so block means carry real spatial structure.
Parameters come from numpy's PCG64 with seed ``1000 * cfg + {0, 1, 2}`` for Q/K/V;
the field is evaluated in float32 and the sum rounded to bf16 (round to nearest even).
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "workload",
    "gen_tensor",
    "gen_qkv",
    "bf16_bits_to_f64",
    "f32_to_bf16_bits",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention-call shape.  Layout of every Q/K/V/O tensor: [B, N, heads, D]."""

    name: str
    cfg: int  # seed base (1000 * cfg)
    B: int
    heads: int
    T: int
    H: int
    W: int
    D: int
    wt: int
    wh: int
    ww: int
    sparsities: Tuple[float, ...]
    sink: bool

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def sparsity(self) -> float:
        """The sparsity the workload is quoted at (the last entry for a sweep is 80%)."""
        return 0.8 if 0.8 in self.sparsities else self.sparsities[0]

    def geom(self) -> dict:
        return dict(B=self.B, heads=self.heads, T=self.T, H=self.H, W=self.W, D=self.D,
                    wt=self.wt, wh=self.wh, ww=self.ww)


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 2, 4, 16, 16, 64, 1, 8, 8, (0.8,), True),
    "video480p": Workload("video480p", 2, 1, 12, 8, 32, 48, 128, 2, 8, 8, (0.8,), True),
    "wan720p": Workload("wan720p", 3, 1, 40, 21, 45, 80, 128, 2, 8, 8, (0.8,), True),
    "imgedit1024": Workload("imgedit1024", 4, 1, 24, 2, 64, 64, 128, 1, 8, 16, (0.6,), False),
    "longvideo": Workload("longvideo", 5, 1, 16, 31, 45, 80, 128, 2, 8, 8,
                          (0.0, 0.5, 0.7, 0.8, 0.9), True),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even) and return the raw uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    r = ((u >> 16) & 1) + 0x7FFF
    out = ((u + r) >> 16).astype(np.uint16)
    out[nan] = 0x7FC0
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bits (uint16) to float64."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def gen_tensor(B: int, T: int, H: int, W: int, heads: int, D: int, seed: int,
               field_amp: float = 0.5, noise: float = 1.0, n_sin: int = 4) -> np.ndarray:
    """Return raw bf16 bits (uint16) of shape [B, T*H*W, heads, D], raster token order."""
    rng = np.random.Generator(np.random.PCG64(seed))
    ft = rng.uniform(0.5, 2.0, size=(B, heads, D, n_sin)).astype(np.float32)
    fh = rng.uniform(0.5, 4.0, size=(B, heads, D, n_sin)).astype(np.float32)
    fw = rng.uniform(0.5, 4.0, size=(B, heads, D, n_sin)).astype(np.float32)
    ph = rng.uniform(0.0, 2.0 * np.pi, size=(B, heads, D, n_sin)).astype(np.float32)
    amp = np.float32(field_amp / np.sqrt(2.0))
    two_pi = np.float32(2.0 * np.pi)
    hh = (np.arange(H, dtype=np.float32) / np.float32(H))[:, None, None, None, None]
    ww = (np.arange(W, dtype=np.float32) / np.float32(W))[None, :, None, None, None]
    out = np.empty((B, T, H, W, heads, D), dtype=np.uint16)
    for b in range(B):
        # phase over (h, w, head, c, j), without the t term
        base = two_pi * (fh[b][None, None] * hh + fw[b][None, None] * ww) + ph[b][None, None]
        for t in range(T):
            ang = base + two_pi * ft[b] * np.float32(t / T)
            field = amp * np.sin(ang, dtype=np.float32).sum(axis=-1, dtype=np.float32)
            eps = rng.standard_normal(size=(H, W, heads, D), dtype=np.float32)
            out[b, t] = f32_to_bf16_bits(field + np.float32(noise) * eps)
    return out.reshape(B, T * H * W, heads, D)


def gen_qkv(wl: Workload, seed_base: Optional[int] = None,
            batch: Optional[int] = None) -> Sequence[np.ndarray]:
    """Q, K, V raw bf16 bits for a workload (seed = 1000*cfg + 0/1/2)."""
    s0 = 1000 * wl.cfg if seed_base is None else seed_base
    B = wl.B if batch is None else batch
    return [gen_tensor(B, wl.T, wl.H, wl.W, wl.heads, wl.D, s0 + i) for i in range(3)]
