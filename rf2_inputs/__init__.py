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
Parameters come from numpy's PCG64 with seed ``1000 * cfg + {0, 1, 2}`` for Q/K/V and
the noise from torch's CPU generator with the same seed; angles and their sin/cos in
float64, the field and the noise in float32, the sum rounded to bf16 (nearest even).
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
    "gen_tensor_torch",
    "gen_pattern_heads",
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
    """Return raw bf16 bits (uint16) of shape [B, T*H*W, heads, D], raster token order.

    Each sinusoid is evaluated through the angle-addition identity,
    sin(a_t + b_h + c_w) = sin(a_t + b_h) cos(c_w) + cos(a_t + b_h) sin(c_w),
    so that only [H, heads*D] and [W, heads*D] tables need sin/cos (float64) and the
    [H, W] field of each frame is one small batched product (float32).  The noise is
    drawn by torch's CPU generator seeded with the same seed; CPU tensors only."""
    import torch

    rng = np.random.Generator(np.random.PCG64(seed))
    gen = torch.Generator(device="cpu")
    gen.manual_seed(int(seed))
    C = heads * D
    ft = rng.uniform(0.5, 2.0, size=(B, C, n_sin))
    fh = rng.uniform(0.5, 4.0, size=(B, C, n_sin))
    fw = rng.uniform(0.5, 4.0, size=(B, C, n_sin))
    ph = rng.uniform(0.0, 2.0 * np.pi, size=(B, C, n_sin))
    amp = field_amp / np.sqrt(2.0)
    two_pi = 2.0 * np.pi
    hh = (np.arange(H) / H)[:, None, None]
    ww = (np.arange(W) / W)[:, None, None]
    out = torch.empty((B, T, H, W, C), dtype=torch.bfloat16)
    for b in range(B):
        cw = two_pi * fw[b][None] * ww                      # [W, C, n]
        qw = np.concatenate([np.cos(cw), np.sin(cw)], axis=-1)
        qw = torch.from_numpy(np.ascontiguousarray(qw.transpose(1, 2, 0), dtype=np.float32))  # [C,2n,W]
        for t in range(T):
            ah = two_pi * (ft[b][None] * (t / T) + fh[b][None] * hh) + ph[b][None]  # [H, C, n]
            pa = np.concatenate([np.sin(ah), np.cos(ah)], axis=-1) * amp
            pa = torch.from_numpy(np.ascontiguousarray(pa.transpose(1, 0, 2), dtype=np.float32))  # [C,H,2n]
            field = torch.bmm(pa, qw).permute(1, 2, 0)                                           # [H,W,C]
            x = torch.randn((H, W, C), generator=gen, dtype=torch.float32)
            if noise != 1.0:
                x.mul_(noise)
            x.add_(field)
            out[b, t] = x.to(torch.bfloat16)
    return out.view(torch.int16).numpy().view(np.uint16).reshape(B, T * H * W, heads, D)


def gen_qkv(wl: Workload, seed_base: Optional[int] = None,
            batch: Optional[int] = None) -> Sequence[np.ndarray]:
    """Q, K, V raw bf16 bits for a workload (seed = 1000*cfg + 0/1/2)."""
    s0 = 1000 * wl.cfg if seed_base is None else seed_base
    B = wl.B if batch is None else batch
    return [gen_tensor(B, wl.T, wl.H, wl.W, wl.heads, wl.D, s0 + i) for i in range(3)]


def gen_tensor_torch(B: int, T: int, H: int, W: int, heads: int, D: int, seed: int,
                     device, field_amp: float = 0.5, n_sin: int = 4):
    """The same recipe as gen_tensor, evaluated with torch on `device` (used to build
    large benchmark inputs quickly).  The field parameters are identical to gen_tensor's;
    the noise comes from the device's generator, so the bits differ from gen_tensor's.
    Returns a bf16 tensor [B, T*H*W, heads, D] on `device`."""
    import torch

    rng = np.random.Generator(np.random.PCG64(seed))
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    C = heads * D
    ft = rng.uniform(0.5, 2.0, size=(B, C, n_sin))
    fh = rng.uniform(0.5, 4.0, size=(B, C, n_sin))
    fw = rng.uniform(0.5, 4.0, size=(B, C, n_sin))
    ph = rng.uniform(0.0, 2.0 * np.pi, size=(B, C, n_sin))
    amp = field_amp / np.sqrt(2.0)
    two_pi = 2.0 * np.pi
    hh = (np.arange(H) / H)[:, None, None]
    ww = (np.arange(W) / W)[:, None, None]
    out = torch.empty((B, T, H, W, C), dtype=torch.bfloat16, device=device)
    for b in range(B):
        cw = two_pi * fw[b][None] * ww
        qw = np.concatenate([np.cos(cw), np.sin(cw)], axis=-1)
        qw = torch.from_numpy(np.ascontiguousarray(qw.transpose(1, 2, 0), dtype=np.float32)).to(device)
        for t in range(T):
            ah = two_pi * (ft[b][None] * (t / T) + fh[b][None] * hh) + ph[b][None]
            pa = np.concatenate([np.sin(ah), np.cos(ah)], axis=-1) * amp
            pa = torch.from_numpy(np.ascontiguousarray(pa.transpose(1, 0, 2), dtype=np.float32)).to(device)
            x = torch.randn((H, W, C), generator=gen, dtype=torch.float32, device=device)
            x.add_(torch.bmm(pa, qw).permute(1, 2, 0))
            out[b, t] = x.to(torch.bfloat16)
    return out.view(B, T * H * W, heads, D)


def gen_pattern_heads(B: int, T: int, H: int, W: int, heads: int, D: int, seed: int,
                      kinds: str, amp: float = 2.0, noise: float = 0.3) -> Sequence[np.ndarray]:
    """Q, K, V raw bf16 bits [B, T*H*W, heads, D] whose heads follow planted attention
    patterns, one letter per head in `kinds`:

      't' - Q = K = amp * u[h, w] + noise * eps: one random vector per spatial position,
            the same in every frame (each token matches its own location in all frames);
      's' - Q = K = amp * v[t] + noise * eps: one random vector per frame (each token
            matches every token of its own frame);
      'x' - Q, K = eps: unstructured.
    u, v, eps ~ N(0, 1) from numpy's PCG64(seed); V = eps for every head.  Rounded to
    bf16 (nearest even)."""
    assert len(kinds) == heads
    rng = np.random.Generator(np.random.PCG64(seed))
    N = T * H * W
    q = np.empty((B, N, heads, D), dtype=np.float32)
    k = np.empty_like(q)
    for b in range(B):
        for h, kind in enumerate(kinds):
            if kind == "t":
                base = np.tile(rng.standard_normal((H * W, D)), (T, 1)) * amp
            elif kind == "s":
                base = np.repeat(rng.standard_normal((T, D)), H * W, axis=0) * amp
            else:
                base = None
            if base is None:
                q[b, :, h] = rng.standard_normal((N, D))
                k[b, :, h] = rng.standard_normal((N, D))
            else:
                q[b, :, h] = base + noise * rng.standard_normal((N, D))
                k[b, :, h] = base + noise * rng.standard_normal((N, D))
    v = rng.standard_normal((B, N, heads, D)).astype(np.float32)
    return [f32_to_bf16_bits(a) for a in (q, k, v)]
