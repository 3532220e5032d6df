"""Plain CPU oracle for the FP8 (e4m3) variant of the block-sparse attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module.  It shares no code with the CUDA
library.

The pages point to pairing the block-sparse attention with quantisation for further
speed (RF2 sciencestack page, TL;DR, its closing remark on integration with quantisation
or distillation); the FP8 form is this build's reading, not a method the pages specify.
Reading used here:
  - Q, K and V are each quantised to e4m3 with one scale per (batch, head, block), the
    block being the same 3D window (or raster block) the mask works on;
  - per block: amax = max |x| over its real tokens and the head's D channels (exact);
    inv = fp32(448) / fp32(amax) and scale = fp32(amax) / fp32(448), both rounded to
    fp32; each element is y = fp32(x * inv) and its code the nearest e4m3 value of y
    (ties to even, saturating at +-448); amax = 0 gives inv = scale = 0;
  - e4m3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; normal values
    2^(e-7) (1 + m/8), subnormals 2^-6 m/8, largest finite 448 (no infinities);
  - the attention of the quantised call is the exact attention over the dequantised
    tensors code * scale (fp64 here); the kernel additionally rounds the probabilities to
    e4m3 for the P V product, which the tolerance of the tests covers.
The quantisation is a decision taken in fp32 (the kernel's precision), so the oracle
takes it in fp32 too and the codes compare bit for bit.

Parity status (tests/test_oracle_fp8.py): e4m3_round against a hand-worked table
(tests/golden/e4m3_round.txt) and torch's float8_e4m3fn cast inside the finite range;
e4m3_code against torch's bit patterns; quantise_blocks: the amax element maps to +-448,
dequantisation error within half an e4m3 step, zero blocks, pad tokens ignored.
"""
from __future__ import annotations

import numpy as np

from .rf2_oracle import Geom, position_valid, permute, default_scale, _softmax_rows

E4M3_MAX = 448.0


def e4m3_round(y) -> np.ndarray:
    """Nearest e4m3 value of y (ties to even), saturated to +-448; fp64 out."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    _, ex = np.frexp(a)                      # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)               # binade of a, at least the subnormal one
    ulp = np.ldexp(1.0, e - 3)
    q = np.round(a / ulp) * ulp              # np.round: half to even
    q = np.minimum(q, E4M3_MAX)
    return np.where(y < 0, -q, q)


def e4m3_code(v) -> np.ndarray:
    """uint8 bit pattern of e4m3 values v (already representable)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    code = np.zeros(a.shape, dtype=np.int64)
    normal = a >= 2.0 ** -6
    _, ex = np.frexp(np.where(normal, a, 1.0))
    e = ex - 1
    m = np.where(normal, a / np.ldexp(1.0, e) * 8 - 8, 0).astype(np.int64)
    code = np.where(normal, ((e + 7) << 3) | m, np.round(a / 2.0 ** -9).astype(np.int64))
    return (code | np.where(np.signbit(v), 128, 0)).astype(np.uint8)


def quantise_blocks(xp: np.ndarray, g: Geom):
    """xp: [B, Npad, heads, D] window order (bf16 values as any float; pad rows ignored).
    Returns (codes [B, Npad, heads, D] e4m3 values in fp64 (pad rows 0), scale [B, heads, Nb]
    fp32, inv [B, heads, Nb] fp32)."""
    B = xp.shape[0]
    valid = position_valid(g)
    x32 = np.asarray(xp, dtype=np.float32) * valid[None, :, None, None].astype(np.float32)
    blocks = x32.reshape(B, g.Nb, g.blk, g.heads, g.D)
    amax = np.abs(blocks).max(axis=(2, 4))                       # [B, Nb, heads], exact
    amax = np.transpose(amax, (0, 2, 1)).astype(np.float32)      # [B, heads, Nb]
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, np.float32(E4M3_MAX) / amax, np.float32(0)).astype(np.float32)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(0)).astype(np.float32)
    inv_b = np.transpose(inv, (0, 2, 1))[:, :, None, :, None]    # [B, Nb, 1, heads, 1]
    y = (blocks * inv_b).astype(np.float32)                      # fp32 product, rounded
    codes = e4m3_round(y).reshape(B, g.Npad, g.heads, g.D)
    return codes, scale, inv


def dequantise(codes: np.ndarray, scale: np.ndarray, g: Geom) -> np.ndarray:
    """code * scale of its (batch, head, block), fp64 [B, Npad, heads, D]."""
    B = codes.shape[0]
    s = np.transpose(scale.astype(np.float64), (0, 2, 1))        # [B, Nb, heads]
    s = np.repeat(s, g.blk, axis=1)[:, :, :, None]               # [B, Npad, heads, 1]
    return codes * s


def fp8_attention_block(qd, kd, vd, g: Geom, b: int, h: int, i: int, kept_ids, scale: float) -> np.ndarray:
    """Rows [blk, D] of query block i over the dequantised tensors (window order), pad
    keys excluded: the reference of the FP8 call."""
    blk = g.blk
    valid = position_valid(g)
    q = qd[b, i * blk:(i + 1) * blk, h]
    rows = np.concatenate([np.arange(j * blk, (j + 1) * blk) for j in kept_ids])
    rows = rows[valid[rows]]
    p = _softmax_rows((q @ kd[b, rows, h].T) * scale)
    return p @ vd[b, rows, h]


def quantised_inputs(q, k, v, g: Geom):
    """Model-order q, k, v -> dequantised window-order tensors and the raw quantisation."""
    out = []
    for x in (q, k, v):
        codes, scale, inv = quantise_blocks(permute(np.asarray(x, dtype=np.float64), g), g)
        out.append((codes, scale, inv, dequantise(codes, scale, g)))
    return out


__all__ = ["E4M3_MAX", "e4m3_round", "e4m3_code", "quantise_blocks", "dequantise", "fp8_attention_block",
           "quantised_inputs", "default_scale"]
