"""Plain fp64 CPU oracle for the RainFusion (v1) mask generators that feed the same
block-sparse attention: the three head patterns, the ARM head classification and the
RainFusion+ dynamic bandwidth.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module.  It shares no code with the CUDA
library.

What it follows (pith.science review of "RainFusion: Adaptive Video Generation
Acceleration via Multi-Dimensional Visual Redundancy"):
  * "What carries the argument": three head patterns (spatial: all locations of nearby
    frames; temporal: the same local region across frames; textural: a sparse lattice of
    keys), a striped band mask for spatial and temporal heads, a checkerboard for
    textural heads; the ARM recall R' = S(Q', K', M') / S(Q', K', M_init) on
    down-sampled queries and keys, with M_init the all-zero (keep everything) mask;
  * "Core claim": local samples are first-frame tokens, global samples are tokens at an
    equal interval; a head is temporal if its local recall reaches alpha, else spatial if
    its global recall does, else textural (Algorithm 1 as the review restates it);
  * "Free parameters": band half-width 1/4 of the axis (9/16 of the work removed),
    checkerboard stride tau = 2 (half of the keys), RainFusion+ picks per head the
    smallest bandwidth of 1/2, 1/4, 1/8 that keeps 90 % recall; alpha and omega are not
    given.
Readings taken where the pages are silent (each listed in the design notes):
  - every mask acts on whole blocks, a block being one 3D window (wt, wh, ww) as in the
    RainFusion2.0 path, so the lists drive the same kernel; the pages' token-level
    checkerboard becomes a checkerboard of windows;
  - a window's temporal coordinate is its temporal block index tb, its spatial coordinate
    its row-major window index sw = hb * nbw + wb inside a temporal slab;
  - spatial band: |tb_i - tb_j| <= R_s; temporal band: |sw_i - sw_j| <= R_t; with
    R = floor(b * C + 1e-6) for bandwidth b and C = nbt (spatial) or nbh * nbw
    (temporal); the 1e-6 guards products such as 0.3 * 10;
  - textural: key window kept iff (hb + wb) mod tau == 0 (every query keeps the same
    keys; tau = 2 keeps half, as the pages state; the printed set formula is garbled);
  - S(Q', K', M) sums, over sampled query rows, the softmax probability (over all sampled
    keys, scale 1/sqrt(D)) of the pairs that M keeps, so R' is the mean kept mass per
    row; M' judges a sampled pair by the windows of its two tokens;
  - local sample: the H * W tokens of frame 0 (queries and keys); global sample: tokens
    0, omega, 2 omega, ... of the raster order, omega = T by default (H * W samples);
  - alpha defaults to 0.9, the recall level the pages use for RainFusion+;
  - RainFusion+ keeps the classification at the static bandwidth and then, for a
    temporal or spatial head, uses the smallest level whose recall (of that head's own
    pattern) reaches the target, else 1/2.

Parity status (what pins each function, in tests/test_oracle_rf1.py):
  rf1_radius / rf1_keeps / rf1_lists : hand-worked lists (tests/golden/rf1_lists.txt); the
                                       pair matrix equals the pair-by-pair definition
  rf1_recall                         : uniform attention (Q = 0) gives hand-worked band
                                       fractions (tests/golden/rf1_uniform_recall.txt);
                                       pair-by-pair brute force; all-keep mask gives 1
  rf1_classify                       : planted temporal / spatial / textural heads;
                                       RainFusion+ on nested bands
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Tuple

import numpy as np

from .rf2_oracle import Geom

TEMPORAL, SPATIAL, TEXTURAL = 0, 1, 2
LOCAL, GLOBAL = 0, 1                      # sample patterns
RF1_LEVELS = (0.125, 0.25, 0.5)          # RainFusion+ bandwidths


@dataclass(frozen=True)
class Rf1Params:
    bandwidth: float = 0.25
    tau: int = 2
    alpha: float = 0.9
    omega: int = 0            # 0: T
    dynamic: bool = False     # RainFusion+
    recall_target: float = 0.9

    def levels(self) -> Tuple[float, ...]:
        """Bandwidths whose recall is measured: the static one, then the RainFusion+ set."""
        return (self.bandwidth,) + RF1_LEVELS


def rf1_radius(bandwidth: float, C: int) -> int:
    """Band half-width in blocks for bandwidth b over an axis of C blocks."""
    return int(math.floor(bandwidth * C + 1e-6))


def block_coords(g: Geom, j: int) -> Tuple[int, int, int, int]:
    """(tb, sw, hb, wb) of block j (blocks row-major over (tb, hb, wb))."""
    P = g.nbh * g.nbw
    tb, sw = divmod(j, P)
    hb, wb = divmod(sw, g.nbw)
    return tb, sw, hb, wb


def rf1_keeps(g: Geom, cls: int, param: int, i: int, j: int) -> bool:
    """Does query block i keep key block j under a head of class cls (param = band
    radius, or tau for a textural head)?"""
    tbi, swi, _, _ = block_coords(g, i)
    tbj, swj, hbj, wbj = block_coords(g, j)
    if cls == TEMPORAL:
        return abs(swi - swj) <= param
    if cls == SPATIAL:
        return abs(tbi - tbj) <= param
    return (hbj + wbj) % param == 0


def rf1_keep_matrix(g: Geom, cls: int, param: int) -> np.ndarray:
    """bool [Nb (query), Nb (key)]: rf1_keeps for every pair, from the block coordinates."""
    j = np.arange(g.Nb)
    P = g.nbh * g.nbw
    tb, sw = j // P, j % P
    hb, wb = sw // g.nbw, sw % g.nbw
    if cls == TEMPORAL:
        return np.abs(sw[:, None] - sw[None, :]) <= param
    if cls == SPATIAL:
        return np.abs(tb[:, None] - tb[None, :]) <= param
    return np.broadcast_to(((hb + wb) % param == 0)[None, :], (g.Nb, g.Nb))


def rf1_lists(g: Geom, cls: np.ndarray, param: np.ndarray):
    """Ascending kept lists per (b, head, query block): list of lists of arrays."""
    out = []
    for b in range(cls.shape[0]):
        per_head = []
        for h in range(cls.shape[1]):
            m = rf1_keep_matrix(g, int(cls[b, h]), int(param[b, h]))
            per_head.append([np.nonzero(m[i])[0].astype(np.int32) for i in range(g.Nb)])
        out.append(per_head)
    return out


def rf1_omega(g: Geom, p: Rf1Params) -> int:
    return g.T if p.omega == 0 else p.omega


def rf1_samples(g: Geom, p: Rf1Params, pattern: int) -> np.ndarray:
    """Raster token indices of the local (frame 0) or global (every omega-th) sample."""
    if pattern == LOCAL:
        return np.arange(g.H * g.W)
    return np.arange(0, g.N, rf1_omega(g, p))


def token_window(g: Geom, n: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """(tb, sw) of the windows holding raster tokens n."""
    t, rest = np.divmod(n, g.H * g.W)
    h, w = np.divmod(rest, g.W)
    return t // g.wt, (h // g.wh) * g.nbw + (w // g.ww)


def _softmax_rows(z: np.ndarray) -> np.ndarray:
    m = np.max(z, axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def rf1_recall(q: np.ndarray, k: np.ndarray, g: Geom, p: Rf1Params) -> np.ndarray:
    """ARM recall [B, heads, 2 patterns, 4 levels] on model-order q, k [B, N, heads, D].

    Pattern LOCAL scores the temporal band on the frame-0 sample, GLOBAL the spatial band
    on the every-omega sample; levels are p.levels()."""
    B = q.shape[0]
    out = np.zeros((B, g.heads, 2, 4))
    for pattern in (LOCAL, GLOBAL):
        idx = rf1_samples(g, p, pattern)
        tb, sw = token_window(g, idx)
        coord, C = (sw, g.nbh * g.nbw) if pattern == LOCAL else (tb, g.nbt)
        dist = np.abs(coord[:, None] - coord[None, :])
        for b in range(B):
            for h in range(g.heads):
                qs = np.asarray(q[b, idx, h], dtype=np.float64)
                ks = np.asarray(k[b, idx, h], dtype=np.float64)
                P = _softmax_rows(qs @ ks.T / math.sqrt(g.D))
                for l, bw in enumerate(p.levels()):
                    inside = dist <= rf1_radius(bw, C)
                    out[b, h, pattern, l] = np.mean(np.sum(P * inside, axis=1))
    return out


def rf1_classify(recall: np.ndarray, g: Geom, p: Rf1Params) -> Tuple[np.ndarray, np.ndarray]:
    """Head class [B, heads] and its mask parameter (band radius, or tau) from the recall."""
    B, Hh = recall.shape[:2]
    cls = np.empty((B, Hh), dtype=np.int32)
    param = np.empty((B, Hh), dtype=np.int32)
    for b in range(B):
        for h in range(Hh):
            if recall[b, h, LOCAL, 0] >= p.alpha:
                c, pattern, C = TEMPORAL, LOCAL, g.nbh * g.nbw
            elif recall[b, h, GLOBAL, 0] >= p.alpha:
                c, pattern, C = SPATIAL, GLOBAL, g.nbt
            else:
                cls[b, h], param[b, h] = TEXTURAL, p.tau
                continue
            bw = p.bandwidth
            if p.dynamic:
                bw = RF1_LEVELS[-1]
                for l, level in enumerate(RF1_LEVELS):
                    if recall[b, h, pattern, 1 + l] >= p.recall_target:
                        bw = level
                        break
            cls[b, h], param[b, h] = c, rf1_radius(bw, C)
    return cls, param


def rf1_kmax(g: Geom, p: Rf1Params) -> int:
    """Longest kept list any head class can produce under these parameters."""
    bws = p.levels() if p.dynamic else (p.bandwidth,)
    best = int(rf1_keep_matrix(g, TEXTURAL, p.tau)[0].sum())
    for c, C in ((TEMPORAL, g.nbh * g.nbw), (SPATIAL, g.nbt)):
        for bw in bws:
            best = max(best, int(rf1_keep_matrix(g, c, rf1_radius(bw, C)).sum(axis=1).max()))
    return best


def rf1_predict_mask(q: np.ndarray, k: np.ndarray, g: Geom, p: Rf1Params):
    """The whole v1 generator: recall -> class -> lists.  Returns (idx [B, heads, Nb,
    kmax] -1 padded, cnt [B, heads, Nb], cls [B, heads], param [B, heads], recall)."""
    recall = rf1_recall(q, k, g, p)
    cls, param = rf1_classify(recall, g, p)
    kmax = rf1_kmax(g, p)
    lists = rf1_lists(g, cls, param)
    B = q.shape[0]
    idx = np.full((B, g.heads, g.Nb, kmax), -1, dtype=np.int32)
    cnt = np.zeros((B, g.heads, g.Nb), dtype=np.int32)
    for b in range(B):
        for h in range(g.heads):
            for i in range(g.Nb):
                lst = lists[b][h][i]
                idx[b, h, i, :len(lst)] = lst
                cnt[b, h, i] = len(lst)
    return idx, cnt, cls, param, recall
