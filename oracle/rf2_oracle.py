"""Plain fp64 CPU oracle for the RainFusion2.0 block-sparse attention hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module.  The CUDA library never calls it,
and it shares no code with the CUDA library (no kernels, helpers, tables or constants).

What it follows ("RainFusion2.0: Temporal-Spatial Awareness and Hardware-Efficient
Block-wise Sparse Attention"):
  * mlsanity index page, Abstract, key insight (1): block-wise mean values serve as the
    representative tokens that predict the sparse mask;
  * same passage, insight (2): a spatiotemporal-aware token permutation;
  * same passage, insight (3): a first-frame sink;
  * sciencestack page, TL;DR: "3D window permutation", "blockwise representative
    tokens", "First Frame Sink", online adaptive mask prediction, 80% sparsity;
  * mlsanity index page, title: block-wise sparse attention.
The pages give no formulas.  Every step below is the plainest reading of those passages;
each reading is listed in the design notes of the repository and restated here:
  - a block is one 3D window (wt, wh, ww) of the padded [T, H, W] token grid; windows
    and the tokens inside a window are both ordered row-major in (t, h, w);
  - the grid is padded at the high end of each axis to window multiples; pad tokens are
    zero, excluded from block means, masked out as keys, and their query rows dropped;
  - the representative token of a block is the mean of its valid tokens, per head;
  - the pooled score is s_ij = qbar_i . kbar_j * scale (scale = 1/sqrt(D) by default);
  - per (batch, head, query block) row, the kept set is the frame-0 key blocks (sink,
    inside the budget) plus the best-scoring other blocks up to
    K_target = ceil((1 - sparsity) * N_valid - 1e-6), clamped to [1, N_valid];
    ties go to the lower block index; the list is ascending;
  - attention of a query block runs over the tokens of its kept key blocks only.

Parity status of each function (what pins it, in tests/test_oracle.py):
  window_positions / permute / unpermute : hand-worked golden tables, round trip, brute force
  pool                                   : constant fields, planted block constants, pad exclusion
  pooled_scores                          : one-hot planted means (closed form)
  select_blocks                          : rank-count brute force, planted orderings, invariants
  sparse_attention                       : dense brute force at 0% sparsity, torch SDPA (fp64),
                                           explicit -inf masked dense attention, closed forms
  schedule_action                        : hand-worked step tables (tests/golden/schedule_actions.txt)
  no_permute geometry (raster blocks)    : hand-worked positions and sink, equality with the
                                           (T, 1, W) grid cut into (1, 1, blk) windows
The end-to-end RF2 numbers themselves are not printed on the pages (no worked example),
so the method's outputs beyond these pins are "parity unpinned by the pages".
"""
from __future__ import annotations

import dataclasses
import functools
import math
from dataclasses import dataclass
from typing import List, Optional, Sequence, Tuple

import numpy as np


# ----------------------------------------------------------------------------- geometry

@dataclass(frozen=True)
class Geom:
    B: int
    heads: int
    T: int
    H: int
    W: int
    D: int
    wt: int
    wh: int
    ww: int
    # "Without 3D permutation" ablation (sciencestack page, Figure 3 (b)): a block is blk
    # consecutive tokens of the raster order instead of a 3D window.
    no_permute: bool = False

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def Tp(self) -> int:
        return -(-self.T // self.wt) * self.wt

    @property
    def Hp(self) -> int:
        return -(-self.H // self.wh) * self.wh

    @property
    def Wp(self) -> int:
        return -(-self.W // self.ww) * self.ww

    @property
    def blk(self) -> int:
        return self.wt * self.wh * self.ww

    @property
    def nbt(self) -> int:
        return self.Tp // self.wt

    @property
    def nbh(self) -> int:
        return self.Hp // self.wh

    @property
    def nbw(self) -> int:
        return self.Wp // self.ww

    @property
    def Nb(self) -> int:
        if self.no_permute:
            return -(-self.N // self.blk)
        return self.nbt * self.nbh * self.nbw

    @property
    def Npad(self) -> int:
        return self.Nb * self.blk


def geom(**kw) -> Geom:
    return Geom(**kw)


def window_positions(g: Geom) -> np.ndarray:
    """Position in the permuted sequence of every real token, shape [T, H, W].

    RF2 abstract, insight (2) / TL;DR "3D window permutation": token (t, h, w) belongs to
    window (t//wt, h//wh, w//ww); windows are numbered row-major over the padded grid and
    tokens inside a window row-major over (t%wt, h%wh, w%ww).

    no_permute: the sequence stays in raster order (Figure 3 (b)), so token n sits at
    position n and block n // blk holds it.
    """
    if g.no_permute:
        return np.arange(g.N).reshape(g.T, g.H, g.W)
    t = np.arange(g.T)[:, None, None]
    h = np.arange(g.H)[None, :, None]
    w = np.arange(g.W)[None, None, :]
    block = ((t // g.wt) * g.nbh + (h // g.wh)) * g.nbw + (w // g.ww)
    offset = ((t % g.wt) * g.wh + (h % g.wh)) * g.ww + (w % g.ww)
    return block * g.blk + offset


@functools.lru_cache(maxsize=32)
def position_to_token(g: Geom) -> np.ndarray:
    """Inverse map, built independently of window_positions: for every permuted position
    p in [0, Npad), the raster token index (t*H + h)*W + w, or -1 for a pad position."""
    out = np.full(g.Npad, -1, dtype=np.int64)
    if g.no_permute:
        # raster blocks: position p holds token p; the tail of the last block is padding
        out[:g.N] = np.arange(g.N)
        out.setflags(write=False)
        return out
    for p in range(g.Npad):
        block, offset = divmod(p, g.blk)
        tb, rest = divmod(block, g.nbh * g.nbw)
        hb, wb = divmod(rest, g.nbw)
        dt, rest = divmod(offset, g.wh * g.ww)
        dh, dw = divmod(rest, g.ww)
        t, h, w = tb * g.wt + dt, hb * g.wh + dh, wb * g.ww + dw
        if t < g.T and h < g.H and w < g.W:
            out[p] = (t * g.H + h) * g.W + w
    out.setflags(write=False)
    return out


def permute(x: np.ndarray, g: Geom) -> np.ndarray:
    """x [B, N, heads, D] in raster order -> xp [B, Npad, heads, D] in window order,
    pad rows zero (RF2 abstract, insight (2))."""
    xp = np.zeros((x.shape[0], g.Npad) + x.shape[2:], dtype=x.dtype)
    xp[:, window_positions(g).reshape(-1)] = x
    return xp


def unpermute(xp: np.ndarray, g: Geom) -> np.ndarray:
    """Inverse of permute; pad rows are dropped.  Uses the independent inverse map."""
    tok = position_to_token(g)
    keep = np.nonzero(tok >= 0)[0]
    x = np.empty((xp.shape[0], g.N) + xp.shape[2:], dtype=xp.dtype)
    x[:, tok[keep]] = xp[:, keep]
    return x


def position_valid(g: Geom) -> np.ndarray:
    """bool [Npad]: the permuted position holds a real (non-pad) token."""
    return position_to_token(g) >= 0


def block_valid_counts(g: Geom) -> np.ndarray:
    """Number of real tokens in each block, int [Nb]."""
    return position_valid(g).reshape(g.Nb, g.blk).sum(axis=1)


def sink_blocks(g: Geom) -> np.ndarray:
    """Block ids of the first-frame sink: every window whose temporal index is 0 (RF2
    abstract, insight (3) 'first-frame sink').  With wt > 1 these windows hold frames
    0..wt-1; a block is kept or dropped as a whole.

    no_permute: the blocks that hold at least one token of frame 0, i.e. those starting
    before token H*W of the raster order."""
    if g.no_permute:
        return np.array([j for j in range(g.Nb) if j * g.blk < g.H * g.W], dtype=np.int64)
    return np.arange(g.nbh * g.nbw)


# ----------------------------------------------------------------------------- mask stage

def pool(xp: np.ndarray, g: Geom) -> np.ndarray:
    """Block-mean representative tokens (RF2 abstract, insight (1)).

    xp [B, Npad, heads, D] (any float) -> [B, heads, Nb, D] fp64, the mean over the real
    tokens of each block; pad positions are ignored whatever they hold."""
    x = np.asarray(xp, dtype=np.float64)
    valid = position_valid(g).astype(np.float64)
    x = x * valid[None, :, None, None]
    sums = x.reshape(x.shape[0], g.Nb, g.blk, g.heads, g.D).sum(axis=2)  # [B, Nb, heads, D]
    cnt = block_valid_counts(g).astype(np.float64)
    with np.errstate(invalid="ignore", divide="ignore"):
        means = sums / cnt[None, :, None, None]
    means[:, cnt == 0] = 0.0
    return np.transpose(means, (0, 2, 1, 3))


def pooled_scores(qbar: np.ndarray, kbar: np.ndarray, scale: float) -> np.ndarray:
    """s[b, head, i, j] = qbar_i . kbar_j * scale (block-level QK^T on the representative
    tokens; RF2 abstract, insight (1) 'sparse mask prediction')."""
    return np.einsum("bhid,bhjd->bhij", qbar, kbar) * scale


def default_scale(D: int, scale: float = 0.0) -> float:
    return 1.0 / math.sqrt(D) if scale == 0.0 else float(scale)


def kept_count(g: Geom, sparsity: float, sink: bool, sink_additive: bool = False) -> int:
    """Length of every kept list (every row keeps the same number of blocks).

    In-budget sink (default): kept = max(K_target, |S|), K_target = ceil((1-s)*N_v - 1e-6)
    clamped to [1, N_v].  Additive sink: |S| + ceil((1-s)*(N_v - |S|) - 1e-6), clamped."""
    nv = int((block_valid_counts(g) > 0).sum())
    ns = len(sink_blocks(g)) if sink else 0
    if sink_additive:
        extra = math.ceil((1.0 - sparsity) * (nv - ns) - 1e-6)
        return ns + min(max(extra, 0), nv - ns)
    k = min(max(math.ceil((1.0 - sparsity) * nv - 1e-6), 1), nv)
    return max(k, ns)


@dataclass
class Selection:
    idx: np.ndarray        # int32 [B, heads, Nb, kept], ascending per row
    near_cut: List[set]    # per flattened row: block ids within the near-cut window
    kept: int
    # per flattened row: block ids within 1e-4 * |c| of the cut alone (no floor); a
    # subset of near_cut, kept so that rows excused only by the floor can be reported
    near_cut_strict: List[set] = dataclasses.field(default_factory=list)


def select_blocks(s: np.ndarray, g: Geom, sparsity: float, sink: bool,
                  sink_additive: bool = False, near_rel: float = 1e-4) -> Selection:
    """Per (b, head, query block) row: the sink blocks plus the top-m other valid blocks
    by pooled score, ties to the lower block id, list ascending (RF2 abstract, insights
    (1) and (3); TL;DR: predicted online for every call).

    near_cut[row] holds the non-sink valid blocks whose score lies within
    near_rel * max(|c|, 1e-2 * max_j |s_ij|) of the cut c, the midpoint between the lowest
    kept and the highest dropped non-sink score; it is empty when the two are further
    apart than that.  A GPU's fp32 ranking may legitimately differ from fp64 there."""
    B, Hh, Nq, Nk = s.shape
    kept = kept_count(g, sparsity, sink, sink_additive)
    valid_blk = block_valid_counts(g) > 0
    sinks = set(sink_blocks(g).tolist()) if sink else set()
    cand = np.array([j for j in range(Nk) if valid_blk[j] and j not in sinks], dtype=np.int64)
    m = kept - len(sinks)
    idx = np.empty((B, Hh, Nq, kept), dtype=np.int32)
    near: List[set] = []
    near_strict: List[set] = []
    sink_arr = np.array(sorted(sinks), dtype=np.int64)
    for b in range(B):
        for h in range(Hh):
            for i in range(Nq):
                row = s[b, h, i]
                sc = row[cand]
                # order by score descending, then by block id ascending
                order = np.lexsort((cand, -sc))
                chosen = cand[order[:m]]
                full = np.sort(np.concatenate([sink_arr, chosen]))
                idx[b, h, i] = full
                ns, ns_strict = set(), set()
                if 0 < m < len(cand):
                    # the cut lies between the lowest kept and the highest dropped score
                    cut = 0.5 * (sc[order[m - 1]] + sc[order[m]])
                    tol = near_rel * max(abs(cut), 1e-2 * float(np.max(np.abs(row))))
                    ns = set(cand[np.abs(sc - cut) <= tol].tolist())
                    ns_strict = set(cand[np.abs(sc - cut) <= near_rel * abs(cut)].tolist())
                near.append(ns)
                near_strict.append(ns_strict)
    return Selection(idx=idx, near_cut=near, kept=kept, near_cut_strict=near_strict)


def predict_mask(qp: np.ndarray, kp: np.ndarray, g: Geom, sparsity: float, sink: bool,
                 sink_additive: bool = False, scale: float = 0.0) -> Selection:
    """Pool, score and select: the whole mask stage on permuted Q and K.  The scale of the
    pooled score does not change the ranking; 1/sqrt(D) is used."""
    qbar, kbar = pool(qp, g), pool(kp, g)
    s = pooled_scores(qbar, kbar, 1.0 / math.sqrt(g.D))
    return select_blocks(s, g, sparsity, sink, sink_additive)


# ----------------------------------------------------------------------------- attention

def _softmax_rows(z: np.ndarray) -> np.ndarray:
    m = np.max(z, axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention_block(qp: np.ndarray, kp: np.ndarray, vp: np.ndarray, g: Geom, b: int, h: int,
                    i: int, kept_ids: Sequence[int], scale: float) -> np.ndarray:
    """Output rows [blk, D] (fp64) of query block i of (b, h), attending to the tokens of
    the kept key blocks only; pad keys are excluded (block-wise sparse attention: RF2
    index page, title, and Abstract, where the work on unimportant tokens is skipped)."""
    blk = g.blk
    valid = position_valid(g)
    q = np.asarray(qp[b, i * blk:(i + 1) * blk, h], dtype=np.float64)
    rows = np.concatenate([np.arange(j * blk, (j + 1) * blk) for j in kept_ids])
    rows = rows[valid[rows]]
    k = np.asarray(kp[b, rows, h], dtype=np.float64)
    v = np.asarray(vp[b, rows, h], dtype=np.float64)
    p = _softmax_rows((q @ k.T) * scale)
    return p @ v


def sparse_attention(qp: np.ndarray, kp: np.ndarray, vp: np.ndarray, idx: np.ndarray, g: Geom,
                     scale: float = 0.0, heads: Optional[Sequence[int]] = None) -> np.ndarray:
    """O [B, Npad, heads, D] fp64 over the kept lists idx [B, heads, Nb, kept].  Only the
    heads listed are computed (others left zero)."""
    sc = default_scale(g.D, scale)
    out = np.zeros((qp.shape[0], g.Npad, g.heads, g.D), dtype=np.float64)
    hs = range(g.heads) if heads is None else heads
    for b in range(qp.shape[0]):
        for h in hs:
            for i in range(g.Nb):
                out[b, i * g.blk:(i + 1) * g.blk, h] = attention_block(
                    qp, kp, vp, g, b, h, i, idx[b, h, i], sc)
    return out


def masked_dense_attention(qp: np.ndarray, kp: np.ndarray, vp: np.ndarray, idx: np.ndarray,
                           g: Geom, scale: float = 0.0) -> np.ndarray:
    """Second path for the oracle's self-check: dense softmax(Q K^T * scale + M) V with an
    explicit additive token mask M (0 for keys of kept blocks that are real tokens,
    -inf elsewhere)."""
    sc = default_scale(g.D, scale)
    valid = position_valid(g)
    out = np.zeros((qp.shape[0], g.Npad, g.heads, g.D), dtype=np.float64)
    for b in range(qp.shape[0]):
        for h in range(g.heads):
            mask = np.full((g.Npad, g.Npad), -np.inf)
            for i in range(g.Nb):
                for j in idx[b, h, i]:
                    mask[i * g.blk:(i + 1) * g.blk, j * g.blk:(j + 1) * g.blk] = 0.0
            mask[:, ~valid] = -np.inf
            q = np.asarray(qp[b, :, h], dtype=np.float64)
            k = np.asarray(kp[b, :, h], dtype=np.float64)
            v = np.asarray(vp[b, :, h], dtype=np.float64)
            out[b, :, h] = _softmax_rows(q @ k.T * sc + mask) @ v
    return out


def dense_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """Full softmax attention over the original tokens: [B, N, heads, D] fp64."""
    qf, kf, vf = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    s = np.einsum("bnhd,bmhd->bhnm", qf, kf) * scale
    return np.einsum("bhnm,bmhd->bnhd", _softmax_rows(s), vf)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, g: Geom, sparsity: float, sink: bool,
              scale: float = 0.0, sink_additive: bool = False) -> Tuple[np.ndarray, Selection]:
    """The whole hot path: permute -> pool -> score -> sink + top-k -> block-sparse
    attention -> unpermute.  Returns (O [B, N, heads, D] fp64, selection)."""
    qp, kp, vp = permute(q, g), permute(k, g), permute(v, g)
    sel = predict_mask(qp, kp, g, sparsity, sink, sink_additive)
    op = sparse_attention(qp, kp, vp, sel.idx, g, scale)
    return unpermute(op, g), sel


# ----------------------------------------------------------------------------- step schedule

DENSE, PREDICT, REUSE = 0, 1, 2


def schedule_action(total_steps: int, dense_fraction: float, predict_interval: int, step: int) -> int:
    """What the attention of diffusion step `step` (0-based, of `total_steps`) runs.

    The first ceil(dense_fraction * total_steps - 1e-6) steps are dense (RainFusion v1
    keeps the first 10 % of the timesteps dense: pith.science review, "Free parameters",
    dense timestep fraction).  After them a new mask is predicted on the first sparse step
    and then on every `predict_interval`-th one; the steps in between reuse the last
    predicted mask.  predict_interval = 1 predicts on every step, as the online method
    does; larger values are a deployment option the pages do not describe."""
    if total_steps < 1 or predict_interval < 1 or not (0.0 <= dense_fraction <= 1.0):
        raise ValueError("bad schedule")
    if not 0 <= step < total_steps:
        raise ValueError("step outside the schedule")
    n_dense = min(max(math.ceil(dense_fraction * total_steps - 1e-6), 0), total_steps)
    if step < n_dense:
        return DENSE
    return PREDICT if (step - n_dense) % predict_interval == 0 else REUSE
