"""Pins for the fp64 CPU oracle, checked against things other than the oracle itself:
hand-worked golden tables, closed forms, brute force on tiny inputs, an independent
library (torch SDPA in fp64) and invariants.  CPU only."""
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from rf2_inputs import WORKLOADS, bf16_bits_to_f64, f32_to_bf16_bits, gen_tensor

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _g(B=1, heads=1, T=2, H=4, W=4, D=8, wt=1, wh=2, ww=2):
    return O.geom(B=B, heads=heads, T=T, H=H, W=W, D=D, wt=wt, wh=wh, ww=ww)


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


# ----------------------------------------------------------------------------- permutation

def test_permutation_matches_hand_worked_tables():
    for ln in _golden_lines("permute_small.txt"):
        lhs, rhs = ln.split(":")
        T, H, W, wt, wh, ww = map(int, lhs.split())
        expect = np.array(list(map(int, rhs.split())))
        g = _g(T=T, H=H, W=W, wt=wt, wh=wh, ww=ww)
        assert g.Npad == len(expect)
        np.testing.assert_array_equal(O.position_to_token(g), expect)
        pos = O.window_positions(g).reshape(-1)
        # forward map: token n sits at the position where the table lists n
        for n in range(g.N):
            assert expect[pos[n]] == n
        # permute of a tensor holding its own raster index reproduces the table
        x = np.arange(g.N, dtype=np.float64).reshape(1, g.N, 1, 1) + 1.0
        xp = O.permute(x, g)[0, :, 0, 0]
        np.testing.assert_array_equal(xp, np.where(expect >= 0, expect + 1.0, 0.0))


def test_permutation_brute_force_window_membership():
    # every block holds exactly its window's coordinates, in row-major order
    g = _g(T=5, H=7, W=9, wt=2, wh=4, ww=4)
    tok = O.position_to_token(g)
    for blk in range(g.Nb):
        tb = blk // (g.nbh * g.nbw)
        hb = (blk // g.nbw) % g.nbh
        wb = blk % g.nbw
        expect = []
        for dt in range(g.wt):
            for dh in range(g.wh):
                for dw in range(g.ww):
                    t, h, w = tb * g.wt + dt, hb * g.wh + dh, wb * g.ww + dw
                    ok = t < g.T and h < g.H and w < g.W
                    expect.append((t * g.H + h) * g.W + w if ok else -1)
        np.testing.assert_array_equal(tok[blk * g.blk:(blk + 1) * g.blk], expect)


@pytest.mark.parametrize("shape", [(4, 16, 16, 1, 8, 8), (3, 7, 10, 2, 4, 4), (2, 64, 64, 1, 8, 16)])
def test_unpermute_inverts_permute(shape):
    T, H, W, wt, wh, ww = shape
    g = _g(B=2, heads=3, T=T, H=H, W=W, D=4, wt=wt, wh=wh, ww=ww)
    x = np.random.default_rng(0).standard_normal((2, g.N, 3, 4))
    xp = O.permute(x, g)
    np.testing.assert_array_equal(O.unpermute(xp, g), x)
    assert np.all(xp[:, ~O.position_valid(g)] == 0.0)
    # every real token appears exactly once
    assert O.position_valid(g).sum() == g.N


def test_sink_blocks_are_first_temporal_window():
    g = _g(T=5, H=7, W=9, wt=2, wh=4, ww=4)
    tok = O.position_to_token(g)
    for b in O.sink_blocks(g):
        toks = tok[b * g.blk:(b + 1) * g.blk]
        toks = toks[toks >= 0]
        assert np.all(toks // (g.H * g.W) < g.wt)
    # and no other block holds a frame-0 token
    others = [b for b in range(g.Nb) if b not in set(O.sink_blocks(g).tolist())]
    for b in others:
        toks = tok[b * g.blk:(b + 1) * g.blk]
        assert np.all(toks[toks >= 0] // (g.H * g.W) >= g.wt)


# ----------------------------------------------------------------------------- pooling

def test_pool_constant_field_and_planted_block_constants():
    g = _g(B=1, heads=2, T=3, H=5, W=6, D=4, wt=2, wh=4, ww=4)
    x = np.full((1, g.N, 2, 4), 3.25)
    np.testing.assert_allclose(O.pool(O.permute(x, g), g), 3.25, rtol=0, atol=0)
    # plant a distinct constant in each block (by writing into the permuted tensor)
    xp = np.zeros((1, g.Npad, 2, 4))
    vals = np.arange(g.Nb, dtype=np.float64) * 1.5 - 4.0
    for b in range(g.Nb):
        xp[0, b * g.blk:(b + 1) * g.blk] = vals[b]
    got = O.pool(xp, g)
    for b in range(g.Nb):
        np.testing.assert_allclose(got[0, :, b], vals[b], rtol=0, atol=1e-15)


def test_pool_ignores_pad_rows_and_divides_by_real_count():
    g = _g(B=1, heads=1, T=1, H=3, W=3, D=2, wt=1, wh=2, ww=2)
    x = np.arange(g.N * 2, dtype=np.float64).reshape(1, g.N, 1, 2)
    xp = O.permute(x, g)
    base = O.pool(xp, g)
    xp_dirty = xp.copy()
    xp_dirty[:, ~O.position_valid(g)] = 1e6
    np.testing.assert_array_equal(O.pool(xp_dirty, g), base)
    # block 1 holds tokens 2 and 5 only (see the golden table): mean of their values
    np.testing.assert_allclose(base[0, 0, 1], (x[0, 2, 0] + x[0, 5, 0]) / 2)
    np.testing.assert_allclose(base[0, 0, 3], x[0, 8, 0])
    np.testing.assert_array_equal(O.block_valid_counts(g), [4, 2, 2, 1])


# ----------------------------------------------------------------------------- scores and selection

def test_pooled_scores_one_hot_closed_form():
    D = 8
    qbar = np.zeros((1, 1, 3, D))
    kbar = np.zeros((1, 1, 4, D))
    for i in range(3):
        qbar[0, 0, i, i] = 2.0
    for j in range(4):
        kbar[0, 0, j, j % D] = float(j + 1)
    s = O.pooled_scores(qbar, kbar, 1 / math.sqrt(D))
    expect = np.zeros((3, 4))
    for i in range(3):
        expect[i, i] = 2.0 * (i + 1) / math.sqrt(D)
    np.testing.assert_allclose(s[0, 0], expect, rtol=1e-15)


def test_kept_counts_match_hand_worked_values():
    for ln in _golden_lines("kept_counts.txt"):
        lhs, rhs = ln.split(":")
        f = lhs.split()
        T, H, W, wt, wh, ww = map(int, f[1:7])
        s, sink = float(f[7]), bool(int(f[8]))
        Nb, ns, kin, kadd = map(int, rhs.split())
        g = _g(T=T, H=H, W=W, wt=wt, wh=wh, ww=ww, D=8)
        assert g.Nb == Nb
        assert (len(O.sink_blocks(g)) if sink else 0) == ns
        assert O.kept_count(g, s, sink) == kin
        assert O.kept_count(g, s, sink, sink_additive=True) == kadd


def _rank_brute_force(row, cand, m):
    """Block j is chosen iff fewer than m candidates beat it (higher score, or equal
    score and lower id): the definition of top-m with ties to the lower id."""
    chosen = []
    for j in cand:
        beats = sum(1 for k in cand if row[k] > row[j] or (row[k] == row[j] and k < j))
        if beats < m:
            chosen.append(j)
    return chosen


@pytest.mark.parametrize("sparsity,sink,additive", [(0.8, True, False), (0.5, True, True),
                                                    (0.6, False, False), (0.0, True, False)])
def test_selection_against_rank_brute_force(sparsity, sink, additive):
    g = _g(B=2, heads=2, T=4, H=8, W=8, D=4, wt=1, wh=4, ww=4)
    rng = np.random.default_rng(7)
    s = rng.standard_normal((2, 2, g.Nb, g.Nb))
    s[0, 0, 0, 5] = s[0, 0, 0, 9] = s[0, 0, 0, 13] = 3.0  # exact ties
    s[1, 1, 2] = 0.5  # a fully tied row
    sel = O.select_blocks(s, g, sparsity, sink, additive)
    sinks = set(O.sink_blocks(g).tolist()) if sink else set()
    cand = [j for j in range(g.Nb) if j not in sinks]
    m = sel.kept - len(sinks)
    for b in range(2):
        for h in range(2):
            for i in range(g.Nb):
                expect = sorted(list(sinks) + _rank_brute_force(s[b, h, i], cand, m))
                assert list(sel.idx[b, h, i]) == expect


def test_selection_planted_one_hot_means():
    # Q block means all-ones, K block means one-hot with a planted magnitude v_j:
    # s_ij = v_j / sqrt(D), so the non-sink choice is the m largest v_j.
    g = _g(B=1, heads=1, T=4, H=8, W=8, D=16, wt=1, wh=4, ww=4)  # Nb=16, sink 4
    v = np.array([5, 1, 9, 2, 7, 3, 8, 6, 0.5, 4, 11, 10, 12, 2.5, 1.5, 13.0])
    qp = np.ones((1, g.Npad, 1, g.D))
    kp = np.zeros((1, g.Npad, 1, g.D))
    for j in range(g.Nb):
        kp[0, j * g.blk:(j + 1) * g.blk, 0, j % g.D] = v[j]
    sel = O.predict_mask(qp, kp, g, sparsity=0.5, sink=True)
    assert sel.kept == 8
    # non-sink blocks 4..15 ranked by v: 15(13),12(12),10(11),11(10) -> top 4
    assert list(sel.idx[0, 0, 0]) == [0, 1, 2, 3, 10, 11, 12, 15]
    # the cut (v=10) is far from the next score (v=8): no near-cut blocks
    assert all(len(n) == 0 for n in sel.near_cut)


def test_selection_invariants_on_generated_inputs():
    wl = WORKLOADS["tiny"]
    g = O.geom(**wl.geom())
    q, k = (bf16_bits_to_f64(gen_tensor(1, wl.T, wl.H, wl.W, wl.heads, wl.D, s)) for s in (11, 12))
    for additive in (False, True):
        sel = O.predict_mask(O.permute(q, g), O.permute(k, g), g, 0.8, True, additive)
        for row in sel.idx.reshape(-1, sel.kept):
            assert np.all(np.diff(row) > 0)
            assert set(O.sink_blocks(g).tolist()) <= set(row.tolist())
            assert len(row) == O.kept_count(g, 0.8, True, additive)


def test_near_cut_window_contains_ties_at_the_cut():
    g = _g(B=1, heads=1, T=2, H=4, W=8, D=4, wt=1, wh=4, ww=4)  # Nb = 4, sink 2
    s = np.array([[[[0.0, 0.0, 1.0, 1.0 + 1e-7]]]] * 1).reshape(1, 1, 1, 4)
    s = np.repeat(s, g.Nb, axis=2)
    sel = O.select_blocks(s, g, 0.25, True)  # K = 3 -> one of blocks 2, 3
    assert list(sel.idx[0, 0, 0]) == [0, 1, 3]
    assert sel.near_cut[0] == {2, 3}
    assert sel.near_cut_strict[0] == {2, 3}


def test_near_cut_floor_is_reported_apart_from_the_strict_window():
    # Cut near zero relative to the row's largest score: the strict window (1e-4 * |c|)
    # is far narrower than the floor (1e-4 * 1e-2 * max|s|).  Blocks 4 and 5 straddle the
    # cut c = 0 (scores +-1e-7); block 3 (score 5e-7) lies inside the floor
    # 1e-4 * 1e-2 * 100 = 1e-4 but outside the strict window of 1e-4 * |c| = 0.
    g = _g(B=1, heads=1, T=1, H=4, W=24, D=4, wt=1, wh=4, ww=4)  # Nb = 6, sink 6 (T = 1)
    row = np.array([100.0, 50.0, 20.0, 5e-7, 1e-7, -1e-7])
    s = np.repeat(row.reshape(1, 1, 1, 6), g.Nb, axis=2)
    sel = O.select_blocks(s, g, 1.0 - 5.0 / 6.0, False)  # K = 5: block 5 dropped
    assert list(sel.idx[0, 0, 0]) == [0, 1, 2, 3, 4]
    assert sel.near_cut[0] == {3, 4, 5}
    assert sel.near_cut_strict[0] == set()  # |c| = 0: the strict window is empty


# ----------------------------------------------------------------------------- attention

def _rand_qkv(g, seed=0):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((g.B, g.N, g.heads, g.D)) for _ in range(3)]


def test_zero_sparsity_equals_dense_attention_brute_force_and_sdpa():
    g = _g(B=1, heads=2, T=3, H=5, W=6, D=8, wt=2, wh=4, ww=4)  # ragged padding on all axes
    q, k, v = _rand_qkv(g, 1)
    scale = 1 / math.sqrt(g.D)
    out, sel = O.attention(q, k, v, g, sparsity=0.0, sink=True)
    assert sel.kept == g.Nb
    # brute force: explicit double loop softmax
    ref = np.zeros_like(q)
    for h in range(g.heads):
        for n in range(g.N):
            z = np.array([np.dot(q[0, n, h], k[0, m, h]) * scale for m in range(g.N)])
            p = np.exp(z - z.max())
            ref[0, n, h] = (p / p.sum()) @ v[0, :, h]
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    # independent library: torch SDPA in fp64 on the CPU
    tq, tk, tv = (torch.from_numpy(a).permute(0, 2, 1, 3) for a in (q, k, v))
    sd = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(out, sd, rtol=0, atol=1e-12)


@pytest.mark.parametrize("sparsity,sink", [(0.8, True), (0.6, False), (0.5, True)])
def test_sparse_equals_masked_dense(sparsity, sink):
    g = _g(B=1, heads=2, T=4, H=6, W=7, D=8, wt=1, wh=4, ww=4)
    q, k, v = _rand_qkv(g, 2)
    qp, kp, vp = (O.permute(a, g) for a in (q, k, v))
    sel = O.predict_mask(qp, kp, g, sparsity, sink)
    a = O.sparse_attention(qp, kp, vp, sel.idx, g)
    b = O.masked_dense_attention(qp, kp, vp, sel.idx, g)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_attention_closed_forms():
    g = _g(B=1, heads=1, T=2, H=5, W=5, D=4, wt=1, wh=4, ww=4)
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, g.N, 1, 4))
    k = rng.standard_normal((1, g.N, 1, 4))
    # constant V -> output equals that constant
    v = np.tile(np.array([1.5, -2.0, 0.25, 7.0]), (1, g.N, 1, 1))
    out, _ = O.attention(q, k, v, g, 0.5, True)
    np.testing.assert_allclose(out, v, rtol=0, atol=1e-13)
    # Q = 0 -> uniform weights: mean of V over the real keys of the kept blocks
    v = rng.standard_normal((1, g.N, 1, 4))
    qp, kp, vp = (O.permute(a, g) for a in (np.zeros_like(q), k, v))
    idx = np.array([[[[0, 3]] * g.Nb]], dtype=np.int32)
    op = O.sparse_attention(qp, kp, vp, idx, g)
    valid = O.position_valid(g)
    rows = [r for j in (0, 3) for r in range(j * g.blk, (j + 1) * g.blk) if valid[r]]
    np.testing.assert_allclose(op[0, 0, 0], vp[0, rows, 0].mean(axis=0), rtol=0, atol=1e-14)
    # a single kept block whose keys are identical -> uniform average of its values
    kp2 = kp.copy()
    kp2[0, 2 * g.blk:3 * g.blk] = kp2[0, 2 * g.blk]
    idx1 = np.full((1, 1, g.Nb, 1), 2, dtype=np.int32)
    op1 = O.sparse_attention(O.permute(q, g), kp2, vp, idx1, g)
    rows2 = [r for r in range(2 * g.blk, 3 * g.blk) if valid[r]]
    np.testing.assert_allclose(op1[0, 5, 0], vp[0, rows2, 0].mean(axis=0), rtol=0, atol=1e-13)


def test_attention_is_permutation_equivariant_in_batch_and_heads():
    g = _g(B=2, heads=3, T=2, H=8, W=8, D=4, wt=1, wh=4, ww=4)
    q, k, v = _rand_qkv(g, 4)
    out, sel = O.attention(q, k, v, g, 0.5, True)
    perm = [2, 0, 1]
    out2, sel2 = O.attention(q[::-1][:, :, perm], k[::-1][:, :, perm], v[::-1][:, :, perm], g, 0.5, True)
    np.testing.assert_allclose(out2, out[::-1][:, :, perm], rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------- input generator

def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e38, np.float32(1 + 2**-8)], dtype=np.float32)
    bits = f32_to_bf16_bits(vals)
    back = bf16_bits_to_f64(bits)
    t = torch.from_numpy(vals).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(back, t)


def test_generator_is_seeded_and_structured():
    a = gen_tensor(1, 2, 8, 8, 2, 16, seed=5)
    b = gen_tensor(1, 2, 8, 8, 2, 16, seed=5)
    np.testing.assert_array_equal(a, b)
    x = bf16_bits_to_f64(a)
    assert abs(x.mean()) < 0.2 and 0.9 < x.std() < 1.4


# ----------------------------------------------------------------------------- step schedule

def _golden_schedules():
    path = os.path.join(os.path.dirname(__file__), "golden", "schedule_actions.txt")
    rows = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        total, frac, interval, acts = line.split()
        rows.append((int(total), float(frac), int(interval), acts))
    return rows


def test_schedule_matches_hand_worked_tables():
    code = {O.DENSE: "D", O.PREDICT: "P", O.REUSE: "R"}
    for total, frac, interval, acts in _golden_schedules():
        assert len(acts) == total
        got = "".join(code[O.schedule_action(total, frac, interval, s)] for s in range(total))
        assert got == acts, (total, frac, interval)


def test_schedule_invariants():
    for total in (1, 2, 7, 30, 50, 100):
        for frac in (0.0, 0.05, 0.1, 0.33, 1.0):
            for interval in (1, 2, 3, 5):
                acts = [O.schedule_action(total, frac, interval, s) for s in range(total)]
                n_dense = sum(a == O.DENSE for a in acts)
                assert n_dense == min(total, math.ceil(frac * total - 1e-6))
                assert all(a == O.DENSE for a in acts[:n_dense])          # dense steps lead
                if n_dense < total:
                    assert acts[n_dense] == O.PREDICT                     # a mask exists before reuse
                assert (O.REUSE in acts) == (interval > 1 and total - n_dense > 1)


# ----------------------------------------------------------------------------- no-permute ablation

def _np_g(T, H, W, wt, wh, ww, B=1, heads=1, D=8):
    return O.geom(B=B, heads=heads, T=T, H=H, W=W, D=D, wt=wt, wh=wh, ww=ww, no_permute=True)


def test_no_permute_matches_hand_worked_table():
    for ln in _golden_lines("no_permute_small.txt"):
        lhs, rhs = ln.split(":")
        f = lhs.split()
        T, H, W, wt, wh, ww = map(int, f[:6])
        s = float(f[6])
        Nb, Npad, last, ns, kin, kadd = map(int, rhs.split())
        g = _np_g(T, H, W, wt, wh, ww)
        assert (g.Nb, g.Npad) == (Nb, Npad)
        cnt = O.block_valid_counts(g)
        assert list(cnt[:-1]) == [g.blk] * (Nb - 1) and cnt[-1] == last
        assert list(O.sink_blocks(g)) == list(range(ns))
        assert O.kept_count(g, s, True) == kin
        assert O.kept_count(g, s, True, sink_additive=True) == kadd


def test_no_permute_keeps_raster_order_and_pads_the_tail():
    g = _np_g(2, 3, 5, 1, 2, 4, heads=2, D=3)
    # entries encode (b, token, head, d): the permuted tensor must hold token p at row p
    x = np.arange(1 * g.N * 2 * 3, dtype=np.float64).reshape(1, g.N, 2, 3) + 1.0
    xp = O.permute(x, g)
    assert xp.shape == (1, 32, 2, 3)
    np.testing.assert_array_equal(xp[:, :g.N], x)
    assert np.all(xp[:, g.N:] == 0)
    np.testing.assert_array_equal(O.unpermute(xp, g), x)
    assert list(O.position_to_token(g)[28:]) == [28, 29, -1, -1]


@pytest.mark.parametrize("T,H,W,blk", [(3, 4, 32, 64), (2, 8, 16, 128), (4, 2, 32, 64)])
def test_no_permute_equals_flat_grid_cut_into_one_row_windows(T, H, W, blk):
    """When a frame is a whole number of blocks, raster blocks are exactly the windows
    (1, 1, blk) of the grid (T, 1, H*W), whose sink (temporal window 0) is frame 0: the
    two geometries must give the same positions, sink, kept lists and outputs."""
    g_np = O.geom(B=1, heads=2, T=T, H=H, W=W, D=16, wt=1, wh=1, ww=blk, no_permute=True)
    g_w = O.geom(B=1, heads=2, T=T, H=1, W=H * W, D=16, wt=1, wh=1, ww=blk)
    assert (g_np.Nb, g_np.Npad) == (g_w.Nb, g_w.Npad)
    np.testing.assert_array_equal(O.window_positions(g_np).reshape(-1), O.window_positions(g_w).reshape(-1))
    np.testing.assert_array_equal(O.position_to_token(g_np), O.position_to_token(g_w))
    np.testing.assert_array_equal(O.sink_blocks(g_np), O.sink_blocks(g_w))
    rng = np.random.default_rng(T * 100 + W)
    q, k, v = (rng.standard_normal((1, T * H * W, 2, 16)) for _ in range(3))
    for s in (0.5, 0.8):
        a, sa = O.attention(q, k, v, g_np, s, True)
        b, sb = O.attention(q, k, v, g_w, s, True)
        np.testing.assert_array_equal(sa.idx, sb.idx)
        np.testing.assert_array_equal(a, b)


def test_no_permute_ragged_tail_is_masked():
    """A partial last block: its pad keys carry no weight (the tail query rows match
    dense attention restricted to the kept real tokens)."""
    g = O.geom(B=1, heads=1, T=3, H=10, W=13, D=8, wt=1, wh=8, ww=8, no_permute=True)
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((1, g.N, 1, 8)) for _ in range(3))
    out, sel = O.attention(q, k, v, g, 0.0, True)
    ref = O.dense_attention(q, k, v, 1 / math.sqrt(8))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    assert sel.kept == g.Nb == 7
