"""Pins for the RainFusion v1 mask generators of the oracle (head patterns, ARM recall,
classification, RainFusion+ bandwidth), checked against hand-worked tables, uniform
attention, pair-by-pair brute force and planted heads.  CPU only."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O
from rf2_inputs import bf16_bits_to_f64, gen_pattern_heads

R1 = O.rf1
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def _g(T, H, W, wt, wh, ww, D=8, heads=1, B=1):
    return O.geom(B=B, heads=heads, T=T, H=H, W=W, D=D, wt=wt, wh=wh, ww=ww)


def test_lists_match_hand_worked_table():
    g = _g(4, 4, 4, 1, 2, 2)
    for ln in _lines("rf1_lists.txt"):
        lhs, rhs = ln.split(":")
        cls, param, row = map(int, lhs.split())
        want = [int(x) for x in rhs.split()]
        assert [j for j in range(g.Nb) if R1.rf1_keeps(g, cls, param, row, j)] == want, ln
        lists = R1.rf1_lists(g, np.array([[cls]]), np.array([[param]]))
        assert lists[0][0][row].tolist() == want, ln


@pytest.mark.parametrize("shape", [(4, 4, 4, 1, 2, 2), (3, 7, 9, 2, 4, 4), (5, 9, 6, 1, 8, 2)])
def test_keep_matrix_equals_pair_definition(shape):
    g = _g(*shape)
    for cls, params in ((R1.TEMPORAL, (0, 1, 3)), (R1.SPATIAL, (0, 1, 2)), (R1.TEXTURAL, (2, 3))):
        for prm in params:
            m = R1.rf1_keep_matrix(g, cls, prm)
            ref = np.array([[R1.rf1_keeps(g, cls, prm, i, j) for j in range(g.Nb)] for i in range(g.Nb)])
            np.testing.assert_array_equal(m, ref)


def test_radius_and_default_band_share():
    """floor(b * C): the default half-width 1/4 of an axis keeps about 7/16 of the pairs
    (the pages' 9/16 reduction) once the axis has many blocks."""
    assert R1.rf1_radius(0.25, 4) == 1 and R1.rf1_radius(0.125, 4) == 0 and R1.rf1_radius(0.5, 11) == 5
    assert R1.rf1_radius(0.3, 10) == 3   # 0.3 * 10 is 2.9999999999999996 in binary
    g = _g(1, 1, 1, 1, 1, 1)
    C = 400
    R = R1.rf1_radius(0.25, C)
    kept = sum(1 for i in range(C) for j in range(C) if abs(i - j) <= R) / C ** 2
    assert abs(kept - 7 / 16) < 5e-3
    del g


def _frac(x):
    return float(Fraction(x))


def test_uniform_attention_recall_matches_hand_worked_table():
    for ln in _lines("rf1_uniform_recall.txt"):
        geo, loc, glo = ln.split(":")
        T, H, W, wt, wh, ww, omega = map(int, geo.split())
        g = _g(T, H, W, wt, wh, ww, D=4)
        p = R1.Rf1Params(omega=omega)
        q = np.zeros((1, g.N, 1, 4))
        k = np.random.default_rng(0).standard_normal((1, g.N, 1, 4))
        rec = R1.rf1_recall(q, k, g, p)
        np.testing.assert_allclose(rec[0, 0, R1.LOCAL], [_frac(x) for x in loc.split()], rtol=0, atol=1e-13)
        np.testing.assert_allclose(rec[0, 0, R1.GLOBAL], [_frac(x) for x in glo.split()], rtol=0, atol=1e-13)


def test_recall_brute_force_pair_by_pair():
    g = _g(3, 5, 6, 1, 2, 4, D=4, heads=2)
    p = R1.Rf1Params(omega=2)
    rng = np.random.default_rng(4)
    q = rng.standard_normal((1, g.N, 2, 4)) * 1.5
    k = rng.standard_normal((1, g.N, 2, 4)) * 1.5
    rec = R1.rf1_recall(q, k, g, p)
    for h in range(2):
        for pattern, samples in ((R1.LOCAL, list(range(g.H * g.W))), (R1.GLOBAL, list(range(0, g.N, 2)))):
            for l, bw in enumerate(p.levels()):
                total = 0.0
                for a in samples:
                    ta, ra = divmod(a, g.H * g.W)
                    logits = [sum(q[0, a, h, d] * k[0, b, h, d] for d in range(4)) / 2.0 for b in samples]
                    mx = max(logits)
                    w = [math.exp(x - mx) for x in logits]
                    keep = 0.0
                    for b, wb in zip(samples, w):
                        tbb, rb = divmod(b, g.H * g.W)
                        if pattern == R1.LOCAL:
                            swa = (ra // g.W // g.wh) * g.nbw + (ra % g.W) // g.ww
                            swb = (rb // g.W // g.wh) * g.nbw + (rb % g.W) // g.ww
                            inside = abs(swa - swb) <= math.floor(bw * g.nbh * g.nbw + 1e-6)
                        else:
                            inside = abs(ta // g.wt - tbb // g.wt) <= math.floor(bw * g.nbt + 1e-6)
                        keep += wb if inside else 0.0
                    total += keep / sum(w)
                assert abs(rec[0, h, pattern, l] - total / len(samples)) < 1e-12


def test_recall_of_the_keep_everything_band_is_one():
    g = _g(2, 4, 4, 1, 2, 2, D=4)
    p = R1.Rf1Params(bandwidth=1.0)
    rng = np.random.default_rng(1)
    rec = R1.rf1_recall(rng.standard_normal((1, g.N, 1, 4)), rng.standard_normal((1, g.N, 1, 4)), g, p)
    np.testing.assert_allclose(rec[0, 0, :, 0], 1.0, atol=1e-14)
    assert np.all(np.diff(rec[0, 0, :, 1:], axis=-1) >= -1e-15)    # nested bands: recall grows


def _planted(kinds, dynamic=False, T=4, H=8, W=8, D=32, wt=1, wh=4, ww=4):
    g = _g(T, H, W, wt, wh, ww, D=D, heads=len(kinds))
    q, k, _ = (bf16_bits_to_f64(a) for a in gen_pattern_heads(1, T, H, W, len(kinds), D, 77, kinds))
    p = R1.Rf1Params(dynamic=dynamic)
    return g, p, R1.rf1_predict_mask(q, k, g, p)


def test_planted_heads_are_classified_as_planted():
    g, p, (idx, cnt, cls, param, rec) = _planted("tsxts")
    assert cls[0].tolist() == [R1.TEMPORAL, R1.SPATIAL, R1.TEXTURAL, R1.TEMPORAL, R1.SPATIAL]
    assert np.all(rec[0, [0, 3], R1.LOCAL, 0] > 0.99)            # own location in frame 0
    assert np.all(rec[0, [1, 4], R1.GLOBAL, 0] > 0.99)           # own frame
    assert rec[0, 2, R1.LOCAL, 0] < 0.9 and rec[0, 2, R1.GLOBAL, 0] < 0.9
    # static radius floor(0.25 * C), tau for textural
    assert param[0].tolist() == [R1.rf1_radius(0.25, 4), R1.rf1_radius(0.25, 4), 2,
                                 R1.rf1_radius(0.25, 4), R1.rf1_radius(0.25, 4)]
    kmax = R1.rf1_kmax(g, p)
    assert idx.shape[-1] == kmax and np.all(cnt <= kmax)
    for h in range(5):
        for i in range(g.Nb):
            row = idx[0, h, i, :cnt[0, h, i]]
            assert np.all(np.diff(row) > 0) and np.all(idx[0, h, i, cnt[0, h, i]:] == -1)


def test_rainfusion_plus_picks_the_smallest_band_that_keeps_the_target():
    _, _, (_, _, cls, param, rec) = _planted("tsx", dynamic=True)
    # planted temporal / spatial heads keep > 90 % even in the narrowest band
    assert cls[0].tolist() == [R1.TEMPORAL, R1.SPATIAL, R1.TEXTURAL]
    assert param[0].tolist() == [R1.rf1_radius(0.125, 4), R1.rf1_radius(0.125, 4), 2]
    # a head whose recall only reaches the target at the widest level
    g = _g(4, 8, 8, 1, 4, 4)
    rec = np.zeros((1, 1, 2, 4))
    rec[0, 0, R1.LOCAL] = [0.95, 0.5, 0.95, 0.97]
    p = R1.Rf1Params(dynamic=True, alpha=0.9, recall_target=0.96)
    cls, param = R1.rf1_classify(rec, g, p)
    assert cls[0, 0] == R1.TEMPORAL and param[0, 0] == R1.rf1_radius(0.5, 4)
    rec[0, 0, R1.LOCAL] = [0.95, 0.5, 0.95, 0.95]                   # none reaches 0.96: widest
    assert R1.rf1_classify(rec, g, p)[1][0, 0] == R1.rf1_radius(0.5, 4)
    rec[0, 0, R1.LOCAL] = [0.95, 0.965, 0.97, 0.99]                 # the narrowest suffices
    assert R1.rf1_classify(rec, g, p)[1][0, 0] == R1.rf1_radius(0.125, 4)


def test_classification_order_and_threshold():
    """Temporal is tested first, then spatial; a recall equal to alpha passes."""
    g = _g(4, 8, 8, 1, 4, 4)
    p = R1.Rf1Params(alpha=0.8)
    rec = np.zeros((1, 3, 2, 4))
    rec[0, 0, :, 0] = [0.8, 0.95]      # both pass: temporal wins
    rec[0, 1, :, 0] = [0.79, 0.8]      # spatial
    rec[0, 2, :, 0] = [0.79, 0.79]     # textural
    cls, _ = R1.rf1_classify(rec, g, p)
    assert cls[0].tolist() == [R1.TEMPORAL, R1.SPATIAL, R1.TEXTURAL]


def test_kmax_matches_hand_worked_counts():
    """Grid 4x4x4, windows (1, 2, 2): nbt = 4, P = 4 windows per slab.  Static 1/4: a
    temporal row keeps 4 slabs x (windows within 1) <= 4 x 3 = 12, a spatial row
    (slabs within 1) x 4 <= 3 x 4 = 12, textural tau 2 keeps 4 x 2 = 8: kmax 12.  With
    RainFusion+ the widest level 1/2 gives radius 2: 4 x 4 = 16 either way."""
    g = _g(4, 4, 4, 1, 2, 2)
    assert R1.rf1_kmax(g, R1.Rf1Params()) == 12
    assert R1.rf1_kmax(g, R1.Rf1Params(dynamic=True)) == 16
    assert R1.rf1_kmax(g, R1.Rf1Params(bandwidth=0.125, tau=3)) == 4   # radius 0: 4 slabs x 1, 1 x 4; tau 3: 4 x 1
