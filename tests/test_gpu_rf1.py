"""GPU parity of the RainFusion v1 mask generators (ARM recall on the tensor cores, head
classes, RainFusion+ bandwidth, kept lists) against the fp64 oracle, and the attention
they drive.  Recall within 2e-4; classes equal wherever the oracle's recall is not within
1e-3 of a threshold it is compared with; kept lists and counts bit-exact for those heads.
The class is also decided by the oracle from the kernel's own fp32 recalls (thresholds as
fp32 values): that decision, and its lists, must equal the kernel's on every head."""
import numpy as np
import pytest
import torch

import oracle as O
import image_diffusion_dits_b200 as rf2
from rf2_inputs import WORKLOADS, bf16_bits_to_f64, gen_pattern_heads, gen_qkv

from _util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu
R1 = O.rf1
RECALL_TOL = 2e-4
DECISION_GAP = 1e-3


def _decided(rec, p):
    """Heads whose class and radius the oracle decides away from every threshold."""
    ok = np.ones(rec.shape[:2], dtype=bool)
    for b in range(rec.shape[0]):
        for h in range(rec.shape[1]):
            vals = [abs(rec[b, h, 0, 0] - p.alpha), abs(rec[b, h, 1, 0] - p.alpha)]
            if p.dynamic:
                vals += [abs(x - p.recall_target) for x in rec[b, h, :, 1:].reshape(-1)]
            ok[b, h] = min(vals) > DECISION_GAP
    return ok


def _check(q, k, g, og, p, heads=None):
    idx, cnt, cls, rec = rf2.v1_predict_mask(to_dev(q), to_dev(k), g, p, checked=True)
    op = R1.Rf1Params(**{f: getattr(p, f) for f in ("bandwidth", "tau", "alpha", "omega", "dynamic",
                                                       "recall_target")})
    qf, kf = bf16_bits_to_f64(q), bf16_bits_to_f64(k)
    hs = list(range(og.heads)) if heads is None else heads
    og_h = O.geom(**{**og.__dict__, "heads": len(hs)})
    ref_rec = R1.rf1_recall(qf[:, :, hs], kf[:, :, hs], og_h, op)
    got_rec = rec.cpu().numpy()[:, hs].astype(np.float64)
    err = np.abs(got_rec - ref_rec).max()
    assert err <= RECALL_TOL, f"recall differs by {err:.2e}"
    ref_cls, ref_prm = R1.rf1_classify(ref_rec, og_h, op)
    dec = _decided(ref_rec, op)
    # The class is an integer decided from floating point: decided again by the oracle
    # from the kernel's own fp32 recalls against the thresholds as fp32 values, it must
    # match the kernel's class and lists on every head, near a threshold or not.
    op32 = R1.Rf1Params(**{**{f: getattr(op, f) for f in ("bandwidth", "tau", "omega", "dynamic")},
                           "alpha": float(np.float32(op.alpha)), "recall_target": float(np.float32(op.recall_target))})
    k_cls, k_prm = R1.rf1_classify(got_rec, og_h, op32)
    assert np.array_equal(cls.cpu().numpy()[:, hs], k_cls)
    k_lists = R1.rf1_lists(og_h, k_cls, k_prm)
    all_idx, all_cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(og.B):
        for hi, h in enumerate(hs):
            for i in range(og.Nb):
                want = k_lists[b][hi][i]
                assert all_idx[b, h, i, :len(want)].tolist() == want.tolist()
                assert int(all_cnt[b, h, i]) == len(want)
    gcls = cls.cpu().numpy()[:, hs]
    assert np.all(gcls[dec] == ref_cls[dec])
    lists = R1.rf1_lists(og_h, ref_cls, ref_prm)
    gidx, gcnt = idx.cpu().numpy()[:, hs], cnt.cpu().numpy()[:, hs]
    for b in range(og.B):
        for hi in range(len(hs)):
            if not dec[b, hi]:
                continue
            for i in range(og.Nb):
                want = lists[b][hi][i]
                assert gcnt[b, hi, i] == len(want)
                np.testing.assert_array_equal(gidx[b, hi, i, :len(want)], want)
                assert np.all(gidx[b, hi, i, len(want):] == -1)
    return idx, cnt, cls, rec, ref_rec, dec


PLANTED = [
    (dict(B=1, heads=5, T=4, H=16, W=16, D=64, wt=1, wh=8, ww=8), "tsxts", dict()),
    (dict(B=2, heads=3, T=5, H=9, W=17, D=128, wt=2, wh=8, ww=8), "sxt", dict(dynamic=True, omega=7)),
    (dict(B=1, heads=4, T=3, H=24, W=40, D=128, wt=1, wh=8, ww=8), "txst", dict(bandwidth=0.5, tau=3)),
    # window slots per frame: 32 (wt = 2, 64-token blocks), 128, and 16 (raster-order
    # local sample: a window's frame slice is not a whole number of 32-key chunks)
    (dict(B=1, heads=3, T=4, H=12, W=20, D=64, wt=2, wh=4, ww=8), "tsx", dict()),
    (dict(B=1, heads=3, T=3, H=16, W=40, D=128, wt=1, wh=8, ww=16), "stx", dict(dynamic=True)),
    (dict(B=1, heads=3, T=8, H=12, W=12, D=64, wt=4, wh=4, ww=4), "xts", dict()),
]


@pytest.mark.parametrize("geo,kinds,prm", PLANTED)
def test_v1_planted_heads(geo, kinds, prm):
    g, og = rf2.Geometry(**geo), O.geom(**geo)
    q, k, _ = gen_pattern_heads(geo["B"], geo["T"], geo["H"], geo["W"], geo["heads"], geo["D"], 400, kinds)
    p = rf2.V1Params(**prm)
    _, _, cls, rec, ref_rec, dec = _check(q, k, g, og, p)
    want = {"t": 0, "s": 1, "x": 2}
    assert dec.all()
    assert cls.cpu().numpy().tolist() == [[want[c] for c in kinds]] * geo["B"]
    print(geo, kinds, "max recall err", float(np.abs(rec.cpu().numpy() - ref_rec).max()))


def test_v1_unstructured_inputs_and_attention():
    """Smooth-field inputs (no planted pattern): recall and lists against the oracle, then
    block-sparse attention over the v1 lists (rows of different lengths) against the
    oracle's attention."""
    geo = dict(B=1, heads=3, T=5, H=9, W=17, D=128, wt=2, wh=8, ww=8)
    g, og = rf2.Geometry(**geo), O.geom(**geo)
    from rf2_inputs import gen_tensor
    q, k, v = (gen_tensor(1, 5, 9, 17, 3, 128, 60 + i) for i in range(3))
    for prm in (dict(), dict(alpha=0.3), dict(alpha=0.0, dynamic=True)):
        idx, cnt, cls, rec, ref_rec, dec = _check(q, k, g, og, rf2.V1Params(**prm))
    out = rf2.sparse_attn(to_dev(q), to_dev(k), to_dev(v), idx, cnt, g, checked=True, raster=True)
    got = to_f64(out)
    qf, kf, vf = (bf16_bits_to_f64(O.permute(a, og)) for a in (q, k, v))
    tok = O.position_to_token(og)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    got_rows, ref_rows = [], []
    for h in range(og.heads):
        for i in range(og.Nb):
            lst = gidx[0, h, i, :gcnt[0, h, i]]
            ref = O.attention_block(qf, kf, vf, og, 0, h, i, lst, 1 / np.sqrt(og.D))
            t = tok[i * og.blk:(i + 1) * og.blk]
            keep = t >= 0
            ref_rows.append(ref[keep])
            got_rows.append(got[0, t[keep], h])
    print(assert_close(np.concatenate(got_rows), np.concatenate(ref_rows), "v1 attention"))


def test_v1_wan720p_sampled_heads():
    """The 720p video shape (40 heads, 3600 local and 3600 global samples): recall of a few
    heads against the oracle, lists of the decided ones bit-exact."""
    wl = WORKLOADS["wan720p"]
    g, og = rf2.Geometry(**wl.geom()), O.geom(**wl.geom())
    q, k, _ = gen_qkv(wl)
    for prm in (dict(alpha=0.3), dict(alpha=0.5, dynamic=True)):
        _, _, cls, rec, ref_rec, dec = _check(q, k, g, og, rf2.V1Params(**prm), heads=[0, 17, 39])
        print(prm, cls.cpu().numpy().tolist(), "max recall err", float(np.abs(rec.cpu().numpy()[:, [0, 17, 39]]
                                                                                 - ref_rec).max()))


def test_v1_is_deterministic():
    geo = dict(B=1, heads=5, T=4, H=16, W=16, D=64, wt=1, wh=8, ww=8)
    g = rf2.Geometry(**geo)
    q, k, _ = gen_pattern_heads(1, 4, 16, 16, 5, 64, 401, "tsxts")
    a = rf2.v1_predict_mask(to_dev(q), to_dev(k), g)
    b = rf2.v1_predict_mask(to_dev(q), to_dev(k), g)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
