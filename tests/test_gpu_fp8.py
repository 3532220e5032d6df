"""GPU parity of the e4m3 variant: quantisation bit-exact against the oracle (codes and
scales), attention over the e4m3 operands against the oracle's attention over the same
dequantised tensors.  Tolerance of the attention (derived in the design notes from the
e4m3 rounding of P): max-abs 1e-1, relative L2 5e-2."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import fp8_oracle as F8
import image_diffusion_dits_b200 as rf2
from rf2_inputs import WORKLOADS, bf16_bits_to_f64, gen_qkv, gen_tensor

from _util import to_dev, to_f64

pytestmark = pytest.mark.gpu

FP8_MAX_ABS = 1e-1
FP8_REL_L2 = 5e-2

QUANT_SHAPES = [
    dict(B=2, heads=3, T=3, H=9, W=10, D=64, wt=1, wh=8, ww=8),
    dict(B=1, heads=2, T=5, H=9, W=17, D=128, wt=2, wh=8, ww=8),
    dict(B=1, heads=2, T=3, H=20, W=19, D=128, wt=1, wh=8, ww=16),
]
ATTN_SHAPES = QUANT_SHAPES[1:]


def _bits(g, seed):
    return [gen_tensor(g.B, g.T, g.H, g.W, g.heads, g.D, seed + i) for i in range(3)]


def _oracle_quant(x, og):
    """Oracle codes in model order (uint8 patterns) and scales [B, heads, Nb]."""
    codes, scale, _ = F8.quantise_blocks(O.permute(bf16_bits_to_f64(x), og), og)
    return F8.e4m3_code(O.unpermute(codes, og)), scale


def _close(got, ref, what):
    err = np.abs(got - ref)
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert np.all(np.isfinite(got)), what
    assert err.max() <= FP8_MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    assert rel <= FP8_REL_L2, f"{what}: rel-L2 {rel:.3e}"
    return {"max_abs": float(err.max()), "rel_l2": rel}


@pytest.mark.parametrize("shape", QUANT_SHAPES)
@pytest.mark.parametrize("no_permute", [False, True])
def test_quantize_bit_exact(shape, no_permute):
    g = rf2.Geometry(**shape, no_permute=no_permute)
    og = O.geom(**shape, no_permute=no_permute)
    q, k, v = _bits(g, 1400)
    q8, k8, v8, sc = rf2.quantize_fp8(to_dev(q), to_dev(k), to_dev(v), g)
    torch.cuda.synchronize()
    for t, (x, x8) in enumerate(((q, q8), (k, k8), (v, v8))):
        codes, scale = _oracle_quant(x, og)
        np.testing.assert_array_equal(x8.cpu().numpy(), codes)
        np.testing.assert_array_equal(sc[t].cpu().numpy(), scale)


def _ref_rows(quant, og, sel, rows):
    deq = [t[3] for t in quant]
    tok = O.position_to_token(og)
    sc = 1 / np.sqrt(og.D)
    out = []
    for (b, h, i) in rows:
        r = F8.fp8_attention_block(deq[0], deq[1], deq[2], og, b, h, i, sel.idx[b, h, i], sc)
        t = tok[i * og.blk:(i + 1) * og.blk]
        out.append((b, h, t[t >= 0], r[t >= 0]))
    return out


@pytest.mark.parametrize("shape", ATTN_SHAPES)
def test_fp8_attention_ragged(shape):
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    q, k, v = _bits(g, 1500)
    qf, kf, vf = (bf16_bits_to_f64(a) for a in (q, k, v))
    sel = O.predict_mask(O.permute(qf, og), O.permute(kf, og), og, 0.5, True)
    idx = torch.from_numpy(sel.idx).cuda()
    cnt = torch.full(sel.idx.shape[:3], sel.kept, dtype=torch.int32, device="cuda")
    q8, k8, v8, sc = rf2.quantize_fp8(to_dev(q), to_dev(k), to_dev(v), g)
    out = rf2.sparse_attn_fp8(q8, k8, v8, sc, idx, cnt, g, checked=True)
    got = to_f64(out)
    quant = F8.quantised_inputs(qf, kf, vf, og)
    rows = [(b, h, i) for b in range(og.B) for h in range(og.heads) for i in range(og.Nb)]
    g_rows, r_rows = [], []
    for b, h, toks, ref in _ref_rows(quant, og, sel, rows):
        g_rows.append(got[b, toks, h])
        r_rows.append(ref)
    stats = _close(np.concatenate(g_rows), np.concatenate(r_rows), "fp8 attention")
    exact = O.sparse_attention(*(O.permute(a, og) for a in (qf, kf, vf)), sel.idx, og)
    ex = O.unpermute(exact, og)
    print(shape, stats, "vs exact attention: rel-L2 %.3e" % (np.linalg.norm(got - ex) / np.linalg.norm(ex)))


def test_fp8_attention_end_to_end_wan720p_sampled():
    wl = WORKLOADS["wan720p"]
    g, og = rf2.Geometry(**wl.geom()), O.geom(**wl.geom())
    q, k, v = gen_qkv(wl)
    out, idx = rf2.attention(to_dev(q), to_dev(k), to_dev(v), g, wl.sparsity, wl.sink, return_idx=True,
                             checked=True, fp8=True)
    got = to_f64(out)
    gidx = idx.cpu().numpy()
    heads = [0, 21, 39]
    og1 = O.geom(**{**wl.geom(), "heads": 1})
    rng = np.random.default_rng(3)
    g_rows, r_rows, e_rows = [], [], []
    for h in heads:
        qf, kf, vf = (bf16_bits_to_f64(a[:, :, [h]]) for a in (q, k, v))
        quant = F8.quantised_inputs(qf, kf, vf, og1)
        deq = [t[3] for t in quant]
        qp, kp, vp = (O.permute(a, og1) for a in (qf, kf, vf))
        tok = O.position_to_token(og1)
        for i in sorted({int(x) for x in rng.integers(0, og.Nb, 6)} | {og.Nb - 1}):
            lst = gidx[0, h, i]
            r = F8.fp8_attention_block(deq[0], deq[1], deq[2], og1, 0, 0, i, lst, 1 / np.sqrt(og.D))
            e = O.attention_block(qp, kp, vp, og1, 0, 0, i, lst, 1 / np.sqrt(og.D))
            t = tok[i * og.blk:(i + 1) * og.blk]
            keep = t >= 0
            g_rows.append(got[0, t[keep], h])
            r_rows.append(r[keep])
            e_rows.append(e[keep])
    stats = _close(np.concatenate(g_rows), np.concatenate(r_rows), "wan720p fp8")
    gr, er = np.concatenate(g_rows), np.concatenate(e_rows)
    print("wan720p fp8", stats, "vs exact attention: rel-L2 %.3e" % (np.linalg.norm(gr - er) / np.linalg.norm(er)))


@pytest.mark.parametrize("shape,no_permute", [
    (dict(B=2, heads=2, T=3, H=9, W=17, D=128, wt=2, wh=8, ww=8), False),    # one launch per batch
    (dict(B=1, heads=2, T=3, H=10, W=13, D=128, wt=1, wh=8, ww=16), True),   # raster blocks, tail of 6
])
def test_fp8_attention_batches_and_raster_blocks(shape, no_permute):
    g = rf2.Geometry(**shape, no_permute=no_permute)
    og = O.geom(**shape, no_permute=no_permute)
    q, k, v = _bits(g, 1600)
    qf, kf, vf = (bf16_bits_to_f64(a) for a in (q, k, v))
    sel = O.predict_mask(O.permute(qf, og), O.permute(kf, og), og, 0.5, True)
    idx = torch.from_numpy(sel.idx).cuda()
    cnt = torch.full(sel.idx.shape[:3], sel.kept, dtype=torch.int32, device="cuda")
    q8, k8, v8, sc = rf2.quantize_fp8(to_dev(q), to_dev(k), to_dev(v), g)
    got = to_f64(rf2.sparse_attn_fp8(q8, k8, v8, sc, idx, cnt, g, checked=True))
    quant = F8.quantised_inputs(qf, kf, vf, og)
    rows = [(b, h, i) for b in range(og.B) for h in range(og.heads) for i in range(og.Nb)]
    g_rows, r_rows = [], []
    for b, h, toks, ref in _ref_rows(quant, og, sel, rows):
        g_rows.append(got[b, toks, h])
        r_rows.append(ref)
    print(shape, no_permute, _close(np.concatenate(g_rows), np.concatenate(r_rows), "fp8 attention"))


def test_fp8_empty_rows_and_bad_indices():
    """A row with no kept block writes zeros; ids outside [0, Nb) are skipped and reported
    (RF2_ERR_BAD_INDEX) while the valid ids of the row are still used."""
    shape = dict(B=1, heads=1, T=2, H=16, W=16, D=128, wt=2, wh=8, ww=8)
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    q, k, v = _bits(g, 1700)
    q8, k8, v8, sc = rf2.quantize_fp8(to_dev(q), to_dev(k), to_dev(v), g)
    idx = torch.tensor([[[[0, 1, 2, 3], [2, 99, -4, 3], [0, 1, 2, 3], [1, 3, 0, 2]]]], dtype=torch.int32,
                       device="cuda")
    cnt = torch.tensor([[[0, 4, 2, 1]]], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = rf2.sparse_attn_fp8(q8, k8, v8, sc, idx, cnt, g, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 5
    got = to_f64(out)
    quant = F8.quantised_inputs(*(bf16_bits_to_f64(a) for a in (q, k, v)), og)
    deq = [t[3] for t in quant]
    tok = O.position_to_token(og)
    t0 = tok[0:128]
    assert np.all(got[0, t0[t0 >= 0], 0] == 0)
    for i, lst in ((1, [2, 3]), (2, [0, 1]), (3, [1])):
        ref = F8.fp8_attention_block(deq[0], deq[1], deq[2], og, 0, 0, i, lst, 1 / np.sqrt(128))
        t = tok[i * 128:(i + 1) * 128]
        _close(got[0, t[t >= 0], 0], ref[t >= 0], f"row {i}")
