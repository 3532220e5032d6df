"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle on the same
seeded bf16 inputs.  Permutations and kept lists are compared bit-exactly (kept lists
outside the near-cut window); attention outputs within max-abs 2e-2 and relative-L2 1e-2."""
import numpy as np
import pytest
import torch

import oracle as O
import image_diffusion_dits_b200 as rf2
from rf2_inputs import WORKLOADS, bf16_bits_to_f64, gen_qkv, gen_tensor

from _util import assert_close, compare_lists, to_bits, to_dev, to_f64

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "video480p", "imgedit1024"]
LARGE = ["wan720p", "longvideo"]

_cache = {}


def _inputs(name):
    if name not in _cache:
        _cache.clear()
        _cache[name] = gen_qkv(WORKLOADS[name])
    return _cache[name]


def _geoms(name):
    wl = WORKLOADS[name]
    return wl, rf2.Geometry(**wl.geom()), O.geom(**wl.geom())


# Ragged shapes: padding on every axis, both block sizes, both head dims, batch > 1.
RAGGED = [
    dict(B=2, heads=3, T=3, H=7, W=10, D=64, wt=1, wh=8, ww=8),
    dict(B=1, heads=2, T=5, H=9, W=17, D=128, wt=2, wh=8, ww=8),
    dict(B=2, heads=1, T=3, H=13, W=9, D=128, wt=1, wh=8, ww=8),
    dict(B=1, heads=2, T=4, H=11, W=21, D=64, wt=2, wh=4, ww=16),
    dict(B=1, heads=1, T=1, H=8, W=8, D=64, wt=1, wh=8, ww=8),      # one block
    dict(B=1, heads=2, T=2, H=16, W=23, D=128, wt=1, wh=8, ww=16),
]


def _rand_bits(g, seed):
    return [gen_tensor(g.B, g.T, g.H, g.W, g.heads, g.D, seed + i) for i in range(3)]


# ----------------------------------------------------------------------------- permutation

@pytest.mark.parametrize("shape", [RAGGED[1], dict(B=1, heads=2, T=4, H=16, W=40, D=128, wt=2, wh=8, ww=8)])
@pytest.mark.parametrize("raster", [False, True])
def test_predict_mask_exact_ties_take_the_lowest_ids(shape, raster):
    """Every key block of a row with the same pooled score (K constant over the grid, so
    every block mean is that constant): the scores tie exactly, in fp64 and in the
    kernels' fp32, and the kept set must be the sink plus the lowest non-sink ids, bit
    for bit (the near-cut window would excuse every candidate here, so the lists are
    compared exactly)."""
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    q, _, _ = _rand_bits(g, 1500)
    rng = np.random.default_rng(1501)
    const = rng.standard_normal(g.D)
    kf = np.broadcast_to(const, (g.B, g.N, g.heads, g.D)).astype(np.float32)
    from rf2_inputs import f32_to_bf16_bits
    k = f32_to_bf16_bits(np.ascontiguousarray(kf))
    for s_, sink in ((0.5, True), (0.7, False), (0.8, True)):
        sel = O.predict_mask(bf16_bits_to_f64(O.permute(q, og)), bf16_bits_to_f64(O.permute(k, og)), og, s_, sink)
        if raster:
            idx, cnt = rf2.predict_mask(to_dev(q), to_dev(k), g, s_, sink, checked=True, raster=True)
        else:
            idx, cnt = rf2.predict_mask(to_dev(O.permute(q, og)), to_dev(O.permute(k, og)), g, s_, sink, checked=True)
        got = idx.cpu().numpy()
        assert np.array_equal(got, sel.idx), (s_, sink)
        assert np.all(cnt.cpu().numpy() == sel.kept)
        # the sink is blocks 0 .. nsink - 1, so the lowest ids of either kind are 0 .. kept - 1
        assert np.array_equal(got.reshape(-1, sel.kept), np.broadcast_to(np.arange(sel.kept), (got.size // sel.kept, sel.kept)))


# 192 blocks of 64 tokens, 48 of them the first-frame sink: 144 candidates per row, enough
# for the cut's histogram bin to overflow its 32 slots when the scores crowd together.
CUT_SHAPE = dict(B=1, heads=2, T=4, H=48, W=64, D=64, wt=1, wh=8, ww=8)


def _block_ids(og):
    """Window block of every model-order token, [N]."""
    t, h, w = np.meshgrid(np.arange(og.T), np.arange(og.H), np.arange(og.W), indexing="ij")
    nbh, nbw = -(-og.H // og.wh), -(-og.W // og.ww)
    return (((t // og.wt) * nbh + h // og.wh) * nbw + w // og.ww).reshape(-1)


@pytest.mark.parametrize("case", ["outlier_column", "levels3", "levels9"])
def test_predict_mask_cut_by_histogram_and_by_search(case):
    """Rows whose cut the top-k finds through its value histogram and rows where it must
    fall back to the bracketed search give the oracle's lists.  outlier_column: one key
    block scaled by 512 takes one end of every row's score range, so the other 143 scores
    share one or two of the 64 bins and the cut's bin overflows (search); the lists are
    compared outside the near-cut window.  levelsL: every key block mean is c u for one
    vector u and an integer c in [-(L-1)/2, (L-1)/2], so each row has L distinct scores,
    exact ties in fp64 and in the kernel's fp32, and the lists must equal the oracle's
    (lowest ids among equal scores) bit for bit: with 3 levels about 48 candidates share
    the cut's score (search), with 9 about 16 (histogram)."""
    from rf2_inputs import f32_to_bf16_bits
    g, og = rf2.Geometry(**CUT_SHAPE), O.geom(**CUT_SHAPE)
    q, k, _ = _rand_bits(g, 1600)
    rng = np.random.default_rng(1601)
    blocks = _block_ids(og)
    if case == "outlier_column":
        kf = bf16_bits_to_f64(k).astype(np.float32)
        kf[:, blocks == 100] *= 512.0   # a non-sink block; a power of two keeps bf16 exact
    else:
        u = rng.standard_normal((g.heads, g.D)).astype(np.float32)
        half = (int(case[len("levels"):]) - 1) // 2
        level = rng.integers(-half, half + 1, size=int(blocks.max()) + 1).astype(np.float32)
        kf = (level[blocks][None, :, None, None] * u[None, None]).astype(np.float32)
        kf = np.broadcast_to(kf, (g.B, g.N, g.heads, g.D))
    k = f32_to_bf16_bits(np.ascontiguousarray(kf))
    qp, kp = O.permute(q, og), O.permute(k, og)
    for s_, sink in ((0.8, True), (0.6, False), (0.9, True)):
        sel = O.predict_mask(bf16_bits_to_f64(qp), bf16_bits_to_f64(kp), og, s_, sink)
        idx, cnt = rf2.predict_mask(to_dev(q), to_dev(k), g, s_, sink, checked=True, raster=True)
        if case == "outlier_column":
            compare_lists(idx.cpu().numpy(), cnt.cpu().numpy(), sel)
        else:
            assert np.array_equal(idx.cpu().numpy(), sel.idx), (s_, sink)
            assert np.all(cnt.cpu().numpy() == sel.kept)


@pytest.mark.parametrize("shape", [
    # one temporal window: all 64 blocks are sink blocks, so no score is computed at all
    dict(B=1, heads=2, T=1, H=64, W=64, D=64, wt=1, wh=8, ww=8),
    # 32 sink blocks: the score columns start exactly at the sink boundary
    dict(B=1, heads=2, T=3, H=32, W=64, D=64, wt=1, wh=8, ww=8),
])
def test_predict_mask_score_columns_from_the_sink_boundary(shape):
    """The scores kernel computes only the columns from the sink count rounded down to 32
    (the top-k reads no sink column's score) and is not launched when every block is a
    sink block; the lists still equal the oracle's, with and without the sink."""
    for s_, sink in ((0.8, True), (0.5, True), (0.8, False)):
        _mask_case(shape, s_, sink, False, seed=1700)


@pytest.mark.parametrize("shape", RAGGED)
def test_permute_unpermute_ragged_bit_exact(shape):
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    x = _rand_bits(g, 101)[0]
    xd = to_dev(x)
    xp = rf2.permute(xd, g)
    np.testing.assert_array_equal(to_bits(xp), O.permute(x, og))
    back = rf2.unpermute(xp, g)
    np.testing.assert_array_equal(to_bits(back), x)


@pytest.mark.parametrize("name", SMALL + LARGE)
def test_permute_unpermute_workloads_bit_exact(name):
    wl, g, og = _geoms(name)
    q, _, _ = _inputs(name)
    xp = rf2.permute(to_dev(q), g)
    np.testing.assert_array_equal(to_bits(xp), O.permute(q, og))
    np.testing.assert_array_equal(to_bits(rf2.unpermute(xp, g)), q)


def test_permute_overwrites_pad_rows_with_zero():
    shape = RAGGED[0]
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    x = to_dev(_rand_bits(g, 7)[0])
    out = torch.full((g.B, g.Npad, g.heads, g.D), 3.0, dtype=torch.bfloat16, device="cuda")
    rf2.permute(x, g, out=out)
    pad = ~O.position_valid(og)
    assert torch.all(out[:, torch.from_numpy(pad).cuda()] == 0)


# ----------------------------------------------------------------------------- mask prediction

def _mask_case(name_or_shape, sparsity, sink, additive, seed=None):
    if isinstance(name_or_shape, str):
        wl, g, og = _geoms(name_or_shape)
        q, k, _ = _inputs(name_or_shape)
    else:
        g, og = rf2.Geometry(**name_or_shape), O.geom(**name_or_shape)
        q, k, _ = _rand_bits(g, seed)
    qp, kp = O.permute(q, og), O.permute(k, og)
    sel = O.predict_mask(bf16_bits_to_f64(qp), bf16_bits_to_f64(kp), og, sparsity, sink, additive)
    idx, cnt = rf2.predict_mask(to_dev(qp), to_dev(kp), g, sparsity, sink, additive,
                                kmax=sel.kept + 3, checked=True)
    return compare_lists(idx.cpu().numpy(), cnt.cpu().numpy(), sel)


@pytest.mark.parametrize("shape", RAGGED)
@pytest.mark.parametrize("additive", [False, True])
def test_predict_mask_ragged(shape, additive):
    for s, sink in ((0.8, True), (0.5, False), (0.0, True), (1.0, True)):
        _mask_case(shape, s, sink, additive, seed=300)


@pytest.mark.parametrize("name", SMALL + LARGE)
@pytest.mark.parametrize("additive", [False, True])
def test_predict_mask_workloads(name, additive):
    wl = WORKLOADS[name]
    for s in wl.sparsities:
        stats = _mask_case(name, s, wl.sink, additive)
        print(name, s, "additive" if additive else "in-budget", stats)


# ----------------------------------------------------------------------------- sparse attention

def _attn_case(g, og, q, k, v, sparsity, sink, heads=None, rows=None, scale=0.0):
    """Oracle kept lists feed both sides; compare all heads (or sampled (head, q-block))."""
    qp, kp, vp = (O.permute(a, og) for a in (q, k, v))
    qf, kf, vf = (bf16_bits_to_f64(a) for a in (qp, kp, vp))
    sel = O.predict_mask(qf, kf, og, sparsity, sink)
    idx = torch.from_numpy(sel.idx).cuda()
    cnt = torch.full(sel.idx.shape[:3], sel.kept, dtype=torch.int32, device="cuda")
    op = rf2.sparse_attn(to_dev(qp), to_dev(kp), to_dev(vp), idx, cnt, g, scale=scale, checked=True)
    got = to_f64(op)
    sc = O.default_scale(og.D, scale)
    valid = O.position_valid(og)
    if rows is None:
        hs = range(og.heads) if heads is None else heads
        rows = [(b, h, i) for b in range(og.B) for h in hs for i in range(og.Nb)]
    ref_rows, got_rows = [], []
    for (b, h, i) in rows:
        ref = O.attention_block(qf, kf, vf, og, b, h, i, sel.idx[b, h, i], sc)
        keep = valid[i * og.blk:(i + 1) * og.blk]
        ref_rows.append(ref[keep])
        got_rows.append(got[b, i * og.blk:(i + 1) * og.blk, h][keep])
    return assert_close(np.concatenate(got_rows), np.concatenate(ref_rows), "sparse_attn")


@pytest.mark.parametrize("shape", RAGGED)
def test_sparse_attn_ragged(shape):
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    q, k, v = (bf16_bits_to_f64(a) for a in _rand_bits(g, 500))
    bits = _rand_bits(g, 500)
    for s, sink in ((0.5, True), (0.0, False)):
        _attn_case(g, og, *bits, s, sink)


@pytest.mark.parametrize("name", SMALL)
def test_sparse_attn_small_workloads_all_rows(name):
    wl, g, og = _geoms(name)
    q, k, v = _inputs(name)
    stats = _attn_case(g, og, q, k, v, wl.sparsity, wl.sink)
    print(name, stats)


@pytest.mark.parametrize("name", LARGE)
def test_sparse_attn_large_workloads_sampled_rows(name):
    wl, g, og = _geoms(name)
    q, k, v = _inputs(name)
    rng = np.random.default_rng(17)
    rows = {(0, int(rng.integers(og.heads)), int(rng.integers(og.Nb))) for _ in range(20)}
    rows |= {(0, 0, 0), (0, og.heads - 1, og.Nb - 1), (0, 1, og.Nb - og.nbw)}  # first, last, partial
    stats = _attn_case(g, og, q, k, v, wl.sparsity, wl.sink, rows=sorted(rows))
    print(name, stats)


@pytest.mark.parametrize("sparsity", [0.0, 0.5, 0.7, 0.9])
def test_sparse_attn_longvideo_sweep_sampled_rows(sparsity):
    """The long-video sparsity sweep (960 blocks; 960 / 480 / 288 / 96 kept per row)."""
    wl, g, og = _geoms("longvideo")
    q, k, v = _inputs("longvideo")
    rng = np.random.default_rng(int(sparsity * 100) + 3)
    rows = {(0, int(rng.integers(og.heads)), int(rng.integers(og.Nb))) for _ in range(3)}
    rows |= {(0, 0, 0), (0, og.heads - 1, og.Nb - 1)}
    stats = _attn_case(g, og, q, k, v, sparsity, wl.sink, rows=sorted(rows))
    print("longvideo", sparsity, stats)


def test_attention_end_to_end_additive_sink():
    """The sink-outside-the-budget reading (RF2_SINK_ADDITIVE) through the fused call."""
    wl, g, og = _geoms("video480p")
    q, k, v = _inputs("video480p")
    out, idx = rf2.attention(to_dev(q), to_dev(k), to_dev(v), g, wl.sparsity, wl.sink, additive=True,
                             return_idx=True, checked=True)
    qf, kf, vf = (bf16_bits_to_f64(O.permute(a, og)) for a in (q, k, v))
    sel = O.predict_mask(qf, kf, og, wl.sparsity, wl.sink, True)
    gidx = idx.cpu().numpy()
    compare_lists(gidx, np.full(gidx.shape[:3], sel.kept), sel)
    got = to_f64(out)
    tok = O.position_to_token(og)
    got_rows, ref_rows = [], []
    sampled = near = 0
    for h in range(og.heads):
        for i in range(0, og.Nb, 7):
            # a row whose list differs near the cut (already checked above) is compared
            # with the oracle's attention over the list the kernel used
            lst = gidx[0, h, i]
            near += 0 if np.array_equal(lst, sel.idx[0, h, i]) else 1
            ref = O.attention_block(qf, kf, vf, og, 0, h, i, lst, 1 / np.sqrt(og.D))
            t = tok[i * og.blk:(i + 1) * og.blk]
            keep = t >= 0
            ref_rows.append(ref[keep])
            got_rows.append(got[0, t[keep], h])
            sampled += 1
    assert sampled == og.heads * len(range(0, og.Nb, 7)) and sampled > 0
    print("video480p additive", {"rows": sampled, "near_cut_rows": near},
          assert_close(np.concatenate(got_rows), np.concatenate(ref_rows), "additive"))


def test_sparse_attn_zero_sparsity_is_dense_attention():
    shape = dict(B=1, heads=2, T=3, H=9, W=10, D=64, wt=1, wh=8, ww=8)
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    q, k, v = _rand_bits(g, 900)
    out, idx = rf2.attention(to_dev(q), to_dev(k), to_dev(v), g, 0.0, True, return_idx=True)
    ref = O.dense_attention(*(bf16_bits_to_f64(a) for a in (q, k, v)), 1 / np.sqrt(g.D))
    assert_close(to_f64(out), ref, "dense")
    assert np.all(idx.cpu().numpy() == np.arange(og.Nb))


def test_sparse_attn_custom_scale():
    shape = RAGGED[1]
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    _attn_case(g, og, *_rand_bits(g, 910), 0.5, True, scale=0.05)


def test_sparse_attn_bad_index_is_skipped_and_reported():
    shape = dict(B=1, heads=1, T=2, H=16, W=16, D=64, wt=1, wh=8, ww=8)
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    q, k, v = _rand_bits(g, 920)
    qp, kp, vp = (to_dev(O.permute(a, og)) for a in (q, k, v))
    idx = torch.tensor([[[[0, 3, 99], [1, -5, 2]] + [[0, 1, 2]] * (og.Nb - 2)]], dtype=torch.int32,
                       device="cuda")
    cnt = torch.full((1, 1, og.Nb), 3, dtype=torch.int32, device="cuda")
    with pytest.raises(rf2.Rf2Error) as ei:
        rf2.sparse_attn(qp, kp, vp, idx, cnt, g, checked=True)
    assert ei.value.code == 5
    # the valid ids of the bad rows are still used
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    op = rf2.sparse_attn(qp, kp, vp, idx, cnt, g, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 5
    qf, kf, vf = (bf16_bits_to_f64(O.permute(a, og)) for a in (q, k, v))
    ref0 = O.attention_block(qf, kf, vf, og, 0, 0, 0, [0, 3], 1 / 8)
    ref1 = O.attention_block(qf, kf, vf, og, 0, 0, 1, [1, 2], 1 / 8)
    got = to_f64(op)
    assert_close(got[0, :64, 0], ref0, "row0")
    assert_close(got[0, 64:128, 0], ref1, "row1")


def test_sparse_attn_empty_row_writes_zeros_and_respects_cnt():
    shape = dict(B=1, heads=1, T=2, H=16, W=16, D=128, wt=2, wh=8, ww=8)
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    q, k, v = _rand_bits(g, 930)
    qp, kp, vp = (to_dev(O.permute(a, og)) for a in (q, k, v))
    idx = torch.tensor([[[[0, 1, 2, 3]] * og.Nb]], dtype=torch.int32, device="cuda")
    cnt = torch.tensor([[[0, 2, 4, 1]]], dtype=torch.int32, device="cuda")
    op = rf2.sparse_attn(qp, kp, vp, idx, cnt, g, checked=True)
    got = to_f64(op)
    assert np.all(got[0, :128] == 0)
    qf, kf, vf = (bf16_bits_to_f64(O.permute(a, og)) for a in (q, k, v))
    for i, lst in ((1, [0, 1]), (2, [0, 1, 2, 3]), (3, [0])):
        ref = O.attention_block(qf, kf, vf, og, 0, 0, i, lst, 1 / np.sqrt(128))
        assert_close(got[0, i * 128:(i + 1) * 128, 0], ref, f"row{i}")


# ----------------------------------------------------------------------------- fused path

@pytest.mark.parametrize("name", SMALL + ["wan720p"])
def test_attention_end_to_end(name):
    wl, g, og = _geoms(name)
    q, k, v = _inputs(name)
    out, idx = rf2.attention(to_dev(q), to_dev(k), to_dev(v), g, wl.sparsity, wl.sink,
                             return_idx=True, checked=True)
    qf, kf, vf = (bf16_bits_to_f64(O.permute(a, og)) for a in (q, k, v))
    sel = O.predict_mask(qf, kf, og, wl.sparsity, wl.sink)
    gidx = idx.cpu().numpy()
    stats = compare_lists(gidx, np.full(gidx.shape[:3], sel.kept), sel)
    got = to_f64(out)
    pos = O.window_positions(og).reshape(-1)
    rng = np.random.default_rng(5)
    heads = range(og.heads) if og.heads * og.Nb <= 2000 else rng.choice(og.heads, 2, replace=False)
    blocks = range(og.Nb) if og.heads * og.Nb <= 2000 else rng.choice(og.Nb, 12, replace=False)
    tok = O.position_to_token(og)
    got_rows, ref_rows = [], []
    sampled = near = 0
    for h in heads:
        for i in blocks:
            # a row whose list differs near the cut (compare_lists checked that it differs
            # only there) is compared with the oracle's attention over the kernel's list
            lst = gidx[0, h, i]
            near += 0 if np.array_equal(lst, sel.idx[0, h, i]) else 1
            ref = O.attention_block(qf, kf, vf, og, 0, h, i, lst, 1 / np.sqrt(og.D))
            t = tok[i * og.blk:(i + 1) * og.blk]
            keep = t >= 0
            ref_rows.append(ref[keep])
            got_rows.append(got[0, t[keep], h])
            sampled += 1
    assert sampled == len(heads) * len(blocks) and sampled > 0
    print(name, stats, {"rows_compared": sampled, "near_cut_rows": near},
          assert_close(np.concatenate(got_rows), np.concatenate(ref_rows), name))
    del pos


def test_attention_is_deterministic():
    wl, g, og = _geoms("video480p")
    q, k, v = (to_dev(a) for a in _inputs("video480p"))
    a = rf2.attention(q, k, v, g, 0.8, True)
    b = rf2.attention(q, k, v, g, 0.8, True)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


# ----------------------------------------------------------------------------- model-order (raster) path

@pytest.mark.parametrize("shape", RAGGED)
def test_predict_mask_raster_equals_window_order(shape):
    """Pooling straight from model order gives the same kept lists as pooling the
    permuted tensors (same rows summed in the same order)."""
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    q, k, _ = _rand_bits(g, 1300)
    for s, sink in ((0.8, True), (0.5, False)):
        a = rf2.predict_mask(to_dev(O.permute(q, og)), to_dev(O.permute(k, og)), g, s, sink, checked=True)
        b = rf2.predict_mask(to_dev(q), to_dev(k), g, s, sink, checked=True, raster=True)
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("name", SMALL + LARGE)
def test_predict_mask_raster_workloads(name):
    wl, g, og = _geoms(name)
    q, k, _ = _inputs(name)
    a = rf2.predict_mask(rf2.permute(to_dev(q), g), rf2.permute(to_dev(k), g), g, wl.sparsity, wl.sink,
                         checked=True)
    b = rf2.predict_mask(to_dev(q), to_dev(k), g, wl.sparsity, wl.sink, checked=True, raster=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("shape", RAGGED)
def test_sparse_attn_raster_equals_window_order(shape):
    """Window gathers and row scatters in model order give, bit for bit, the
    window-order kernel's output on permuted tensors, unpermuted."""
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    q, k, v = _rand_bits(g, 1400)
    qf, kf = (bf16_bits_to_f64(O.permute(a, og)) for a in (q, k))
    sel = O.predict_mask(qf, kf, og, 0.5, True)
    idx = torch.from_numpy(sel.idx).cuda()
    cnt = torch.full(sel.idx.shape[:3], sel.kept, dtype=torch.int32, device="cuda")
    win = rf2.sparse_attn(*(to_dev(O.permute(a, og)) for a in (q, k, v)), idx, cnt, g, checked=True)
    ras = rf2.sparse_attn(to_dev(q), to_dev(k), to_dev(v), idx, cnt, g, checked=True, raster=True)
    assert torch.equal(rf2.unpermute(win, g).view(torch.int16), ras.view(torch.int16))


@pytest.mark.parametrize("name", ["video480p", "wan720p"])
def test_sparse_attn_raster_workloads(name):
    wl, g, og = _geoms(name)
    q, k, v = (to_dev(a) for a in _inputs(name))
    idx, cnt = rf2.predict_mask(q, k, g, wl.sparsity, wl.sink, checked=True, raster=True)
    win = rf2.sparse_attn(rf2.permute(q, g), rf2.permute(k, g), rf2.permute(v, g), idx, cnt, g, checked=True)
    ras = rf2.sparse_attn(q, k, v, idx, cnt, g, checked=True, raster=True)
    assert torch.equal(rf2.unpermute(win, g).view(torch.int16), ras.view(torch.int16))


# ----------------------------------------------------------------------------- step schedule

def test_step_attention_follows_its_schedule():
    """Dense steps equal the fused call at 0 % sparsity, predict steps equal the fused
    call at the target sparsity, reuse steps attend with the layer's last predicted lists
    (bit for bit), and every layer keeps its own lists."""
    wl, g, og = _geoms("video480p")
    sched = rf2.Schedule(total_steps=10, dense_fraction=0.1, predict_interval=3)   # D P R R P R R P R R
    sa = rf2.StepAttention(g, 0.5, wl.sink, schedule=sched)
    inputs = {}
    for layer in (0, 1):
        for step in range(3):
            inputs[layer, step] = [to_dev(gen_tensor(g.B, g.T, g.H, g.W, g.heads, g.D, 7000 + 100 * layer + 10 * step + i))
                                   for i in range(3)]
    same = lambda a, b: torch.equal(a.view(torch.int16), b.view(torch.int16))
    for layer in (0, 1):
        q, k, v = inputs[layer, 0]
        assert same(sa(layer, 0, q, k, v), rf2.attention(q, k, v, g, 0.0, wl.sink))          # dense
    for layer in (0, 1):
        q, k, v = inputs[layer, 1]
        assert same(sa(layer, 1, q, k, v), rf2.attention(q, k, v, g, 0.5, wl.sink))          # predict
    for layer in (0, 1):
        q, k, v = inputs[layer, 2]
        idx, cnt = sa.lists(layer)
        ref = rf2.sparse_attn(q, k, v, idx, cnt, g, raster=True)
        assert same(sa(layer, 2, q, k, v), ref)                                               # reuse
        q1, k1, _ = inputs[layer, 1]
        i1, c1 = rf2.predict_mask(q1, k1, g, 0.5, wl.sink, raster=True)
        assert torch.equal(idx, i1) and torch.equal(cnt, c1)   # the lists of that layer's predict step
    with pytest.raises(RuntimeError):
        rf2.StepAttention(g, 0.5, wl.sink, schedule=sched)(0, 2, *inputs[0, 2])               # reuse before predict


def test_step_attention_at_720p_shape_against_the_oracle():
    """StepAttention's dense and predict steps compared with the oracle directly (not with
    other CUDA calls): the Wan-720p grid, windows and head dim with 4 heads.  The predict
    step's lists must equal the oracle's outside the near-cut window and its output the
    oracle's attention over those lists; the dense step's output the oracle's attention
    over every block, on sampled query blocks including partial windows."""
    wl = WORKLOADS["wan720p"]
    shape = dict(wl.geom(), heads=4)
    g, og = rf2.Geometry(**shape), O.geom(**shape)
    q, k, v = (gen_tensor(og.B, og.T, og.H, og.W, og.heads, og.D, 8100 + i) for i in range(3))
    qd, kd, vd = (to_dev(a) for a in (q, k, v))
    sa = rf2.StepAttention(g, wl.sparsity, wl.sink, schedule=rf2.Schedule(total_steps=10, dense_fraction=0.1))
    o_dense = to_f64(sa(0, 0, qd, kd, vd))
    o_pred = to_f64(sa(0, 1, qd, kd, vd))
    idx, cnt = sa.lists(0)
    qf, kf, vf = (bf16_bits_to_f64(O.permute(a, og)) for a in (q, k, v))
    sel = O.predict_mask(qf, kf, og, wl.sparsity, wl.sink)
    gidx = idx.cpu().numpy()
    print("720p-shape predict step lists", compare_lists(gidx, cnt.cpu().numpy(), sel))
    tok = O.position_to_token(og)
    blocks = [0, og.nbw - 1, og.Nb // 2, og.Nb - og.nbw, og.Nb - 1]   # first, partial w, middle, partial t/h
    for what, out, lists in (("dense", o_dense, None), ("predict", o_pred, gidx)):
        got_rows, ref_rows = [], []
        for h in range(og.heads):
            for i in blocks:
                lst = np.arange(og.Nb) if lists is None else lists[0, h, i]
                ref = O.attention_block(qf, kf, vf, og, 0, h, i, lst, 1 / np.sqrt(og.D))
                t = tok[i * og.blk:(i + 1) * og.blk]
                keep = t >= 0
                ref_rows.append(ref[keep])
                got_rows.append(out[0, t[keep], h])
        print("720p-shape", what, assert_close(np.concatenate(got_rows), np.concatenate(ref_rows), what))


# ----------------------------------------------------------------------------- no-permute ablation

NO_PERMUTE = [
    dict(B=2, heads=2, T=3, H=10, W=13, D=64, wt=1, wh=8, ww=8),     # 7 blocks of 64, tail of 6
    dict(B=1, heads=2, T=5, H=9, W=17, D=128, wt=2, wh=8, ww=8),     # 6 blocks of 128, tail of 125
    dict(B=1, heads=3, T=2, H=16, W=16, D=128, wt=1, wh=8, ww=16),   # frames are whole blocks
]


@pytest.mark.parametrize("shape", NO_PERMUTE)
def test_no_permute_mask_and_attention_ragged(shape):
    """RF2_NO_PERMUTE (raster blocks): kept lists bit-exact outside the near-cut window,
    attention within tolerance, model-order and padded-order calls bit-identical."""
    g = rf2.Geometry(**shape, no_permute=True)
    og = O.geom(**shape, no_permute=True)
    q, k, v = _rand_bits(g, 1300)
    qp, kp, vp = (O.permute(a, og) for a in (q, k, v))          # raster order, tail padded
    qf, kf, vf = (bf16_bits_to_f64(a) for a in (qp, kp, vp))
    for s, sink, additive in ((0.5, True, False), (0.5, True, True), (0.7, False, False)):
        sel = O.predict_mask(qf, kf, og, s, sink, additive)
        idx_r, cnt_r = rf2.predict_mask(to_dev(q), to_dev(k), g, s, sink, additive, checked=True, raster=True)
        compare_lists(idx_r.cpu().numpy(), cnt_r.cpu().numpy(), sel)
        idx_w, cnt_w = rf2.predict_mask(to_dev(qp), to_dev(kp), g, s, sink, additive, checked=True)
        assert torch.equal(idx_r, idx_w) and torch.equal(cnt_r, cnt_w)
    sel = O.predict_mask(qf, kf, og, 0.5, True)
    idx = torch.from_numpy(sel.idx).cuda()
    cnt = torch.full(sel.idx.shape[:3], sel.kept, dtype=torch.int32, device="cuda")
    o_r = rf2.sparse_attn(to_dev(q), to_dev(k), to_dev(v), idx, cnt, g, checked=True, raster=True)
    o_w = rf2.sparse_attn(to_dev(qp), to_dev(kp), to_dev(vp), idx, cnt, g, checked=True)
    assert torch.equal(o_r.view(torch.int16), o_w[:, :og.N].contiguous().view(torch.int16))
    got = to_f64(o_r)
    sc = 1 / np.sqrt(og.D)
    ref = np.zeros_like(got)
    for b in range(og.B):
        for h in range(og.heads):
            for i in range(og.Nb):
                rows = O.attention_block(qf, kf, vf, og, b, h, i, sel.idx[b, h, i], sc)
                lo, hi = i * og.blk, min((i + 1) * og.blk, og.N)
                ref[b, lo:hi, h] = rows[:hi - lo]
    print(shape, assert_close(got, ref, "no_permute sparse_attn"))
    out, gidx = rf2.attention(to_dev(q), to_dev(k), to_dev(v), g, 0.5, True, return_idx=True, checked=True)
    compare_lists(gidx.cpu().numpy(), cnt.cpu().numpy(), sel)
    ref_e2e, _ = O.attention(bf16_bits_to_f64(q), bf16_bits_to_f64(k), bf16_bits_to_f64(v), og, 0.5, True)
    if torch.equal(gidx.cpu(), torch.from_numpy(sel.idx)):
        assert_close(to_f64(out), ref_e2e, "no_permute attention")


def test_no_permute_wan720p_end_to_end_sampled():
    """The ablation at the 720p video shape: 591 raster blocks of 128 tokens (last one
    80 tokens), 29 sink blocks, 119 kept per row at 80 % sparsity."""
    wl = WORKLOADS["wan720p"]
    g = rf2.Geometry(**wl.geom(), no_permute=True)
    og = O.geom(**wl.geom(), no_permute=True)
    q, k, v = _inputs("wan720p")
    out, idx = rf2.attention(to_dev(q), to_dev(k), to_dev(v), g, wl.sparsity, wl.sink,
                             return_idx=True, checked=True)
    qf, kf, vf = (bf16_bits_to_f64(O.permute(a, og)) for a in (q, k, v))
    sel = O.predict_mask(qf, kf, og, wl.sparsity, wl.sink)
    assert sel.kept == 119 and og.Nb == 591
    gidx = idx.cpu().numpy()
    stats = compare_lists(gidx, np.full(gidx.shape[:3], sel.kept), sel)
    got = to_f64(out)
    rng = np.random.default_rng(11)
    picks = {(int(rng.integers(og.heads)), int(rng.integers(og.Nb))) for _ in range(10)}
    picks |= {(0, 0), (og.heads - 1, og.Nb - 1), (3, 28)}     # first, ragged last, last sink block
    got_rows, ref_rows = [], []
    for h, i in sorted(picks):
        if not np.array_equal(gidx[0, h, i], sel.idx[0, h, i]):
            continue
        rows = O.attention_block(qf, kf, vf, og, 0, h, i, sel.idx[0, h, i], 1 / np.sqrt(og.D))
        lo, hi = i * og.blk, min((i + 1) * og.blk, og.N)
        ref_rows.append(rows[:hi - lo])
        got_rows.append(got[0, lo:hi, h])
    print("wan720p no_permute", stats, assert_close(np.concatenate(got_rows), np.concatenate(ref_rows), "wan720p"))


@pytest.mark.parametrize("method,fp8", [("rf1", False), ("rf2", True), ("rf1", True)])
def test_step_attention_other_generators_and_fp8(method, fp8):
    """The schedule with the RainFusion v1 generator and/or e4m3 operands: every step equals
    the direct call sequence it stands for, bit for bit."""
    wl = WORKLOADS["video480p"]
    g = rf2.Geometry(**wl.geom())
    sched = rf2.Schedule(total_steps=4, dense_fraction=0.25, predict_interval=2)      # D P R P
    p1 = rf2.V1Params(alpha=0.3)
    sa = rf2.StepAttention(g, 0.5, wl.sink, schedule=sched, method=method, v1_params=p1, fp8=fp8)
    same = lambda a, b: torch.equal(a.view(torch.int16), b.view(torch.int16))

    def attend(q, k, v, idx, cnt):
        if not fp8:
            return rf2.sparse_attn(q, k, v, idx, cnt, g, raster=True)
        return rf2.sparse_attn_fp8(*rf2.quantize_fp8(q, k, v, g), idx, cnt, g)

    def predict(q, k):
        if method == "rf1":
            idx, cnt, _, _ = rf2.v1_predict_mask(q, k, g, p1, kmax=sa.kept)
            return idx, cnt
        return rf2.predict_mask(q, k, g, 0.5, wl.sink, raster=True)

    dense = (torch.arange(g.Nb, dtype=torch.int32, device="cuda").expand(g.B, g.heads, g.Nb, g.Nb).contiguous(),
             torch.full((g.B, g.heads, g.Nb), g.Nb, dtype=torch.int32, device="cuda"))
    last = None
    for step in range(4):
        q, k, v = (to_dev(gen_tensor(g.B, g.T, g.H, g.W, g.heads, g.D, 8000 + 10 * step + i)) for i in range(3))
        got = sa(0, step, q, k, v)
        act = sched.action(step)
        if act == 0:
            ref = attend(q, k, v, *dense)
        else:
            if act == 1:
                last = predict(q, k)
            ref = attend(q, k, v, *last)
        assert same(got, ref), (method, fp8, step)
    if method == "rf1":
        assert sa.head_classes(0).shape == (g.B, g.heads)


def test_bounded_wait_times_out_reports_and_leaves_the_context_usable():
    """A wait on a barrier that nothing completes ends by its time limit with
    RF2_ERR_TIMEOUT in the status word, a second CTA with a long limit gives up on seeing
    it, and the context keeps working (a parity-checked call afterwards)."""
    from image_diffusion_dits_b200 import _lib
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    rc = _lib.load().rf2_selftest_wait_timeout(status.data_ptr(), 0.05, 3.0, torch.cuda.current_stream().cuda_stream)
    e1.record()
    torch.cuda.synchronize()
    assert rc == 0
    assert int(status.item()) == _lib.RF2_ERR_TIMEOUT
    elapsed = e0.elapsed_time(e1) / 1e3
    assert 0.04 <= elapsed < 2.5, elapsed          # the long wait stopped early
    test_attention_end_to_end("tiny")


def test_attention_captures_in_a_cuda_graph():
    """The fused call allocates nothing and never synchronises, so it can be captured in a
    CUDA graph: a replay reproduces the eager result bit for bit, and a replay after new
    inputs are copied into the captured buffers gives the new inputs' result."""
    wl, g, og = _geoms("video480p")
    q, k, v = (to_dev(a) for a in _inputs("video480p"))
    ws = torch.empty(rf2.workspace_size(g, wl.sparsity, wl.sink), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    rf2.attention(q, k, v, g, wl.sparsity, wl.sink, ws=ws, out=out)        # eager, also first-use setup
    torch.cuda.synchronize()
    ref = out.clone()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            rf2.attention(q, k, v, g, wl.sparsity, wl.sink, ws=ws, out=out)
    torch.cuda.current_stream().wait_stream(side)
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    q2, k2, v2 = (to_dev(a) for a in _rand_bits(g, 4242))
    for dst, src in ((q, q2), (k, k2), (v, v2)):
        dst.copy_(src)
    graph.replay()
    torch.cuda.synchronize()
    ref2 = rf2.attention(q2, k2, v2, g, wl.sparsity, wl.sink)
    assert torch.equal(out.view(torch.int16), ref2.view(torch.int16))
    del graph
