"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol
include/rf2.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

import oracle as O
import image_diffusion_dits_b200 as rf2
from image_diffusion_dits_b200 import _lib
from rf2_inputs import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(rf2_[a-z_0-9]+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    declared = _declared()
    assert declared, "no declarations found"
    assert declared == set(_lib.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def _g(**kw):
    base = dict(B=1, heads=2, T=4, H=16, W=16, D=64, wt=1, wh=8, ww=8)
    base.update(kw)
    return rf2.Geometry(**base)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_kept_count_matches_oracle(name):
    wl = WORKLOADS[name]
    g = rf2.Geometry(**wl.geom())
    og = O.geom(**wl.geom())
    for s in wl.sparsities:
        for additive in (False, True):
            assert rf2.kept_count(g, s, wl.sink, additive) == O.kept_count(og, s, wl.sink, additive)
            assert rf2.kept_count(g, s, not wl.sink, additive) == O.kept_count(og, s, not wl.sink, additive)


def test_kept_count_sweep_matches_oracle():
    og = O.geom(B=1, heads=1, T=31, H=45, W=80, D=128, wt=2, wh=8, ww=8)
    g = rf2.Geometry(**og.__dict__)
    for i in range(0, 101):
        s = i / 100
        for sink in (False, True):
            for additive in (False, True):
                assert rf2.kept_count(g, s, sink, additive) == O.kept_count(og, s, sink, additive), (s, sink, additive)


def test_workspace_size_covers_buffers():
    wl = WORKLOADS["wan720p"]
    g = rf2.Geometry(**wl.geom())
    ws_attn = rf2.workspace_size(g, 0.8, True)
    ws_mask = rf2.workspace_size(g, 0.8, True, attention=False)
    # mask: three bf16 parts of each block mean of Q and K, the pooled scores
    assert ws_mask >= 2 * 3 * g.B * g.heads * g.Nb * g.D * 2 + g.B * g.heads * g.Nb * g.Nb * 4
    # attention: the mask scratch and the kept lists and counts; no permuted copies of
    # Q/K/V/O (the kernels gather the windows from model order)
    lists = g.B * g.heads * g.Nb * (132 + 1) * 4
    assert ws_attn >= ws_mask + lists
    assert ws_attn < ws_mask + lists + 4096


def _call_status(fn, *args):
    return fn(*args)


def test_invalid_arguments_are_rejected_without_launch():
    lib = _lib.load()
    good = _g().c()
    p = 1 << 20  # a 16-byte-aligned fake address; never dereferenced (rejected first)
    # null pointers
    assert lib.rf2_permute(None, p, ctypes.byref(good), None) == _lib.RF2_ERR_INVALID_ARG
    assert lib.rf2_unpermute(p, None, ctypes.byref(good), None) == _lib.RF2_ERR_INVALID_ARG
    # misaligned pointers
    assert lib.rf2_permute(p + 2, p, ctypes.byref(good), None) == _lib.RF2_ERR_ALIGNMENT
    # unsupported head_dim / block size
    bad_d = _g(D=96).c()
    assert lib.rf2_permute(p, p, ctypes.byref(bad_d), None) == _lib.RF2_ERR_UNSUPPORTED
    bad_blk = _g(wh=4).c()
    assert lib.rf2_permute(p, p, ctypes.byref(bad_blk), None) == _lib.RF2_ERR_UNSUPPORTED
    # non-positive sizes and null geometry
    zero = _g(T=0).c()
    assert lib.rf2_permute(p, p, ctypes.byref(zero), None) == _lib.RF2_ERR_INVALID_ARG
    assert lib.rf2_permute(p, p, None, None) == _lib.RF2_ERR_INVALID_ARG
    # kmax below the kept count
    k = lib.rf2_kept_count(ctypes.byref(good), 0.8, 1, 0)
    assert k == 4
    assert lib.rf2_predict_mask(p, p, ctypes.byref(good), 0.8, 1, 0, p, p, k - 1, p, 1 << 30, None) == \
        _lib.RF2_ERR_INVALID_ARG
    # sparsity outside [0, 1]
    assert lib.rf2_kept_count(ctypes.byref(good), 1.5, 1, 0) == -_lib.RF2_ERR_INVALID_ARG
    assert lib.rf2_workspace_size(ctypes.byref(good), -0.1, 1, 0, 1) == 0
    # workspace missing or too small
    assert lib.rf2_predict_mask(p, p, ctypes.byref(good), 0.8, 1, 0, p, p, k, None, 0, None) == \
        _lib.RF2_ERR_WORKSPACE
    assert lib.rf2_predict_mask(p, p, ctypes.byref(good), 0.8, 1, 0, p, p, k, p, 16, None) == \
        _lib.RF2_ERR_WORKSPACE
    assert lib.rf2_attention(p, p, p, ctypes.byref(good), 0.8, 1, 0.0, p, None, p, 16, 0, None) == \
        _lib.RF2_ERR_WORKSPACE
    # non-finite scale
    assert lib.rf2_sparse_attn(p, p, p, p, p, k, ctypes.byref(good), float("nan"), p, None, 0, None) == \
        _lib.RF2_ERR_INVALID_ARG
    # too many blocks for the kept-list capacity
    big = _g(T=64, H=64, W=64).c()  # 4096 blocks
    assert lib.rf2_permute(p, p, ctypes.byref(big), None) == _lib.RF2_ERR_UNSUPPORTED


def test_status_strings():
    lib = _lib.load()
    for code in range(8):
        assert lib.rf2_status_string(code)
    assert b"unknown" in lib.rf2_status_string(99)


def test_binding_refuses_cpu_tensors():
    import torch
    g = _g()
    x = torch.zeros((1, g.N, g.heads, g.D), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        rf2.permute(x, g)


def test_schedule_action_matches_oracle_and_rejects_bad_input():
    import oracle as O
    lib = _lib.load()
    for total in (1, 3, 10, 50):
        for frac in (0.0, 0.1, 0.5, 1.0):
            for interval in (1, 2, 4):
                sc = _lib.Rf2Schedule(total, frac, interval)
                for s in range(total):
                    assert lib.rf2_schedule_action(ctypes.byref(sc), s) == O.schedule_action(total, frac, interval, s)
    sc = _lib.Rf2Schedule(10, 0.1, 1)
    assert lib.rf2_schedule_action(ctypes.byref(sc), 10) == -_lib.RF2_ERR_INVALID_ARG
    assert lib.rf2_schedule_action(ctypes.byref(sc), -1) == -_lib.RF2_ERR_INVALID_ARG
    for bad in (_lib.Rf2Schedule(0, 0.1, 1), _lib.Rf2Schedule(10, 1.5, 1), _lib.Rf2Schedule(10, 0.1, 0)):
        assert lib.rf2_schedule_action(ctypes.byref(bad), 0) == -_lib.RF2_ERR_INVALID_ARG
    assert lib.rf2_schedule_action(None, 0) == -_lib.RF2_ERR_INVALID_ARG
    assert rf2.Schedule(50, 0.1, 5).action(5) == _lib.RF2_STEP_PREDICT


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_no_permute_kept_count_and_workspace_match_oracle(name):
    """RF2_NO_PERMUTE: the library's flat geometry (blocks of consecutive raster tokens,
    sink = blocks holding frame 0) agrees with the oracle's own restatement."""
    wl = WORKLOADS[name]
    g = rf2.Geometry(**wl.geom(), no_permute=True)
    og = O.geom(**wl.geom(), no_permute=True)
    assert (g.Nb, g.Npad) == (og.Nb, og.Npad)
    for i in range(0, 101, 5):
        s = i / 100
        for sink in (False, True):
            for additive in (False, True):
                assert rf2.kept_count(g, s, sink, additive) == O.kept_count(og, s, sink, additive), (s, sink, additive)
    ws_mask = rf2.workspace_size(g, 0.8, True, attention=False)
    assert ws_mask >= 2 * 3 * g.B * g.heads * g.Nb * g.D * 2 + g.B * g.heads * g.Nb * g.Nb * 4
    ws_w = rf2.workspace_size(rf2.Geometry(**wl.geom()), 0.8, True, attention=False)
    assert (ws_mask < ws_w) == (g.Nb < rf2.Geometry(**wl.geom()).Nb)


def test_no_permute_geometry_has_no_window_permutation():
    g = _g(no_permute=True)
    x = __import__("torch").zeros((g.B, g.N, g.heads, g.D))
    with pytest.raises(ValueError):
        rf2.permute(x, g)
    with pytest.raises(ValueError):
        rf2.unpermute(x, g)


V1_GEOMS = [dict(B=1, heads=2, T=4, H=16, W=16, D=64, wt=1, wh=8, ww=8),
            dict(B=2, heads=3, T=5, H=9, W=17, D=128, wt=2, wh=8, ww=8),
            dict(B=1, heads=40, T=21, H=45, W=80, D=128, wt=2, wh=8, ww=8)]
V1_PARAMS = [dict(), dict(dynamic=True), dict(bandwidth=0.5, tau=3), dict(bandwidth=0.125, tau=4, dynamic=True),
             dict(bandwidth=1.0, tau=1)]


@pytest.mark.parametrize("geo", V1_GEOMS)
def test_v1_kmax_matches_oracle(geo):
    g = rf2.Geometry(**geo)
    og = O.geom(**geo)
    for prm in V1_PARAMS:
        assert rf2.v1_kmax(g, rf2.V1Params(**prm)) == O.rf1.rf1_kmax(og, O.rf1.Rf1Params(**prm)), prm
        assert rf2.v1_workspace_size(g, rf2.V1Params(**prm)) > 0


def test_v1_rejects_bad_parameters():
    g = rf2.Geometry(**V1_GEOMS[0])
    for bad in (dict(bandwidth=0.0), dict(bandwidth=1.5), dict(tau=0), dict(alpha=1.2), dict(omega=-1),
                dict(recall_target=-0.1)):
        with pytest.raises(rf2.Rf2Error) as ei:
            rf2.v1_kmax(g, rf2.V1Params(**bad))
        assert ei.value.code == _lib.RF2_ERR_INVALID_ARG, bad
    with pytest.raises(rf2.Rf2Error) as ei:
        rf2.v1_kmax(rf2.Geometry(**V1_GEOMS[0], no_permute=True))
    assert ei.value.code == _lib.RF2_ERR_UNSUPPORTED


def test_selftest_wait_timeout_rejects_bad_arguments_without_launch():
    lib = _lib.load()
    assert lib.rf2_selftest_wait_timeout(None, 0.01, 0.1, None) == _lib.RF2_ERR_INVALID_ARG
    assert lib.rf2_selftest_wait_timeout(8, 0.0, 0.1, None) == _lib.RF2_ERR_INVALID_ARG
    assert lib.rf2_selftest_wait_timeout(8, 0.2, 0.1, None) == _lib.RF2_ERR_INVALID_ARG
    assert lib.rf2_selftest_wait_timeout(8, 0.1, 6.0, None) == _lib.RF2_ERR_INVALID_ARG
    assert lib.rf2_selftest_wait_timeout(6, 0.01, 0.1, None) == _lib.RF2_ERR_INVALID_ARG   # misaligned


def test_fp8_paths_refuse_unsupported_shapes_before_any_launch():
    """The e4m3 attention needs D = 128 and 128-token blocks: other shapes are refused on
    the host (no device call is made, so this runs without a GPU)."""
    lib = _lib.load()
    g = _g(D=64)                                     # 64-token blocks, D = 64
    cg = g.c()
    p = 1 << 20                                      # aligned stand-in addresses, never dereferenced
    st = lib.rf2_sparse_attn_fp8(p, p, p, p, p, p, 4, ctypes.byref(cg), 0.0, p, 0, 0, None)
    assert st == _lib.RF2_ERR_UNSUPPORTED
    ws = lib.rf2_workspace_size(ctypes.byref(cg), 0.5, 1, _lib.RF2_FP8, 1)
    assert ws > 0
    st = lib.rf2_attention(p, p, p, ctypes.byref(cg), 0.5, 1, 0.0, p, None, p, ws, _lib.RF2_FP8, None)
    assert st == _lib.RF2_ERR_UNSUPPORTED


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """No CPU fallback: loading the library from a path without it raises."""
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.load(str(tmp_path / "librf2.so"))


from hypothesis import given, settings, strategies as st   # noqa: E402


_WINDOWS = [(1, 8, 8), (2, 8, 8), (1, 8, 16), (2, 4, 8), (1, 4, 16), (4, 4, 4), (2, 4, 16)]


@settings(max_examples=60, deadline=None)
@given(T=st.integers(1, 9), H=st.integers(1, 40), W=st.integers(1, 40), win=st.sampled_from(_WINDOWS),
       bw=st.sampled_from([0.05, 0.125, 0.25, 0.3, 0.5, 0.75, 1.0]), tau=st.integers(1, 5), dyn=st.booleans())
def test_v1_kmax_random_geometries_match_oracle(T, H, W, win, bw, tau, dyn):
    wt, wh, ww = win
    geo = dict(B=1, heads=1, T=T, H=H, W=W, D=64, wt=wt, wh=wh, ww=ww)
    og = O.geom(**geo)
    if og.Nb > 1024:
        return
    prm = dict(bandwidth=bw, tau=tau, dynamic=dyn)
    assert rf2.v1_kmax(rf2.Geometry(**geo), rf2.V1Params(**prm)) == O.rf1.rf1_kmax(og, O.rf1.Rf1Params(**prm))


@settings(max_examples=60, deadline=None)
@given(T=st.integers(1, 9), H=st.integers(1, 40), W=st.integers(1, 40), win=st.sampled_from(_WINDOWS),
       s=st.floats(0.0, 1.0), sink=st.booleans(), additive=st.booleans(), flat=st.booleans())
def test_kept_count_random_geometries_match_oracle(T, H, W, win, s, sink, additive, flat):
    wt, wh, ww = win
    geo = dict(B=1, heads=1, T=T, H=H, W=W, D=64, wt=wt, wh=wh, ww=ww)
    og = O.geom(**geo, no_permute=flat)
    if og.Nb > 1024:
        return
    g = rf2.Geometry(**geo, no_permute=flat)
    assert (g.Nb, g.Npad) == (og.Nb, og.Npad)
    assert rf2.kept_count(g, s, sink, additive) == O.kept_count(og, s, sink, additive)
