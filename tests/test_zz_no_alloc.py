"""rf2_predict_mask_noalloc against rf2_predict_mask, through the C ABI.

The no-allocation variant exists for callers that may not call cudaMalloc (code inside a
framework that owns every device allocation, or a plug-in that must not allocate after
start-up): it keeps its scratch in a fixed device array inside the library.  This file
is collected last so that a failure here comes after every other test has run.  The
kept lists are integers, so the two entry points must agree exactly, on consecutive calls
with different shapes (the shared scratch keeps the previous call's contents)."""
import ctypes

import numpy as np
import pytest
import torch

import image_diffusion_dits_b200 as rf2
from image_diffusion_dits_b200 import _lib
from rf2_inputs import WORKLOADS, gen_qkv

pytestmark = pytest.mark.gpu


def _permuted(name, seed_base=None):
    wl = WORKLOADS[name]
    g = rf2.Geometry(**wl.geom())
    q, k, _ = gen_qkv(wl, seed_base=seed_base)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    return wl, g, rf2.permute(to_dev(q), g), rf2.permute(to_dev(k), g)


def _noalloc(qp, kp, g, sparsity, sink, flags, kmax):
    lib = _lib.load()
    idx = torch.full((g.B, g.heads, g.Nb, kmax), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((g.B, g.heads, g.Nb), -7, dtype=torch.int32, device="cuda")
    cg = g.c()
    st = lib.rf2_predict_mask_noalloc(qp.data_ptr(), kp.data_ptr(), ctypes.byref(cg), sparsity, int(sink),
                                      flags, idx.data_ptr(), cnt.data_ptr(), kmax,
                                      torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.rf2_status_string(st)
    return idx, cnt


def test_noalloc_matches_predict_mask_on_consecutive_calls():
    cases = [("video480p", 0.8, True, _lib.RF2_SINK_ADDITIVE, None),
             ("imgedit1024", 0.6, False, 0, None),
             ("video480p", 0.5, True, 0, 77)]
    for name, s, sink, flags, seed in cases:
        wl, g, qp, kp = _permuted(name, seed)
        kept = rf2.kept_count(g, s, sink, additive=bool(flags & _lib.RF2_SINK_ADDITIVE))
        kmax = kept + 2
        ref_idx, ref_cnt = rf2.predict_mask(qp, kp, g, s, sink, additive=bool(flags & _lib.RF2_SINK_ADDITIVE),
                                            kmax=kmax)
        idx, cnt = _noalloc(qp, kp, g, s, sink, flags, kmax)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx), name
        assert torch.equal(cnt, ref_cnt), name
        assert int(cnt[0, 0, 0]) == kept


def test_noalloc_checked_mode_returns_the_device_status():
    """With RF2_CHECKED the call waits for its work and returns the device status word
    (0 here), and its lists still equal rf2_predict_mask's."""
    wl, g, qp, kp = _permuted("tiny")
    kept = rf2.kept_count(g, wl.sparsity, wl.sink)
    ref_idx, ref_cnt = rf2.predict_mask(qp, kp, g, wl.sparsity, wl.sink, kmax=kept)
    for _ in range(2):
        idx, cnt = _noalloc(qp, kp, g, wl.sparsity, wl.sink, _lib.RF2_CHECKED, kept)
        assert torch.equal(idx, ref_idx) and torch.equal(cnt, ref_cnt)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = _lib.load()
    wl = WORKLOADS["wan720p"]
    g = rf2.Geometry(**wl.geom())
    assert rf2.workspace_size(g, 0.8, True, attention=False) > _lib.RF2_NOALLOC_SCRATCH_BYTES
    cg = g.c()
    p = torch.empty(16, dtype=torch.uint8, device="cuda").data_ptr()
    st = lib.rf2_predict_mask_noalloc(p, p, ctypes.byref(cg), 0.8, 1, 0, p, p, 132, None)
    assert st == _lib.RF2_ERR_WORKSPACE


def test_noalloc_model_order_matches_window_order():
    """With RF2_RASTER the no-allocation call pools straight from model-order Q and K and
    must give the same lists as rf2_predict_mask on the permuted tensors."""
    wl = WORKLOADS["video480p"]
    g = rf2.Geometry(**wl.geom())
    q, k, _ = gen_qkv(wl)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    qd, kd = to_dev(q), to_dev(k)
    kept = rf2.kept_count(g, wl.sparsity, wl.sink)
    ref_idx, ref_cnt = rf2.predict_mask(rf2.permute(qd, g), rf2.permute(kd, g), g, wl.sparsity, wl.sink,
                                        kmax=kept)
    for _ in range(2):
        idx, cnt = _noalloc(qd, kd, g, wl.sparsity, wl.sink, _lib.RF2_RASTER, kept)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx) and torch.equal(cnt, ref_cnt)


def test_noalloc_no_permute_matches_predict_mask():
    """RF2_NO_PERMUTE (raster blocks) through the no-allocation call: the same lists as
    rf2_predict_mask with the same flags."""
    wl = WORKLOADS["video480p"]
    g = rf2.Geometry(**wl.geom(), no_permute=True)
    q, k, _ = gen_qkv(wl)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    qd, kd = to_dev(q), to_dev(k)
    kept = rf2.kept_count(g, wl.sparsity, wl.sink)
    ref_idx, ref_cnt = rf2.predict_mask(qd, kd, g, wl.sparsity, wl.sink, kmax=kept, raster=True)
    idx, cnt = _noalloc(qd, kd, g, wl.sparsity, wl.sink, _lib.RF2_RASTER | _lib.RF2_NO_PERMUTE, kept)
    torch.cuda.synchronize()
    assert torch.equal(idx, ref_idx) and torch.equal(cnt, ref_cnt)
    assert int(cnt[0, 0, 0]) == kept
