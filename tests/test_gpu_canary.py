"""Guard bands around every output and workspace buffer (the stand-in for a memory checker,
which is not available here).

Each entry point gets its outputs, and its workspace, as views into larger device buffers
whose margins before and after hold a sentinel byte pattern; after the call the margins
must be unchanged.  A store past the end of a partial window's rows, past a -1 padded list
tail, or past the end of the workspace would change them.  The geometries are ragged:
partial windows on every axis, batch > 1, both block sizes and both head dims.  The
numerical results are checked elsewhere (test_gpu_parity.py and the others); here only
the margins, plus the few invariants of the written regions that need no oracle."""
import ctypes

import numpy as np
import pytest
import torch

import image_diffusion_dits_b200 as rf2
from image_diffusion_dits_b200 import _lib
from rf2_inputs import gen_tensor

from _util import to_dev

pytestmark = pytest.mark.gpu

MARGIN = 4096      # bytes of sentinel before and after each buffer (keeps 256-byte alignment)
SENTINEL = 0xA5

RAGGED = [
    dict(B=2, heads=3, T=3, H=7, W=10, D=64, wt=1, wh=8, ww=8),
    dict(B=1, heads=2, T=5, H=9, W=17, D=128, wt=2, wh=8, ww=8),
    dict(B=1, heads=2, T=4, H=11, W=21, D=64, wt=2, wh=4, ww=16),
    dict(B=2, heads=2, T=3, H=10, W=19, D=128, wt=2, wh=8, ww=8),
]


class Guarded:
    """A device buffer of `shape`/`dtype` with sentinel margins on both sides."""

    def __init__(self, shape, dtype, fill=None):
        self.shape = tuple(shape)
        self.nbytes = int(np.prod(self.shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((2 * MARGIN + self.nbytes,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.t = self.raw[MARGIN:MARGIN + self.nbytes].view(dtype).view(self.shape)
        if fill is not None:
            self.t.fill_(fill)

    def ptr(self):
        return self.t.data_ptr()

    def assert_margins(self, what):
        torch.cuda.synchronize()
        head = self.raw[:MARGIN]
        tail = self.raw[MARGIN + self.nbytes:]
        bad_h = int((head != SENTINEL).sum())
        bad_t = int((tail != SENTINEL).sum())
        assert bad_h == 0 and bad_t == 0, f"{what}: {bad_h} bytes before and {bad_t} after the buffer were written"


def _ws(nbytes):
    return Guarded((nbytes,), torch.uint8)


def _inputs(shape, seed=300):
    g = rf2.Geometry(**shape)
    q, k, v = (to_dev(gen_tensor(g.B, g.T, g.H, g.W, g.heads, g.D, seed + i)) for i in range(3))
    return g, q, k, v


def _stream():
    return torch.cuda.current_stream().cuda_stream


@pytest.mark.parametrize("shape", RAGGED)
def test_permute_and_unpermute_stay_inside_their_outputs(shape):
    g, q, _, _ = _inputs(shape)
    lib = _lib.load()
    cg = g.c()
    xp = Guarded((g.B, g.Npad, g.heads, g.D), torch.bfloat16)
    assert lib.rf2_permute(q.data_ptr(), xp.ptr(), ctypes.byref(cg), _stream()) == 0
    xp.assert_margins("rf2_permute")
    x = Guarded((g.B, g.N, g.heads, g.D), torch.bfloat16)
    assert lib.rf2_unpermute(xp.ptr(), x.ptr(), ctypes.byref(cg), _stream()) == 0
    x.assert_margins("rf2_unpermute")
    assert torch.equal(x.t, q)


@pytest.mark.parametrize("shape", RAGGED)
@pytest.mark.parametrize("raster", [False, True])
def test_predict_mask_and_sparse_attn_stay_inside_their_outputs(shape, raster):
    g, q, k, v = _inputs(shape)
    if not raster:
        q, k, v = (rf2.permute(t, g) for t in (q, k, v))
    rows = g.N if raster else g.Npad
    lib = _lib.load()
    cg = g.c()
    flags = _lib.RF2_CHECKED | (_lib.RF2_RASTER if raster else 0)
    kept = rf2.kept_count(g, 0.5, True)
    kmax = kept + 3  # a -1 padded tail after every list
    idx = Guarded((g.B, g.heads, g.Nb, kmax), torch.int32)
    cnt = Guarded((g.B, g.heads, g.Nb), torch.int32)
    ws = _ws(rf2.workspace_size(g, 0.5, True, attention=False))
    st = lib.rf2_predict_mask(q.data_ptr(), k.data_ptr(), ctypes.byref(cg), 0.5, 1, flags, idx.ptr(), cnt.ptr(),
                              kmax, ws.ptr(), ws.nbytes, _stream())
    assert st == 0, lib.rf2_status_string(st)
    for b, n in ((idx, "idx"), (cnt, "cnt"), (ws, "workspace")):
        b.assert_margins(f"rf2_predict_mask {n}")
    assert bool((cnt.t == kept).all())
    assert bool((idx.t[..., kept:] == -1).all())

    o = Guarded((g.B, rows, g.heads, g.D), torch.bfloat16)
    status = Guarded((1,), torch.int32, fill=0)
    st = lib.rf2_sparse_attn(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.ptr(), cnt.ptr(), kmax, ctypes.byref(cg),
                             0.0, o.ptr(), status.ptr(), flags, _stream())
    assert st == 0, lib.rf2_status_string(st)
    o.assert_margins("rf2_sparse_attn o")
    status.assert_margins("rf2_sparse_attn status")
    assert bool(torch.isfinite(o.t.float()).all())


@pytest.mark.parametrize("shape", RAGGED)
@pytest.mark.parametrize("fp8", [False, True])
def test_attention_stays_inside_output_lists_and_workspace(shape, fp8):
    if fp8 and (shape["D"] != 128 or shape["wt"] * shape["wh"] * shape["ww"] != 128):
        pytest.skip("the e4m3 path has D = 128 and 128-token blocks only")
    g, q, k, v = _inputs(shape)
    lib = _lib.load()
    cg = g.c()
    flags = _lib.RF2_CHECKED | (_lib.RF2_FP8 if fp8 else 0)
    nbytes = lib.rf2_workspace_size(ctypes.byref(cg), 0.5, 1, flags, 1)
    assert nbytes > 0
    ws = _ws(nbytes)
    o = Guarded((g.B, g.N, g.heads, g.D), torch.bfloat16)
    kept = rf2.kept_count(g, 0.5, True)
    idx = Guarded((g.B, g.heads, g.Nb, kept), torch.int32)
    st = lib.rf2_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(cg), 0.5, 1, 0.0, o.ptr(),
                           idx.ptr(), ws.ptr(), ws.nbytes, flags, _stream())
    assert st == 0, lib.rf2_status_string(st)
    for b, n in ((o, "o"), (idx, "idx_out"), (ws, "workspace")):
        b.assert_margins(f"rf2_attention{' (e4m3)' if fp8 else ''} {n}")


@pytest.mark.parametrize("shape", [s for s in RAGGED if s["D"] == 128 and s["wt"] * s["wh"] * s["ww"] == 128])
def test_quantize_and_fp8_attention_stay_inside_their_outputs(shape):
    g, q, k, v = _inputs(shape)
    lib = _lib.load()
    cg = g.c()
    q8, k8, v8 = (Guarded((g.B, g.N, g.heads, g.D), torch.uint8) for _ in range(3))
    sc = Guarded((3, g.B, g.heads, g.Nb), torch.float32)
    st = lib.rf2_quantize_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(cg), 0, q8.ptr(), k8.ptr(),
                              v8.ptr(), sc.ptr(), _stream())
    assert st == 0, lib.rf2_status_string(st)
    for b, n in ((q8, "q8"), (k8, "k8"), (v8, "v8"), (sc, "scales")):
        b.assert_margins(f"rf2_quantize_fp8 {n}")
    idx, cnt = rf2.predict_mask(q, k, g, 0.5, True, raster=True)
    o = Guarded((g.B, g.N, g.heads, g.D), torch.bfloat16)
    status = Guarded((1,), torch.int32, fill=0)
    st = lib.rf2_sparse_attn_fp8(q8.ptr(), k8.ptr(), v8.ptr(), sc.ptr(), idx.data_ptr(), cnt.data_ptr(),
                                 idx.shape[-1], ctypes.byref(cg), 0.0, o.ptr(), status.ptr(), _lib.RF2_CHECKED,
                                 _stream())
    assert st == 0, lib.rf2_status_string(st)
    o.assert_margins("rf2_sparse_attn_fp8 o")
    status.assert_margins("rf2_sparse_attn_fp8 status")


@pytest.mark.parametrize("shape", [RAGGED[1], RAGGED[3]])
def test_v1_generator_stays_inside_its_outputs(shape):
    g, q, k, _ = _inputs(shape)
    lib = _lib.load()
    cg = g.c()
    params = rf2.V1Params()
    cp = params.c()
    kmax = rf2.v1_kmax(g, params) + 2
    idx = Guarded((g.B, g.heads, g.Nb, kmax), torch.int32)
    cnt = Guarded((g.B, g.heads, g.Nb), torch.int32)
    cls = Guarded((g.B, g.heads), torch.int32)
    rec = Guarded((g.B, g.heads, 2, 4), torch.float32)
    ws = _ws(rf2.v1_workspace_size(g, params))
    st = lib.rf2_v1_predict_mask(q.data_ptr(), k.data_ptr(), ctypes.byref(cg), ctypes.byref(cp), _lib.RF2_CHECKED,
                                 idx.ptr(), cnt.ptr(), kmax, cls.ptr(), rec.ptr(), ws.ptr(), ws.nbytes, _stream())
    assert st == 0, lib.rf2_status_string(st)
    for b, n in ((idx, "idx"), (cnt, "cnt"), (cls, "head_class"), (rec, "recall"), (ws, "workspace")):
        b.assert_margins(f"rf2_v1_predict_mask {n}")
    c = cnt.t.cpu().numpy()
    i = idx.t.cpu().numpy()
    for r, n in zip(i.reshape(-1, kmax), c.reshape(-1)):
        assert 0 < n <= kmax and np.all(r[n:] == -1)


@pytest.mark.parametrize("shape", [RAGGED[0], RAGGED[1]])
def test_noalloc_mask_stays_inside_its_outputs(shape):
    g, q, k, _ = _inputs(shape)
    lib = _lib.load()
    cg = g.c()
    kept = rf2.kept_count(g, 0.5, True)
    kmax = kept + 3
    idx = Guarded((g.B, g.heads, g.Nb, kmax), torch.int32)
    cnt = Guarded((g.B, g.heads, g.Nb), torch.int32)
    st = lib.rf2_predict_mask_noalloc(q.data_ptr(), k.data_ptr(), ctypes.byref(cg), 0.5, 1,
                                      _lib.RF2_RASTER | _lib.RF2_CHECKED, idx.ptr(), cnt.ptr(), kmax, _stream())
    assert st == 0, lib.rf2_status_string(st)
    idx.assert_margins("rf2_predict_mask_noalloc idx")
    cnt.assert_margins("rf2_predict_mask_noalloc cnt")
    assert bool((idx.t[..., kept:] == -1).all())
