"""B200 (sm_100a) RainFusion2.0 block-sparse attention: Python binding of librf2.so.

Every function here marshals torch tensors (device memory, current stream) into the C ABI
of include/rf2.h; all computation runs in the library's CUDA kernels.  There is no CPU
path: the functions raise if the library is missing or a tensor is not on a CUDA device.

Layouts: model-order Q/K/V/O are [B, T*H*W, heads, D] bf16 (raster token order);
permuted tensors are [B, Npad, heads, D] bf16 in 3D-window order.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
from typing import Optional, Tuple

import torch

from . import _lib
from ._lib import RF2_CHECKED, RF2_SINK_ADDITIVE, Rf2Geom

__all__ = [
    "Geometry", "Rf2Error", "permute", "unpermute", "kept_count", "workspace_size",
    "predict_mask", "sparse_attn", "attention", "library", "Schedule", "StepAttention",
    "V1Params", "v1_kmax", "v1_workspace_size", "v1_predict_mask", "quantize_fp8", "sparse_attn_fp8",
]


class Rf2Error(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = _lib.load().rf2_status_string(code).decode()
        super().__init__(f"{where}: {msg} (status {code})")
        self.code = code


@dataclasses.dataclass(frozen=True)
class Geometry:
    """Shape of one attention call: batch, heads, token grid, head_dim, 3D window.

    no_permute selects the "without 3D permutation" ablation (RF2_NO_PERMUTE): blocks of
    blk = wt*wh*ww consecutive raster tokens instead of 3D windows, and a sink of the
    blocks that hold frame 0."""

    B: int
    heads: int
    T: int
    H: int
    W: int
    D: int
    wt: int
    wh: int
    ww: int
    no_permute: bool = False

    @property
    def N(self) -> int:
        return self.T * self.H * self.W

    @property
    def blk(self) -> int:
        return self.wt * self.wh * self.ww

    @property
    def Nb(self) -> int:
        c = lambda a, b: -(-a // b)
        if self.no_permute:
            return c(self.N, self.blk)
        return c(self.T, self.wt) * c(self.H, self.wh) * c(self.W, self.ww)

    @property
    def flags(self) -> int:
        return _lib.RF2_NO_PERMUTE if self.no_permute else 0

    @property
    def Npad(self) -> int:
        return self.Nb * self.blk

    def c(self) -> Rf2Geom:
        return Rf2Geom(self.B, self.heads, self.T, self.H, self.W, self.D, self.wt, self.wh, self.ww)


def library() -> ctypes.CDLL:
    return _lib.load()


def _check(code: int, where: str) -> None:
    if code != 0:
        raise Rf2Error(code, where)


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _cuda_bf16(t: torch.Tensor, name: str, shape) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
    if t.dtype != torch.bfloat16 or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected contiguous bf16 {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def _flags(g: Geometry, additive: bool, checked: bool, raster: bool = False) -> int:
    return ((RF2_SINK_ADDITIVE if additive else 0) | (RF2_CHECKED if checked else 0) |
            (_lib.RF2_RASTER if raster else 0) | g.flags)


def _windows_only(g: Geometry, where: str) -> None:
    if g.no_permute:
        raise ValueError(f"{where}: a no_permute geometry has no window permutation")


def permute(x: torch.Tensor, g: Geometry, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _windows_only(g, "permute")
    _cuda_bf16(x, "x", (g.B, g.N, g.heads, g.D))
    if out is None:
        out = torch.empty((g.B, g.Npad, g.heads, g.D), dtype=torch.bfloat16, device=x.device)
    cg = g.c()
    _check(library().rf2_permute(x.data_ptr(), out.data_ptr(), ctypes.byref(cg), _stream(x)), "rf2_permute")
    return out


def unpermute(xp: torch.Tensor, g: Geometry, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    _windows_only(g, "unpermute")
    _cuda_bf16(xp, "xp", (g.B, g.Npad, g.heads, g.D))
    if out is None:
        out = torch.empty((g.B, g.N, g.heads, g.D), dtype=torch.bfloat16, device=xp.device)
    cg = g.c()
    _check(library().rf2_unpermute(xp.data_ptr(), out.data_ptr(), ctypes.byref(cg), _stream(xp)),
           "rf2_unpermute")
    return out


def kept_count(g: Geometry, sparsity: float, sink: bool, additive: bool = False) -> int:
    cg = g.c()
    k = library().rf2_kept_count(ctypes.byref(cg), float(sparsity), int(sink), _flags(g, additive, False))
    if k < 0:
        raise Rf2Error(-k, "rf2_kept_count")
    return k


def workspace_size(g: Geometry, sparsity: float, sink: bool, additive: bool = False,
                   attention: bool = True) -> int:
    cg = g.c()
    n = library().rf2_workspace_size(ctypes.byref(cg), float(sparsity), int(sink),
                                     _flags(g, additive, False), int(attention))
    if n == 0:
        raise Rf2Error(_lib.RF2_ERR_INVALID_ARG, "rf2_workspace_size")
    return n


def predict_mask(qp: torch.Tensor, kp: torch.Tensor, g: Geometry, sparsity: float, sink: bool,
                 additive: bool = False, kmax: Optional[int] = None, checked: bool = False,
                 ws: Optional[torch.Tensor] = None,
                 out: Optional[Tuple[torch.Tensor, torch.Tensor]] = None,
                 raster: bool = False) -> Tuple[torch.Tensor, torch.Tensor]:
    """Kept block lists idx [B, heads, Nb, kmax] (ascending, -1 padded) and counts.
    qp, kp: window order [B, Npad, heads, D], or model order [B, N, heads, D] when raster."""
    rows = g.N if raster else g.Npad
    _cuda_bf16(qp, "qp", (g.B, rows, g.heads, g.D))
    _cuda_bf16(kp, "kp", (g.B, rows, g.heads, g.D))
    k = kept_count(g, sparsity, sink, additive) if kmax is None else kmax
    if out is None:
        idx = torch.empty((g.B, g.heads, g.Nb, k), dtype=torch.int32, device=qp.device)
        cnt = torch.empty((g.B, g.heads, g.Nb), dtype=torch.int32, device=qp.device)
    else:
        idx, cnt = out
        if idx.dtype != torch.int32 or cnt.dtype != torch.int32 or idx.shape[-1] != k:
            raise ValueError("out must be int32 (idx [B, heads, Nb, kmax], cnt [B, heads, Nb])")
    nbytes = workspace_size(g, sparsity, sink, additive, attention=False)
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=qp.device)
    cg = g.c()
    _check(library().rf2_predict_mask(qp.data_ptr(), kp.data_ptr(), ctypes.byref(cg), float(sparsity),
                                      int(sink), _flags(g, additive, checked, raster), idx.data_ptr(), cnt.data_ptr(),
                                      k, ws.data_ptr(), ws.numel(), _stream(qp)), "rf2_predict_mask")
    return idx, cnt


def sparse_attn(qp: torch.Tensor, kp: torch.Tensor, vp: torch.Tensor, idx: torch.Tensor,
                cnt: torch.Tensor, g: Geometry, scale: float = 0.0, checked: bool = False,
                out: Optional[torch.Tensor] = None,
                status: Optional[torch.Tensor] = None, raster: bool = False) -> torch.Tensor:
    """O over the kept blocks; qp/kp/vp/out in window order [B, Npad, heads, D], or in
    model order [B, N, heads, D] when raster."""
    rows = g.N if raster else g.Npad
    for t, n in ((qp, "qp"), (kp, "kp"), (vp, "vp")):
        _cuda_bf16(t, n, (g.B, rows, g.heads, g.D))
    if idx.dtype != torch.int32 or cnt.dtype != torch.int32 or not idx.is_contiguous():
        raise ValueError("idx and cnt must be contiguous int32")
    if out is None:
        out = torch.empty_like(qp)
    if status is None and checked:
        status = torch.zeros(1, dtype=torch.int32, device=qp.device)
    cg = g.c()
    _check(library().rf2_sparse_attn(qp.data_ptr(), kp.data_ptr(), vp.data_ptr(), idx.data_ptr(),
                                     cnt.data_ptr(), idx.shape[-1], ctypes.byref(cg), float(scale),
                                     out.data_ptr(), 0 if status is None else status.data_ptr(),
                                     _flags(g, False, checked, raster), _stream(qp)), "rf2_sparse_attn")
    return out


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Geometry, sparsity: float,
              sink: bool = True, scale: float = 0.0, additive: bool = False,
              return_idx: bool = False, checked: bool = False,
              ws: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None, fp8: bool = False):
    """The whole RF2 path on model-order tensors: mask prediction, then block-sparse
    attention; the window permutation is done by the kernels' gathers and scatters.
    fp8: quantise Q, K, V to e4m3 after the mask prediction and attend on e4m3 operands."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _cuda_bf16(t, n, (g.B, g.N, g.heads, g.D))
    extra = _lib.RF2_FP8 if fp8 else 0
    cg0 = g.c()
    nbytes = library().rf2_workspace_size(ctypes.byref(cg0), float(sparsity), int(sink),
                                          _flags(g, additive, False) | extra, 1)
    if nbytes == 0:
        raise Rf2Error(_lib.RF2_ERR_INVALID_ARG, "rf2_workspace_size")
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    idx = None
    if return_idx:
        kk = kept_count(g, sparsity, sink, additive)
        idx = torch.empty((g.B, g.heads, g.Nb, kk), dtype=torch.int32, device=q.device)
    cg = g.c()
    _check(library().rf2_attention(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(cg),
                                   float(sparsity), int(sink), float(scale), out.data_ptr(),
                                   0 if idx is None else idx.data_ptr(), ws.data_ptr(), ws.numel(),
                                   _flags(g, additive, checked) | extra, _stream(q)), "rf2_attention")
    return (out, idx) if return_idx else out


def quantize_fp8(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Geometry, out=None):
    """Per-(batch, head, block) e4m3 quantisation of model-order q, k, v (rf2_quantize_fp8).
    Returns (q8, k8, v8) uint8 [B, N, heads, D] holding e4m3 codes, and scales
    [3, B, heads, Nb] float32."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _cuda_bf16(t, n, (g.B, g.N, g.heads, g.D))
    if out is None:
        out = tuple(torch.empty((g.B, g.N, g.heads, g.D), dtype=torch.uint8, device=q.device) for _ in range(3)) + (
            torch.empty((3, g.B, g.heads, g.Nb), dtype=torch.float32, device=q.device),)
    q8, k8, v8, sc = out
    cg = g.c()
    _check(library().rf2_quantize_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), ctypes.byref(cg), g.flags,
                                      q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), sc.data_ptr(), _stream(q)),
           "rf2_quantize_fp8")
    return q8, k8, v8, sc


def sparse_attn_fp8(q8: torch.Tensor, k8: torch.Tensor, v8: torch.Tensor, scales: torch.Tensor, idx: torch.Tensor,
                    cnt: torch.Tensor, g: Geometry, scale: float = 0.0, checked: bool = False,
                    out: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Block-sparse attention over e4m3 operands (rf2_sparse_attn_fp8); model order."""
    for t, n in ((q8, "q8"), (k8, "k8"), (v8, "v8")):
        if not t.is_cuda or t.dtype != torch.uint8 or tuple(t.shape) != (g.B, g.N, g.heads, g.D) or not t.is_contiguous():
            raise ValueError(f"{n}: expected contiguous CUDA uint8 {(g.B, g.N, g.heads, g.D)}")
    if scales.dtype != torch.float32 or tuple(scales.shape) != (3, g.B, g.heads, g.Nb):
        raise ValueError("scales: expected float32 [3, B, heads, Nb]")
    if idx.dtype != torch.int32 or cnt.dtype != torch.int32 or not idx.is_contiguous():
        raise ValueError("idx and cnt must be contiguous int32")
    if out is None:
        out = torch.empty((g.B, g.N, g.heads, g.D), dtype=torch.bfloat16, device=q8.device)
    if status is None and checked:
        status = torch.zeros(1, dtype=torch.int32, device=q8.device)
    cg = g.c()
    _check(library().rf2_sparse_attn_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), scales.data_ptr(),
                                         idx.data_ptr(), cnt.data_ptr(), idx.shape[-1], ctypes.byref(cg),
                                         float(scale), out.data_ptr(), 0 if status is None else status.data_ptr(),
                                         _flags(g, False, checked), _stream(q8)), "rf2_sparse_attn_fp8")
    return out


@dataclasses.dataclass(frozen=True)
class Schedule:
    """Step schedule of one generation (rf2_schedule_action): the leading dense_fraction of
    the steps run dense (the pages keep the first 10 % dense), then a new mask is predicted
    every predict_interval sparse steps (1: every step, as the online method does) and
    reused in between."""

    total_steps: int
    dense_fraction: float = 0.1
    predict_interval: int = 1

    def action(self, step: int) -> int:
        sc = _lib.Rf2Schedule(int(self.total_steps), float(self.dense_fraction), int(self.predict_interval))
        a = library().rf2_schedule_action(ctypes.byref(sc), int(step))
        if a < 0:
            raise Rf2Error(-a, "rf2_schedule_action")
        return a


@dataclasses.dataclass(frozen=True)
class V1Params:
    """Parameters of the RainFusion v1 mask generators (rf2_v1_params): band half-width as
    a fraction of the axis, checkerboard stride of textural heads, recall threshold of
    the head classification, global sampling interval (0: T), RainFusion+ dynamic
    bandwidth and its recall target."""

    bandwidth: float = 0.25
    tau: int = 2
    alpha: float = 0.9
    omega: int = 0
    dynamic: bool = False
    recall_target: float = 0.9

    def c(self) -> _lib.Rf2V1Params:
        return _lib.Rf2V1Params(float(self.bandwidth), int(self.tau), float(self.alpha), int(self.omega),
                                int(bool(self.dynamic)), float(self.recall_target))


def v1_kmax(g: Geometry, params: V1Params = V1Params()) -> int:
    cg, cp = g.c(), params.c()
    k = library().rf2_v1_kmax(ctypes.byref(cg), ctypes.byref(cp), g.flags)
    if k < 0:
        raise Rf2Error(-k, "rf2_v1_kmax")
    return k


def v1_workspace_size(g: Geometry, params: V1Params = V1Params()) -> int:
    cg, cp = g.c(), params.c()
    n = library().rf2_v1_workspace_size(ctypes.byref(cg), ctypes.byref(cp), g.flags)
    if n == 0:
        raise Rf2Error(_lib.RF2_ERR_INVALID_ARG, "rf2_v1_workspace_size")
    return n


def v1_predict_mask(q: torch.Tensor, k: torch.Tensor, g: Geometry, params: V1Params = V1Params(),
                    kmax: Optional[int] = None, checked: bool = False, ws: Optional[torch.Tensor] = None):
    """RainFusion v1 kept lists from model-order q, k [B, N, heads, D]: ARM classifies every
    head (temporal / spatial / textural) from its sampled recall and the lists follow the
    class's block mask.  Returns (idx [B, heads, Nb, kmax], cnt [B, heads, Nb],
    head_class [B, heads], recall [B, heads, 2, 4]); feed idx, cnt to sparse_attn(...,
    raster=True)."""
    for t, n in ((q, "q"), (k, "k")):
        _cuda_bf16(t, n, (g.B, g.N, g.heads, g.D))
    kk = v1_kmax(g, params) if kmax is None else kmax
    dev = q.device
    idx = torch.empty((g.B, g.heads, g.Nb, kk), dtype=torch.int32, device=dev)
    cnt = torch.empty((g.B, g.heads, g.Nb), dtype=torch.int32, device=dev)
    cls = torch.empty((g.B, g.heads), dtype=torch.int32, device=dev)
    rec = torch.empty((g.B, g.heads, 2, 4), dtype=torch.float32, device=dev)
    nbytes = v1_workspace_size(g, params)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    cg, cp = g.c(), params.c()
    _check(library().rf2_v1_predict_mask(q.data_ptr(), k.data_ptr(), ctypes.byref(cg), ctypes.byref(cp),
                                         _flags(g, False, checked), idx.data_ptr(), cnt.data_ptr(), kk,
                                         cls.data_ptr(), rec.data_ptr(), ws.data_ptr(), ws.numel(), _stream(q)),
           "rf2_v1_predict_mask")
    return idx, cnt, cls, rec


class StepAttention:
    """Block-sparse attention of one generation under a Schedule, on model-order tensors:
    dense steps attend to every block, predict steps run the mask prediction of their layer
    and attend with it, reuse steps attend with the layer's last predicted lists.

    method: "rf2" predicts with the pooled-score top-k (rf2_predict_mask); "rf1" with the
    RainFusion v1 generators (rf2_v1_predict_mask, parameters v1_params; sparsity and sink
    are then unused).  fp8: every step quantises its Q, K, V to e4m3 (rf2_quantize_fp8) and
    attends with rf2_sparse_attn_fp8.  Every step runs on the library's kernels."""

    def __init__(self, g: Geometry, sparsity: float = 0.8, sink: bool = True, schedule: Optional[Schedule] = None,
                 additive: bool = False, method: str = "rf2", v1_params: Optional[V1Params] = None,
                 fp8: bool = False):
        if method not in ("rf2", "rf1"):
            raise ValueError("method must be 'rf2' or 'rf1'")
        self.g, self.sparsity, self.sink, self.additive = g, float(sparsity), bool(sink), bool(additive)
        self.method, self.fp8 = method, bool(fp8)
        self.v1_params = v1_params if v1_params is not None else V1Params()
        self.schedule = schedule if schedule is not None else Schedule(1, 0.0, 1)
        self.kept = (kept_count(g, sparsity, sink, additive) if method == "rf2" else v1_kmax(g, self.v1_params))
        self._lists = {}   # layer -> (idx, cnt) of its last prediction
        self._classes = {}  # layer -> head classes of its last v1 prediction
        self._dense = None
        self._ws = None
        self._q8 = None

    def lists(self, layer):
        """The kept lists (idx, cnt) the layer's last predict step produced."""
        return self._lists[layer]

    def head_classes(self, layer):
        """The RainFusion v1 head classes [B, heads] of the layer's last predict step."""
        return self._classes[layer]

    def _attend(self, q, k, v, idx, cnt, out):
        if not self.fp8:
            return sparse_attn(q, k, v, idx, cnt, self.g, out=out, raster=True)
        self._q8 = quantize_fp8(q, k, v, self.g, out=self._q8)
        return sparse_attn_fp8(*self._q8, idx, cnt, self.g, out=out)

    def __call__(self, layer, step: int, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
        g = self.g
        act = self.schedule.action(step)
        if act == _lib.RF2_STEP_DENSE:
            if self._dense is None:
                idx = torch.arange(g.Nb, dtype=torch.int32, device=q.device).expand(g.B, g.heads, g.Nb, g.Nb)
                cnt = torch.full((g.B, g.heads, g.Nb), g.Nb, dtype=torch.int32, device=q.device)
                self._dense = (idx.contiguous(), cnt)
            return self._attend(q, k, v, *self._dense, out)
        if act == _lib.RF2_STEP_PREDICT:
            if self.method == "rf1":
                if self._ws is None:
                    self._ws = torch.empty(v1_workspace_size(g, self.v1_params), dtype=torch.uint8, device=q.device)
                idx, cnt, cls, _ = v1_predict_mask(q, k, g, self.v1_params, kmax=self.kept, ws=self._ws)
                self._lists[layer], self._classes[layer] = (idx, cnt), cls
            else:
                if self._ws is None:
                    self._ws = torch.empty(workspace_size(g, self.sparsity, self.sink, self.additive, attention=False),
                                           dtype=torch.uint8, device=q.device)
                buf = self._lists.get(layer)
                self._lists[layer] = predict_mask(q, k, g, self.sparsity, self.sink, self.additive, kmax=self.kept,
                                                  ws=self._ws, out=buf, raster=True)
        elif layer not in self._lists:
            raise RuntimeError(f"step {step} reuses the mask of layer {layer!r}, which has none predicted yet")
        return self._attend(q, k, v, *self._lists[layer], out)


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
