#!/usr/bin/env python
"""Benchmark of the RainFusion2.0 block-sparse attention path on B200.

One step = the whole hot path on one Wan2.2-shaped 720p attention call (B=1, 40 heads,
21x45x80 latent tokens, head_dim 128, window 2x8x8, 80% sparsity, first-frame sink) on
model-order tensors, through the library's C ABI: rf2_predict_mask (block-mean pooling,
pooled scores, sink + top-k) and rf2_sparse_attn (block-sparse attention), both with
RF2_RASTER, so the 3D-window permutation and its inverse happen in the kernels' window
gathers and row scatters.  The stand-alone permute/unpermute kernels are timed after
the step, for the record.

Prints one JSON line (rank 0).  `value` is dense-equivalent TFLOP/s (4*B*heads*N^2*D
over the unpadded N, per call) summed over ranks; `ms_per_step` is ms per call.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same call.
Multi-GPU (torchrun): every rank runs its own call (independent replicas, weak scaling);
the only collectives are the barrier and the max over ranks of the timings.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "wan720p"


def _args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="rf2", choices=["rf2", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--sparsity", type=float, default=None)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-variants", action="store_true",
                   help="skip the untimed-for-the-metric variant legs (no-permute ablation, RainFusion v1)")
    p.add_argument("--no-configs", action="store_true", help="skip the other workloads of the table")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--heads", type=int, default=None,
                   help="override the head count (smaller captures for profiling)")
    return p.parse_args()


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def _geometry_numbers(g, kept):
    dense = 4.0 * g.B * g.heads * float(g.N) ** 2 * g.D
    kept_flop = 4.0 * g.B * g.heads * g.Nb * kept * g.blk * g.blk * g.D
    # real (unpadded) rows of Q and K read once, kept lists and counts written once
    mask_bytes = 2.0 * g.B * g.N * g.heads * g.D * 2 + 4.0 * g.B * g.heads * g.Nb * (kept + 1)
    permute_bytes = 3.0 * g.B * (g.N + g.Npad) * g.heads * g.D * 2
    unpermute_bytes = 1.0 * g.B * (g.N + g.Npad) * g.heads * g.D * 2
    return dense, kept_flop, mask_bytes, permute_bytes, unpermute_bytes


# DRAM traffic of one sparse_attn_kernel launch on the wan720p-shaped call, from ncu
# (dram__bytes_read.sum + dram__bytes_write.sum) on an 8-head slice of the call, scaled by
# 40 / 8 (every head is an independent set of CTAs, so traffic grows with the head count),
# valid only while the kernel source has the hash below; null otherwise.
NCU_ATTN_TRAFFIC = {"kernel_source_sha": "fecc4ae4b6e445a3", "bytes_per_launch": 5 * (541.100032e6 + 166.780672e6),
                    "how": "ncu --set full, dram__bytes_read.sum + dram__bytes_write.sum of one launch on an "
                           "8-head slice of the call (541.1 + 166.8 MB), x5 for 40 heads"}


def _attn_traffic(kernel_src_sha):
    if NCU_ATTN_TRAFFIC["kernel_source_sha"] != kernel_src_sha:
        return None
    return NCU_ATTN_TRAFFIC["bytes_per_launch"]


def kernel_source_sha():
    h = hashlib.sha256()
    for fn in ("attn.cu", "sm100_ptx.cuh"):
        with open(os.path.join(ROOT, "image_diffusion_dits_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [ln.split(",") for ln in (self.out or "").strip().splitlines() if ln.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (the job's time is its slowest rank's)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def job_throughput(flop_per_call, world, ms_per_call):
    """Whole-job dense-equivalent TFLOP/s: every rank runs one call per step, so the job
    processes world * flop_per_call per (max over ranks) step time."""
    return flop_per_call * world / (ms_per_call * 1e-3) / 1e12


def run_cpu_baseline(wl, sparsity, seconds, rows_cap=64):
    """The fp64 oracle on a bounded sample of the call, on inputs it generates itself (the
    reference arm, which has no GPU results): one head's mask stage, then attention of
    sampled query blocks of that head, scaled to the full call."""
    import numpy as np
    import torch

    import oracle as O
    from rf2_inputs import bf16_bits_to_f64, gen_tensor

    og = O.geom(**wl.geom())
    cores = len(os.sched_getaffinity(0))
    torch.set_num_threads(cores)
    # a single head of the call is generated (the oracle's cost is per head)
    one = dict(wl.geom())
    one["heads"] = 1
    g1 = O.geom(**one)
    q, k, v = (bf16_bits_to_f64(gen_tensor(1, wl.T, wl.H, wl.W, 1, wl.D, 1000 * wl.cfg + i)) for i in range(3))
    qp, kp, vp = (O.permute(a, g1) for a in (q, k, v))
    t0 = time.perf_counter()
    sel = O.predict_mask(qp, kp, g1, sparsity, wl.sink)
    t_mask_head = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    order = rng.permutation(g1.Nb)
    sc = 1.0 / math.sqrt(wl.D)
    done = 0
    t0 = time.perf_counter()
    while done < min(rows_cap, g1.Nb) and time.perf_counter() - t0 < seconds:
        i = int(order[done])
        O.attention_block(qp, kp, vp, g1, 0, 0, i, sel.idx[0, 0, i], sc)
        done += 1
    t_attn = time.perf_counter() - t0
    per_row = t_attn / done
    call_s = (per_row * og.Nb + t_mask_head) * og.heads * og.B
    return {"call_s": call_s, "cores": cores, "rows": done, "per_row_s": per_row,
            "mask_head_s": t_mask_head}


def run_cpu_baseline_and_parity(wl, sparsity, q, k, v, idx, o, seconds, attn_heads=4):
    """The fp64 oracle on the very inputs of the timed GPU step (copied back to the host),
    timed on the host cores, and the parity of the step's results against it:
      - mask stage (pool, pooled scores, sink + top-k) on every head of the call, timed in
        full; the GPU's kept lists are compared with the oracle's on every row (exact rows,
        rows that differ only inside the near-cut window, rows excused only by that
        window's floor, rows that differ elsewhere);
      - attention on `attn_heads` sampled heads, a time-bounded sample of query blocks on
        each (the first and last block and a partial window among them), timed and scaled
        linearly to all heads and query blocks (labelled extrapolated); the GPU's output
        rows are compared with the oracle's attention over the list the kernel used.
    B = 1 workloads only (the configurations all have B = 1)."""
    import numpy as np
    import torch

    import oracle as O
    from rf2_inputs import bf16_bits_to_f64

    assert wl.B == 1
    cores = len(os.sched_getaffinity(0))
    torch.set_num_threads(cores)
    og = O.geom(**wl.geom())
    one = dict(wl.geom())
    one["heads"] = 1
    g1 = O.geom(**one)
    sc = 1.0 / math.sqrt(wl.D)
    bits = lambda t: t.detach().view(torch.int16).cpu().numpy().view(np.uint16)
    qb, kb, vb, ob = bits(q), bits(k), bits(v), bits(o)
    gidx = idx.cpu().numpy()
    kept = gidx.shape[-1]
    lists = {"rows": 0, "exact": 0, "near_cut_rows": 0, "floor_only_rows": 0, "mismatch_rows": 0}
    t_mask = 0.0
    sels = {}
    rng = np.random.default_rng(11)
    attn_h = sorted(rng.choice(og.heads, min(attn_heads, og.heads), replace=False).tolist())
    for h in range(og.heads):
        qh, kh = (O.permute(bf16_bits_to_f64(a[:, :, h:h + 1]), g1) for a in (qb, kb))
        t0 = time.perf_counter()
        sel = O.predict_mask(qh, kh, g1, sparsity, wl.sink)
        t_mask += time.perf_counter() - t0
        if h in attn_h:
            sels[h] = sel
        for i in range(og.Nb):
            a, b = gidx[0, h, i], sel.idx[0, 0, i]
            lists["rows"] += 1
            if np.array_equal(a, b):
                lists["exact"] += 1
                continue
            diff = set(a.tolist()) ^ set(b.tolist())
            if diff <= sel.near_cut[i]:
                lists["near_cut_rows"] += 1
                lists["floor_only_rows"] += 0 if diff <= sel.near_cut_strict[i] else 1
            else:
                lists["mismatch_rows"] += 1
    tok = O.position_to_token(og)
    per_head_budget = seconds / max(len(attn_h), 1)
    err_sq = ref_sq = 0.0
    max_abs = 0.0
    rows = 0
    t_attn = 0.0
    for h in attn_h:
        qh, kh, vh = (O.permute(bf16_bits_to_f64(a[:, :, h:h + 1]), g1) for a in (qb, kb, vb))
        order = [0, og.Nb - 1, og.Nb - og.nbw] + rng.permutation(og.Nb).tolist()
        seen = set()
        t0 = time.perf_counter()
        for i in order:
            if i in seen or i < 0:
                continue
            if seen and time.perf_counter() - t0 > per_head_budget:
                break
            seen.add(i)
            ref = O.attention_block(qh, kh, vh, g1, 0, 0, i, gidx[0, h, i], sc)
            t = tok[i * og.blk:(i + 1) * og.blk]
            keep = t >= 0
            got = bf16_bits_to_f64(ob[0, t[keep], h])
            d = got - ref[keep]
            err_sq += float((d * d).sum())
            ref_sq += float((ref[keep] ** 2).sum())
            max_abs = max(max_abs, float(np.abs(d).max()))
            rows += 1
        t_attn += time.perf_counter() - t0
    per_row = t_attn / max(rows, 1)
    call_s = t_mask + per_row * og.Nb * og.heads
    return {"call_s": call_s, "cores": cores, "mask_all_heads_s": t_mask, "attn_rows": rows,
            "attn_heads": attn_h, "attn_per_row_s": per_row,
            "parity": {"lists": lists, "attn_rows": rows, "attn_max_abs": max_abs,
                       "attn_rel_l2": math.sqrt(err_sq / max(ref_sq, 1e-300)),
                       "tolerance": {"max_abs": 2e-2, "rel_l2": 1e-2}}}


def run_configs(rf2, dev, stream, peaks, iters, skip=()):
    """Every other workload of the table through the same two calls as the step
    (rf2_predict_mask + rf2_sparse_attn, model order): ms per call, kept-tile TFLOP/s and
    its fraction of the bf16 peak, and the mask stage's GB/s and fraction of HBM; the long
    video at every sparsity of its sweep."""
    import torch

    from rf2_inputs import WORKLOADS, gen_tensor_torch

    out = {}
    for name, wl in WORKLOADS.items():
        if name in skip:
            continue
        g = rf2.Geometry(**wl.geom())
        q, k, v = (gen_tensor_torch(g.B, g.T, g.H, g.W, g.heads, g.D, 1000 * wl.cfg + i, dev) for i in range(3))
        o = torch.empty_like(q)
        for sp in wl.sparsities:
            kept = rf2.kept_count(g, sp, wl.sink)
            dense, kept_flop, mask_bytes, _, _ = _geometry_numbers(g, kept)
            idx = torch.empty((g.B, g.heads, g.Nb, kept), dtype=torch.int32, device=dev)
            cnt = torch.empty((g.B, g.heads, g.Nb), dtype=torch.int32, device=dev)
            ws = torch.empty(rf2.workspace_size(g, sp, wl.sink, attention=False), dtype=torch.uint8, device=dev)
            t_mask, t_attn = _time_legs(stream, iters, [
                lambda: rf2.predict_mask(q, k, g, sp, wl.sink, kmax=kept, ws=ws, out=(idx, cnt), raster=True),
                lambda: rf2.sparse_attn(q, k, v, idx, cnt, g, out=o, raster=True)])
            ach = kept_flop / (t_attn * 1e-3) / 1e12
            gbs = mask_bytes / (t_mask * 1e-3) / 1e9
            out[f"{name}@{sp:g}"] = {
                "geometry": f"B={wl.B} heads={wl.heads} grid={wl.T}x{wl.H}x{wl.W} D={wl.D} "
                            f"window={wl.wt}x{wl.wh}x{wl.ww} sink={wl.sink}",
                "kept": f"{kept}/{g.Nb}", "ms_per_call": t_mask + t_attn,
                "dense_equiv_TFLOP/s": dense / ((t_mask + t_attn) * 1e-3) / 1e12,
                "sparse_attn_ms": t_attn, "kept_TFLOP/s": ach, "frac_bf16_burst": ach / peaks["bf16_tflops"],
                "predict_mask_ms": t_mask, "mask_GB/s": gbs, "mask_frac_hbm": gbs / peaks["hbm_gbs"]}
            del idx, cnt, ws
        del q, k, v, o
        torch.cuda.empty_cache()
    return out


def _time_legs(stream, iters, legs):
    """Mean device time (ms) of each callable in `legs`, run in order per iteration, after
    two warm-up iterations; CUDA events on the launching stream."""
    import torch

    for _ in range(2):
        for f in legs:
            f()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(legs) + 1)] for _ in range(iters)]
    for it in range(iters):
        ev[it][0].record(stream)
        for j, f in enumerate(legs):
            f()
            ev[it][j + 1].record(stream)
    torch.cuda.synchronize()
    return [statistics.mean(ev[it][j].elapsed_time(ev[it][j + 1]) for it in range(iters)) for j in range(len(legs))]


def run_variants(rf2, g, wl, sparsity, q, k, v, o, stream, dev, iters):
    """Legs outside the headline step, on the same inputs: the "without 3D permutation"
    ablation (blocks of consecutive raster tokens) and the RainFusion v1 generators (ARM
    classification, RainFusion+) feeding the same attention kernel."""
    import numpy as np
    import torch

    out = {}
    gnp = rf2.Geometry(**wl.geom(), no_permute=True)
    kept = rf2.kept_count(gnp, sparsity, wl.sink)
    idx = torch.empty((g.B, g.heads, gnp.Nb, kept), dtype=torch.int32, device=dev)
    cnt = torch.empty((g.B, g.heads, gnp.Nb), dtype=torch.int32, device=dev)
    ws = torch.empty(rf2.workspace_size(gnp, sparsity, wl.sink, attention=False), dtype=torch.uint8, device=dev)
    t_mask, t_attn = _time_legs(stream, iters, [
        lambda: rf2.predict_mask(q, k, gnp, sparsity, wl.sink, kmax=kept, ws=ws, out=(idx, cnt), raster=True),
        lambda: rf2.sparse_attn(q, k, v, idx, cnt, gnp, out=o, raster=True)])
    flop = 4.0 * gnp.blk * gnp.blk * gnp.D * float(cnt.sum().item())
    out["no_permute"] = {"blocks": gnp.Nb, "kept": kept, "predict_mask_ms": t_mask, "sparse_attn_ms": t_attn,
                         "kept_TFLOP/s": flop / (t_attn * 1e-3) / 1e12}
    del idx, cnt, ws
    # e4m3 operands: quantisation, then the attention over the same kept lists as the
    # headline step (lists from the bf16 mask prediction)
    if g.D == 128 and g.blk == 128:
        kept = rf2.kept_count(g, sparsity, wl.sink)
        idx = torch.empty((g.B, g.heads, g.Nb, kept), dtype=torch.int32, device=dev)
        cnt = torch.empty((g.B, g.heads, g.Nb), dtype=torch.int32, device=dev)
        rf2.predict_mask(q, k, g, sparsity, wl.sink, kmax=kept, out=(idx, cnt), raster=True)
        q8s = rf2.quantize_fp8(q, k, v, g)
        t_quant, t_attn = _time_legs(stream, iters, [
            lambda: rf2.quantize_fp8(q, k, v, g, out=q8s),
            lambda: rf2.sparse_attn_fp8(*q8s, idx, cnt, g, out=o)])
        flop = 4.0 * g.blk * g.blk * g.D * float(cnt.sum().item())
        peaks = _peaks()
        achieved = flop / (t_attn * 1e-3) / 1e12
        # algorithmic HBM bytes of the quantisation: bf16 Q, K, V read once, e4m3 written
        qbytes = 3 * (g.B * g.N * g.heads * g.D) * (2 + 1)
        out["fp8"] = {"quantize_ms": t_quant, "quantize_bytes": qbytes,
                      "quantize_GB/s": qbytes / (t_quant * 1e-3) / 1e9,
                      "sparse_attn_fp8_ms": t_attn, "kept_TFLOP/s": achieved,
                      "roofline": {"bound": "tensor", "achieved": achieved, "peak": 2 * peaks["bf16_tflops"],
                                   "unit": "TFLOP/s", "frac": achieved / (2 * peaks["bf16_tflops"]),
                                   "peak_source": peaks["source"] + " burst bf16 x 2 (nominal fp8/bf16 ratio)"}}
        del q8s, idx, cnt
    for name, prm in (("rf1", rf2.V1Params()), ("rf1_plus", rf2.V1Params(dynamic=True)),
                      ("rf1_alpha0.3", rf2.V1Params(alpha=0.3))):
        ws = torch.empty(rf2.v1_workspace_size(g, prm), dtype=torch.uint8, device=dev)
        res = {}

        def predict():
            res["lists"] = rf2.v1_predict_mask(q, k, g, prm, ws=ws)

        def attend():
            idx1, cnt1 = res["lists"][:2]
            rf2.sparse_attn(q, k, v, idx1, cnt1, g, out=o, raster=True)

        t_pred, t_attn = _time_legs(stream, iters, [predict, attend])
        idx1, cnt1, cls, _ = res["lists"]
        flop = 4.0 * g.blk * g.blk * g.D * float(cnt1.sum().item())
        out[name] = {"params": dataclasses_asdict(prm), "v1_predict_mask_ms": t_pred, "sparse_attn_ms": t_attn,
                     "classes_t_s_x": np.bincount(cls.cpu().numpy().reshape(-1), minlength=3).tolist(),
                     "mean_kept": float(cnt1.float().mean().item()), "blocks": g.Nb,
                     "kept_TFLOP/s": flop / (t_attn * 1e-3) / 1e12}
    return out


def dataclasses_asdict(x):
    import dataclasses

    return dataclasses.asdict(x)


def main():
    a = _args()
    import torch

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from rf2_inputs import WORKLOADS

    wl = WORKLOADS[a.workload]
    if a.heads is not None:
        import dataclasses

        wl = dataclasses.replace(wl, heads=a.heads)
    sparsity = wl.sparsity if a.sparsity is None else a.sparsity
    metric = "ms/call and dense-equiv TFLOP/s at 80% sparsity, Wan-720p-shaped attention"
    unit = "dense-equiv TFLOP/s"

    if a.impl == "reference":
        if rank != 0:
            return 0
        import oracle as O

        g = O.geom(**wl.geom())
        kept = O.kept_count(g, sparsity, wl.sink)
        dense = _geometry_numbers(g, kept)[0]
        per_step = []
        cb = None
        for step in range(a.warmup + a.steps):
            cb = run_cpu_baseline(wl, sparsity, seconds=max(2.0, a.cpu_seconds / max(a.steps, 1)), rows_cap=8)
            if step >= a.warmup:
                per_step.append(cb["call_s"])
        call_s = statistics.mean(per_step)
        val = dense / call_s / 1e12 * world
        line = {"impl": "reference", "metric": metric, "value": val, "unit": unit, "n_gpus": world,
                "steps": a.steps, "warmup": a.warmup, "ms_per_step": call_s * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": f"{wl.name}: B={wl.B} heads={wl.heads} grid={wl.T}x{wl.H}x{wl.W} "
                                       f"D={wl.D} window={wl.wt}x{wl.wh}x{wl.ww} sparsity={sparsity} sink={wl.sink}"},
                "cpu_baseline": {"value": val, "unit": unit, "cores": cb["cores"], "kind": "oracle",
                                 "sample": f"per step: attention of {cb['rows']} sampled query blocks of one "
                                           f"head plus that head's mask stage, scaled to all "
                                           f"{wl.heads} heads x {g.Nb} query blocks"},
                "e2e": {"value": val, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import image_diffusion_dits_b200 as rf2
    from rf2_inputs import gen_tensor_torch

    if world > 1:
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    g = rf2.Geometry(**wl.geom())
    kept = rf2.kept_count(g, sparsity, wl.sink)
    dense, kept_flop, mask_bytes, perm_bytes, unperm_bytes = _geometry_numbers(g, kept)

    seed0 = 1000 * wl.cfg + 100 * rank
    q, k, v = (gen_tensor_torch(g.B, g.T, g.H, g.W, g.heads, g.D, seed0 + i, dev) for i in range(3))
    o = torch.empty_like(q)
    idx = torch.empty((g.B, g.heads, g.Nb, kept), dtype=torch.int32, device=dev)
    cnt = torch.empty((g.B, g.heads, g.Nb), dtype=torch.int32, device=dev)
    mws = torch.empty(rf2.workspace_size(g, sparsity, wl.sink, attention=False), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    n_seg = 2

    def step(record):
        if record:
            record[0].record(stream)
        rf2.predict_mask(q, k, g, sparsity, wl.sink, kmax=kept, ws=mws, out=(idx, cnt), raster=True)
        if record:
            record[1].record(stream)
        rf2.sparse_attn(q, k, v, idx, cnt, g, out=o, status=status, raster=True)
        if record:
            record[2].record(stream)

    launches_per_step = 3 + 1  # pool, scores, top-k; attention
    for _ in range(a.warmup):
        step(None)
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} after warm-up")

    seg_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_seg + 1)] for _ in range(a.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        start.record(stream)
        for s in range(a.steps):
            step(seg_ev[s])
        end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    # the step's results, kept for the parity check against the oracle at the end
    o_step, idx_step = o.clone(), idx.clone()
    total_ms = start.elapsed_time(end)
    seg_ms = [sum(seg_ev[s][i].elapsed_time(seg_ev[s][i + 1]) for s in range(a.steps)) / a.steps
              for i in range(n_seg)]
    reduced = max_over_ranks([total_ms] + seg_ms, dev)
    total_ms, seg_ms = reduced[0], reduced[1:]
    ms_per_step = total_ms / a.steps
    value = job_throughput(dense, world, ms_per_step)

    # The stand-alone window permutation and its inverse (rf2_permute / rf2_unpermute),
    # timed after the step: Q, K, V permuted and O unpermuted once per iteration.
    shp = (g.B, g.Npad, g.heads, g.D)
    xp = torch.empty(shp, dtype=torch.bfloat16, device=dev)
    perm_ev = []
    for it in range(max(a.steps, 3) + 1):  # the first iteration warms up
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        for t in (q, k, v):
            rf2.permute(t, g, out=xp)
        ev[1].record(stream)
        rf2.unpermute(xp, g, out=o)
        ev[2].record(stream)
        if it:
            perm_ev.append(ev)
    torch.cuda.synchronize(dev)
    perm_ms = statistics.mean(ev[0].elapsed_time(ev[1]) for ev in perm_ev)
    unperm_ms = statistics.mean(ev[1].elapsed_time(ev[2]) for ev in perm_ev)
    del xp
    peaks = _peaks()

    # The mask stage alone: rf2_predict_mask back to back (its inputs as in the step).  In
    # the step it follows the previous attention call, whose output is still dirty in L2
    # and whose clock is the power-capped one; this isolates the mask kernels' own rate.
    best = float("nan")
    try:
        times = []
        for rep in range(4):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            ev[0].record(stream)
            for _ in range(10):
                rf2.predict_mask(q, k, g, sparsity, wl.sink, kmax=kept, ws=mws, out=(idx, cnt), raster=True)
            ev[1].record(stream)
            torch.cuda.synchronize(dev)
            if rep:  # the first repetition warms up
                times.append(ev[0].elapsed_time(ev[1]) / 10)
        best = min(times)
    except Exception as exc:  # a measurement for the record only: never fail the bench on it
        print(f"mask stage alone not measured: {exc}", file=sys.stderr)
    mask_alone_ms = max_over_ranks([best], dev)[0]  # every rank takes part, measured or not
    if not math.isfinite(mask_alone_ms):
        mask_alone_ms = None

    # end to end through the public fused call: pinned host inputs in, host output back
    e2e = None
    if not a.no_e2e:
        # End to end through the public fused call: every call copies its inputs from pinned
        # host memory and its output back.  Calls are pipelined as a serving loop would run
        # them: call i+1's host-to-device copies and call i-1's device-to-host copy run on
        # two copy streams while call i computes (two device input/output sets); the timed
        # region spans the first copy in to the last copy out.
        hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
        ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
        ws = torch.empty(rf2.workspace_size(g, sparsity, wl.sink), dtype=torch.uint8, device=dev)
        din = [[torch.empty_like(q) for _ in range(3)] for _ in range(2)]
        dout = [torch.empty_like(q) for _ in range(2)]
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("in_ready", "in_free", "out_ready", "out_free")}
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        for it in range(a.warmup + a.steps):
            b = it % 2
            if it == a.warmup:
                if world > 1:
                    torch.distributed.barrier()
                torch.cuda.synchronize(dev)
                e0.record(h2d)
            if it >= 2:
                h2d.wait_event(ev["in_free"][b])
            with torch.cuda.stream(h2d):
                for d, h in zip(din[b], (hq, hk, hv)):
                    d.copy_(h, non_blocking=True)
            ev["in_ready"][b].record(h2d)
            stream.wait_event(ev["in_ready"][b])
            if it >= 2:
                stream.wait_event(ev["out_free"][b])
            rf2.attention(*din[b], g, sparsity, wl.sink, ws=ws, out=dout[b])
            ev["in_free"][b].record(stream)
            ev["out_ready"][b].record(stream)
            d2h.wait_event(ev["out_ready"][b])
            with torch.cuda.stream(d2h):
                ho[b].copy_(dout[b], non_blocking=True)
            ev["out_free"][b].record(d2h)
        e1.record(d2h)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks([e0.elapsed_time(e1) / a.steps], dev)[0]
        e2e = {"value": job_throughput(dense, world, e2e_ms), "unit": unit, "ms_per_call": e2e_ms,
               "h2d_bytes_per_step": 3 * q.numel() * 2, "d2h_bytes_per_step": o.numel() * 2,
               "pipelined": "copies of neighbouring calls overlap the call's compute (2 copy streams)"}
        del ws, din, dout

    variants = None if a.no_variants else run_variants(rf2, g, wl, sparsity, q, k, v, o, stream, dev,
                                                        iters=max(3, min(a.steps, 5)))

    configs = None
    if not a.no_configs and a.heads is None:
        configs = run_configs(rf2, dev, stream, peaks, iters=3, skip=(wl.name,))

    cpu = None
    parity = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cb = run_cpu_baseline_and_parity(wl, sparsity, q, k, v, idx_step, o_step, a.cpu_seconds)
        cpu = {"value": dense / cb["call_s"] / 1e12, "unit": unit, "cores": cb["cores"], "kind": "oracle",
               "ms_per_call": cb["call_s"] * 1e3,
               "sample": f"fp64 NumPy oracle on the step's own inputs: mask stage on all {wl.heads} heads timed in "
                         f"full ({cb['mask_all_heads_s']:.1f} s); attention of {cb['attn_rows']} query blocks of "
                         f"heads {cb['attn_heads']} timed ({cb['attn_per_row_s'] * 1e3:.0f} ms each) and scaled "
                         f"to {wl.heads} heads x {g.Nb} query blocks (extrapolated)"}
        parity = cb["parity"]
    del o_step, idx_step

    attn_ms = seg_ms[1]
    achieved = kept_flop / (attn_ms * 1e-3) / 1e12
    sha = kernel_source_sha()
    traffic = _attn_traffic(sha)
    mask_gbs = mask_bytes / (seg_ms[0] * 1e-3) / 1e9
    line = {
        "metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{wl.name}: B={wl.B} heads={wl.heads} grid={wl.T}x{wl.H}x{wl.W} "
                               f"(padded {g.Npad} tokens) D={wl.D} window={wl.wt}x{wl.wh}x{wl.ww} "
                               f"sparsity={sparsity} sink={wl.sink} kept={kept}/{g.Nb}",
                   "step": "rf2_predict_mask + rf2_sparse_attn on model-order Q/K/V (RF2_RASTER)",
                   "l2": "inputs larger than L2 (774 MB per tensor); no flush",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"], "traffic": traffic,
                     "traffic_source": NCU_ATTN_TRAFFIC["how"] if traffic is not None else None,
                     "kernel": "sparse_attn_kernel<128,128>", "peak_source": peaks["source"] + " burst",
                     "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]
                                           if peaks.get("bf16_tflops_sustained") else None),
                     "kernel_source_sha": sha},
        "stages_ms": {"predict_mask": seg_ms[0], "sparse_attn": seg_ms[1]},
        "mask_stage": {"ms": seg_ms[0], "GB/s": mask_gbs, "frac_hbm": mask_gbs / peaks["hbm_gbs"],
                       "bytes": mask_bytes},
        "mask_stage_alone": (None if mask_alone_ms is None else
                             {"ms": mask_alone_ms, "GB/s": mask_bytes / (mask_alone_ms * 1e-3) / 1e9,
                              "frac_hbm": mask_bytes / (mask_alone_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                              "note": "rf2_predict_mask back to back, best of 3 x 10 calls"}),
        "permute_kernels": {"note": "stand-alone rf2_permute x3 / rf2_unpermute, outside the step",
                            "permute_qkv_ms": perm_ms, "permute_GB/s": perm_bytes / (perm_ms * 1e-3) / 1e9,
                            "unpermute_ms": unperm_ms,
                            "unpermute_GB/s": unperm_bytes / (unperm_ms * 1e-3) / 1e9},
        "clocks": clk.summary(),
        "gpu_launches": launches_per_step * a.steps,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "parity_vs_oracle": parity,
        "configs": configs,
        "variants": variants,
    }
    if configs is not None:
        configs = {f"{wl.name}@{sparsity:g}": {
            "geometry": line["config"]["workload"], "kept": f"{kept}/{g.Nb}", "ms_per_call": ms_per_step,
            "dense_equiv_TFLOP/s": value / world, "sparse_attn_ms": attn_ms, "kept_TFLOP/s": achieved,
            "frac_bf16_burst": achieved / peaks["bf16_tflops"], "predict_mask_ms": seg_ms[0],
            "mask_GB/s": mask_gbs, "mask_frac_hbm": mask_gbs / peaks["hbm_gbs"], "note": "the headline step"},
            **configs}
        line["configs"] = configs
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
