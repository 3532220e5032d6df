"""Helpers shared by the GPU parity tests (test-side only)."""
from __future__ import annotations

import numpy as np
import torch

import oracle as O
from rf2_inputs import bf16_bits_to_f64

# Tolerances for bf16 inputs with fp32 accumulation against the fp64 oracle.
ATOL_MAX = 2e-2
REL_L2 = 1e-2


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bits -> CUDA bf16 tensor (same bits)."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return bf16_bits_to_f64(to_bits(t))


def assert_close(got: np.ndarray, ref: np.ndarray, what: str = "") -> dict:
    err = np.abs(got - ref)
    max_abs = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert max_abs <= ATOL_MAX, f"{what}: max-abs {max_abs:.3e} > {ATOL_MAX}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    return {"max_abs": max_abs, "rel_l2": rel}


def compare_lists(gpu_idx: np.ndarray, gpu_cnt: np.ndarray, sel: "O.Selection") -> dict:
    """Bit-exact comparison of kept lists outside the near-cut window of each row.
    Returns counts of rows that matched exactly, rows that differed only near the cut, and
    among those the rows that the 1e-4 * |cut| window alone would not excuse (excused only
    by the window's floor for cuts near zero)."""
    kept = sel.kept
    flat_o = sel.idx.reshape(-1, kept)
    flat_g = gpu_idx.reshape(len(flat_o), -1)
    cnt = gpu_cnt.reshape(-1)
    assert np.all(cnt == kept), "kept counts differ"
    assert np.all(flat_g[:, kept:] == -1), "entries after the kept count must be -1"
    exact, near_rows, near_blocks, floor_rows = 0, 0, 0, 0
    strict = sel.near_cut_strict if sel.near_cut_strict else sel.near_cut
    for r in range(len(flat_o)):
        a = flat_g[r, :kept]
        b = flat_o[r]
        if np.array_equal(a, b):
            exact += 1
            continue
        assert np.all(np.diff(a) > 0), f"row {r}: GPU list not ascending/unique"
        diff = set(a.tolist()) ^ set(b.tolist())
        assert diff <= sel.near_cut[r], f"row {r}: lists differ outside the near-cut window: {sorted(diff)}"
        near_rows += 1
        near_blocks += len(diff) // 2
        floor_rows += 0 if diff <= strict[r] else 1
    return {"rows": len(flat_o), "exact": exact, "near_cut_rows": near_rows, "near_cut_swaps": near_blocks,
            "floor_only_rows": floor_rows}
