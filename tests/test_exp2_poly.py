"""Host-side check of the attention kernel's FMA-pipe exp2 (sm100_ptx.cuh, exp2_poly):
the constants are read from the CUDA header and the fp32 evaluation is emulated in
NumPy (fused multiply-adds emulated in float64 and rounded once), then compared with
exp2 in float64 over the argument range the softmax uses."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "image_diffusion_dits_b200", "csrc", "sm100_ptx.cuh")


def _coeffs():
    src = open(HDR).read()
    body = src[src.index("float exp2_poly(float x)"):]
    body = body[:body.index("}")]
    nums = [float(v) for v in re.findall(r"fmaf\([^;]*?([0-9]\.[0-9]+)f\)", body)]
    c3 = float(re.search(r"fmaf\(([0-9.]+)f, f,", body).group(1))
    return c3, nums  # nums: c2, c1, c0 in Horner order


def _fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def _exp2_poly(x):
    c3, (c2, c1, c0) = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    return (p.view(np.int32) + (t.view(np.int32) << np.int32(23))).view(np.float32)


def test_exp2_poly_relative_error_bound():
    x = np.linspace(-100.0, 8.0, 1_000_001).astype(np.float32)
    got = _exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1e-4, rel.max()


def test_exp2_poly_special_arguments():
    got = _exp2_poly(np.array([0.0, 1.0, -1.0, 8.0, -np.inf, -1e30], dtype=np.float32))
    np.testing.assert_allclose(got[:4], [1.0, 2.0, 0.5, 256.0], rtol=1e-4)
    # masked keys (-inf) and huge negative arguments give 2^-125: zero once rounded to bf16
    assert np.all(got[4:] < 3e-38) and np.all(got[4:] >= 0)
