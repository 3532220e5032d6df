"""Pins for the FP8 (e4m3) quantisation oracle: hand-worked rounding table, torch's
float8_e4m3fn cast (an independent library) inside the finite range, and invariants of
the per-block quantisation.  CPU only."""
import os

import numpy as np
import torch

import oracle as O
from oracle import fp8_oracle as F8
from rf2_inputs import bf16_bits_to_f64, gen_tensor

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_e4m3_rounding_matches_hand_worked_table():
    with open(os.path.join(GOLDEN, "e4m3_round.txt")) as f:
        rows = [ln.split(":") for ln in f if ln.strip() and not ln.startswith("#")]
    for x, want, code in rows:
        got = F8.e4m3_round(float(x))
        assert float(got) == float(want), x
        assert int(F8.e4m3_code(got)) == int(code, 16), x


def test_e4m3_rounding_matches_torch_in_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1.0, 30.0, 120.0)])
    x = np.concatenate([x, np.linspace(-448, 448, 4001), 2.0 ** np.arange(-12, 9)]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn)
    np.testing.assert_array_equal(F8.e4m3_round(x), ref.float().double().numpy())
    np.testing.assert_array_equal(F8.e4m3_code(F8.e4m3_round(x)), ref.view(torch.uint8).numpy())


def _g(**kw):
    base = dict(B=2, heads=3, T=3, H=9, W=10, D=64, wt=1, wh=8, ww=8)
    base.update(kw)
    return O.geom(**base)


def test_quantisation_invariants():
    g = _g()
    x = bf16_bits_to_f64(gen_tensor(g.B, g.T, g.H, g.W, g.heads, g.D, 5))
    xp = O.permute(x, g)
    xp_pad = xp.copy()
    xp_pad[:, ~O.position_valid(g)] = 1e6          # pad rows must not matter
    codes, scale, inv = F8.quantise_blocks(xp_pad, g)
    codes0, scale0, _ = F8.quantise_blocks(xp, g)
    np.testing.assert_array_equal(codes, codes0)
    np.testing.assert_array_equal(scale, scale0)
    assert np.all(codes[:, ~O.position_valid(g)] == 0)
    blocks = codes.reshape(g.B, g.Nb, g.blk, g.heads, g.D)
    # the largest magnitude of every block maps to 448 exactly
    np.testing.assert_array_equal(np.abs(blocks).max(axis=(2, 4)), 448.0)
    # dequantised values within half an e4m3 step of x (plus the fp32 roundings)
    deq = F8.dequantise(codes, scale, g)
    valid = O.position_valid(g)
    err = np.abs(deq - xp)[:, valid]
    s = np.repeat(np.transpose(scale, (0, 2, 1)), g.blk, axis=1)[:, valid][..., None]
    step = np.maximum(np.abs(xp[:, valid]) / s, 2.0 ** -6) * 2.0 ** -3    # e4m3 step of the code
    assert np.all(err <= (0.5 * step + 1e-6 * np.abs(xp[:, valid]) / s) * s * (1 + 1e-6) + 1e-30)


def test_zero_block_quantises_to_zero_with_zero_scale():
    g = _g(B=1, heads=1)
    xp = np.zeros((1, g.Npad, 1, g.D))
    codes, scale, inv = F8.quantise_blocks(xp, g)
    assert np.all(codes == 0) and np.all(scale == 0) and np.all(inv == 0)


def test_fp8_reference_equals_exact_attention_on_representable_inputs():
    """When every element is already an e4m3 value and every block's amax is 448, the
    scale is 1, quantisation is exact, and the FP8 reference equals exact attention."""
    g = _g(B=1, heads=2, D=16)
    rng = np.random.default_rng(2)
    q, k, v = (F8.e4m3_round(rng.uniform(-300, 300, (1, g.N, 2, 16))) for _ in range(3))
    first_token = O.position_to_token(g).reshape(g.Nb, g.blk)[:, 0]   # a real token of every block
    for x in (q, k, v):
        x[0, first_token, :, 0] = 448.0
    quant = F8.quantised_inputs(q, k, v, g)
    valid = O.position_valid(g)
    for x, (codes, scale, inv, deq) in zip((q, k, v), quant):
        assert np.all(scale == 1.0) and np.all(inv == 1.0)
        np.testing.assert_array_equal(deq[:, valid], O.permute(x, g)[:, valid])
    qp, kp, vp = (O.permute(x, g) for x in (q, k, v))
    sel = O.predict_mask(qp, kp, g, 0.5, True)
    for h in range(2):
        for i in range(g.Nb):
            got = F8.fp8_attention_block(quant[0][3], quant[1][3], quant[2][3], g, 0, h, i, sel.idx[0, h, i], 0.01)
            ref = O.attention_block(qp, kp, vp, g, 0, h, i, sel.idx[0, h, i], 0.01)
            np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)
