"""Host-side bound for the packed f16 exp2 of the e4m3 attention kernel (attn_fp8.cu).

Its softmax forms the exp2 arguments in fp32, with x <= 8 (the running max moves once
a score exceeds it by 8), rounds each pair to f16 and takes 2^x of both in one f16
operation; P is then rounded further for the P V product.  This checks, with exact
exp2 in float64, that rounding the argument to f16 and the result to f16 perturbs P by
less than the bf16 rounding of P itself, over the argument range the softmax uses,
and that masked keys (-inf) give exactly 0.  (The hardware result is compared with the
fp64 oracle by the GPU parity tests.)
"""
import numpy as np


def test_f16_exp2_error_below_bf16_rounding_of_p():
    def f16_exp2(x):
        return np.exp2(x.astype(np.float16).astype(np.float64)).astype(np.float16).astype(np.float64)

    # |x| <= 8: the f16 argument (11 significant bits) and result perturb P by less than
    # 2^-9, the largest relative rounding error of P in bf16
    x = np.linspace(-8.0, 8.0, 2_000_001)
    ref = np.exp2(x)
    rel = np.abs(f16_exp2(x) - ref) / ref
    assert rel.max() < 2.0 ** -9, rel.max()
    # x < -8: P < 2^-8 while the row holds a P >= 2^-8 (the running max is at most 8
    # above the largest argument); measured against that P the error stays below 2^-8,
    # the bf16 rounding step of P at 2^-8
    x = np.linspace(-30.0, -8.0, 2_000_001)
    ref = np.exp2(x)
    assert (np.abs(f16_exp2(x) - ref) / 2.0 ** -8).max() < 2.0 ** -8


def test_f16_exp2_special_arguments():
    x = np.array([0.0, 1.0, -1.0, 8.0, -np.inf, -30.0], dtype=np.float64)
    p16 = np.exp2(x.astype(np.float16).astype(np.float64)).astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(p16[:4], [1.0, 2.0, 0.5, 256.0])
    assert p16[4] == 0.0 and p16[5] == 0.0  # masked keys and deep underflow give 0
