"""Pins of the oracle's optional power-of-two prescale of the weight residual.

The layer quantizes R * 2^e instead of R, with e the largest integer that keeps
the largest group scale 2^e * max|R| / 6 within the E4M3 range (<= 448), and
scales the group sum back by 2^-e before the low-rank branch and the bias.
Checked against what the arithmetic fixes: the exponent by exact rational
inequalities, the codes by the scale-invariance of the quantizer when the
scales stay normal, the direction of the back-scaling by an fp64 product of
the dequantized operands, and the point of the option (small weights) by the
error against the exact product.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL

pytestmark = pytest.mark.filterwarnings("ignore")


def _smax(R):
    amax = np.float32(np.max(np.abs(R)))
    return Fraction(float(np.float32(amax) / np.float32(6.0)))


@pytest.mark.parametrize("scale", [1e-6, 3e-5, 1e-3, 0.02, 0.7, 5.0, 2000.0, 2688.0 / 3.0])
def test_exponent_is_the_largest_that_fits_e4m3(scale):
    rng = np.random.default_rng(int(scale * 1e6) % 2**31)
    R = (rng.standard_normal((128, 48)) * scale).astype(np.float32)
    e = O.prescale_exponent("nvfp4", R)
    s = _smax(R)
    assert Fraction(2) ** e * s <= 448 < Fraction(2) ** (e + 1) * s
    assert O.prescale_exponent("fp4g32", R) == e
    assert O.prescale_exponent("int4", R) == 0 and O.prescale_exponent("w8a8", R) == 0


def test_exponent_edges():
    assert O.prescale_exponent("nvfp4", np.zeros((64, 16), np.float32)) == 0
    R = np.zeros((64, 16), np.float32)
    R[3, 5] = 2688.0            # largest scale exactly 448: no shift
    assert O.prescale_exponent("nvfp4", R) == 0
    R[3, 5] = 2688.0 / 8        # 56: shift by 3
    assert O.prescale_exponent("nvfp4", R) == 3
    R[3, 5] = 2688.0 * 4        # 1792: shift down by 2
    assert O.prescale_exponent("nvfp4", R) == -2


def test_normal_scales_shift_by_exactly_e_and_codes_stay():
    """E4M3 rounding of 2^e s is 2^e times the rounding of s while both are normal,
    and RN(1/(2^e sd)) = 2^-e RN(1/sd): the codes cannot change."""
    rng = np.random.default_rng(3)
    R = (rng.standard_normal((256, 64)) * 0.5).astype(np.float32)
    e = O.prescale_exponent("nvfp4", R)
    assert e > 0
    c0, s0 = O.weight_quant("nvfp4", R)
    c1, s1 = O.weight_quant("nvfp4", R, e)
    d0 = np.array([O.lib().oracle_e4m3_decode(int(v)) for v in s0.ravel()], dtype=np.float64)
    d1 = np.array([O.lib().oracle_e4m3_decode(int(v)) for v in s1.ravel()], dtype=np.float64)
    normal = d0 >= 2.0 ** -6
    assert normal.mean() > 0.99
    np.testing.assert_array_equal(d1[normal], np.ldexp(d0[normal], e))
    rows = np.repeat(normal.reshape(s0.shape), 16, axis=1)   # code-wise mask (nibble pairs below)
    unpack = lambda c: np.stack([c & 15, c >> 4], axis=-1).reshape(c.shape[0], -1)
    np.testing.assert_array_equal(unpack(c1)[rows], unpack(c0)[rows])


def _fp64_layer(fmt, res, bias_bits, e):
    """Y from the dequantized operands in fp64: (q_x s_x)(q_w s_w)^T 2^-e + XL1 L2 + b."""
    cx, sx, XL1 = res["act"]
    cw, sw = res["wq"]
    Xd = O.dequant(fmt, cx, sx).astype(np.float64)
    Wd = O.dequant(fmt, cw, sw).astype(np.float64)
    Y = np.ldexp(Xd @ Wd.T, -e)
    if res["prep"]["rank"]:
        Y += XL1.astype(np.float64) @ O.bf16_decode(res["prep"]["L2"]).astype(np.float64)
    if bias_bits is not None:
        Y += O.bf16_decode(bias_bits).astype(np.float64)[None, :]
    return Y


def test_prescaled_layer_scales_the_group_sum_back():
    d = WL.make_small(96, 256, 128, rank=16, bias=True, seed=21)
    W = (d["W"].float() * 0.05).to(torch.bfloat16)      # small weights: subnormal-range scales
    Xb, Wb, bb = WL.bf16_bits(d["X"]), WL.bf16_bits(W), WL.bf16_bits(d["bias"])
    res = O.layer("nvfp4", Xb, Wb, 16, bias_bits=bb, pow2_prescale=True)
    e = res["w_exp"]
    assert e > 0
    ref = _fp64_layer("nvfp4", res, bb, e)
    y = O.bf16_decode(res["Y"]).astype(np.float64)
    rms = np.sqrt(np.mean(ref ** 2))
    assert np.all(np.abs(y - ref) <= 2.0 ** -7 * np.abs(ref) + 1e-4 * rms)


def test_prescale_recovers_small_weights():
    """Plain W4A4 (no smoothing, rank 0) of a weight whose group scales would sit
    in the E4M3 subnormal range: the prescaled layer is closer to X W."""
    d = WL.make_small(128, 512, 256, rank=0, seed=22, x_outliers=0)
    W = (d["W"].float() * 0.02).to(torch.bfloat16)      # N(0, 4e-4)
    Xb, Wb = WL.bf16_bits(d["X"]), WL.bf16_bits(W)
    exact = O.bf16_decode(Xb).astype(np.float64) @ O.bf16_decode(Wb).astype(np.float64)
    err = {}
    for pre in (False, True):
        res = O.layer("nvfp4", Xb, Wb, 0, smooth=False, pow2_prescale=pre)
        err[pre] = np.linalg.norm(O.bf16_decode(res["Y"]) - exact) / np.linalg.norm(exact)
    assert err[True] < 0.8 * err[False], err
