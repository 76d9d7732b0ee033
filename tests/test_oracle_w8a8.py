"""Pins of the oracle's W8A8 setting (SVDQuant paper, Sec. 5.1: 8-bit weights and
activations, per-token dynamic activation scales, per-channel weight scales,
a rank-16 branch; Sec. 3: q_max = 127 for signed 8-bit integers)."""
import numpy as np
import pytest

import oracle as O
import workloads as WL


def _brute_int8(v):
    """Scale amax/127 in fp32; each code the nearest integer (ties even) of
    v * (1/s) within [-127, 127], by search over all 255 codes."""
    v = np.asarray(v, dtype=np.float32)
    s = np.float32(np.max(np.abs(v))) / np.float32(127)
    if s == 0:
        return np.zeros(v.size, np.int8), s
    inv = np.float32(1) / s
    grid = np.arange(-127, 128)
    out = []
    for x in v * inv:
        d = np.abs(grid - float(x))
        c = grid[d == d.min()]
        out.append(c[0] if len(c) == 1 else [t for t in c if t % 2 == 0][0])
    return np.array(out, np.int8), s


def test_per_token_and_per_channel_scales_brute_force():
    rng = np.random.default_rng(8)
    X = (rng.standard_normal((6, 96)) * 10.0 ** rng.uniform(-2, 2, (6, 1))).astype(np.float32)
    X[2, 5] *= 50.0                                   # an outlier sets its row's scale only
    Xb = O.bf16_round(X)
    codes, scales, _ = O.act_quant("w8a8", Xb, None, None)
    x = O.bf16_decode(Xb)
    for m in range(6):
        c, s = _brute_int8(x[m])
        assert scales[m] == s and np.array_equal(codes[m], c)
    R = (rng.standard_normal((96, 5)) * 0.03).astype(np.float32)
    cw, sw = O.weight_quant("w8a8", R)
    assert cw.shape == (5, 96) and sw.shape == (5,)
    for n in range(5):
        c, s = _brute_int8(R[:, n])
        assert sw[n] == s and np.array_equal(cw[n], c)


def test_zero_row_gives_zero_codes_and_scale():
    Xb = O.bf16_round(np.zeros((2, 64)))
    codes, scales, _ = O.act_quant("w8a8", Xb, None, None)
    assert not codes.any() and not scales.any()


def test_w8a8_gemm_is_the_exact_integer_product_scaled_once():
    """r = 0: y = bf16(fp32(sum qx qw) * (s_x s_w)) -- against an int64 matmul."""
    d = WL.make_small(16, 256, 24, seed=12)
    Xb = WL.bf16_bits(d["X"])
    act = O.act_quant("w8a8", Xb, None, None)
    R = (np.random.default_rng(2).standard_normal((256, 24)) * 0.05).astype(np.float32)
    wq = O.weight_quant("w8a8", R)
    Y = O.bf16_decode(O.linear("w8a8", act, wq, None, None, 24))
    dot = act[0].astype(np.int64) @ wq[0].astype(np.int64).T
    ref = (dot.astype(np.float32) * (act[1][:, None] * wq[1][None, :])).astype(np.float32)
    assert np.array_equal(Y, O.bf16_decode(O.bf16_round(ref.astype(np.float64))))


def test_w8a8_layer_is_close_to_the_16_bit_product():
    """8-bit with the rank-16 branch reaches the bf16 product far closer than
    the 4-bit formats (the reason the paper's 8-bit results match 16-bit)."""
    d = WL.make_small(64, 256, 96, seed=13, w_outlier_rows=4)
    Xb, Wb = WL.bf16_bits(d["X"]), WL.bf16_bits(d["W"])
    exact = O.bf16_decode(Xb).astype(np.float64) @ O.bf16_decode(Wb).astype(np.float64)
    err = {}
    for fmt, r in (("w8a8", 16), ("nvfp4", 32)):
        Y = O.bf16_decode(O.layer(fmt, Xb, Wb, r)["Y"]).astype(np.float64)
        err[fmt] = np.linalg.norm(Y - exact) / np.linalg.norm(exact)
    assert err["w8a8"] < 0.02 and err["w8a8"] < err["nvfp4"] / 4
