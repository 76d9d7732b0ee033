"""Pins of the oracle's number formats against their definitions and independent libraries.

The oracle decodes every format from its bit fields and rounds by searching for
the nearest representable value.  These tests tie that to (a) the published
format tables (golden fixtures), (b) independent rounding routines in numpy
(float16) and torch (bfloat16, float8_e4m3fn), and (c) the tie rules.
"""
import numpy as np
import pytest
import torch

import oracle as O


def test_e2m1_decode_matches_published_table(golden):
    L = O.lib()
    for row in golden("e2m1_grid.txt"):
        c, v = row[0].split()
        got = L.oracle_e2m1_decode(int(c))
        assert got == float(v) and np.signbit(got) == np.signbit(float(v)), (c, got, v)


def test_e4m3_decode_points_and_order(golden):
    L = O.lib()
    for row in golden("e4m3_points.txt"):
        c, v = row[0].split()
        assert L.oracle_e4m3_decode(int(c, 16)) == float(v)
    vals = [L.oracle_e4m3_decode(c) for c in range(0x7F)]
    assert all(b > a for a, b in zip(vals, vals[1:])), "finite E4M3 codes must increase"
    assert np.isnan(L.oracle_e4m3_decode(0x7F))
    # every finite code agrees with torch's float8_e4m3fn decoding
    t = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(np.array(vals, dtype=np.float32), t)


def test_e4m3_rounding_matches_torch_below_saturation():
    rng = np.random.default_rng(1)
    vals = np.array([O.lib().oracle_e4m3_decode(c) for c in range(0x7F)], dtype=np.float64)
    mids = (vals[1:] + vals[:-1]) / 2           # exact ties, representable in fp32
    x = np.concatenate([
        rng.uniform(0, 448, 20000), np.exp(rng.uniform(np.log(1e-4), np.log(448), 20000)),
        mids, vals, np.nextafter(mids.astype(np.float32), 0), np.nextafter(mids.astype(np.float32), 1000),
        [0.0, 2.0 ** -10, 2.0 ** -10 * 1.0001, 2.0 ** -9 * 1.5, 448.0, 460.0],
    ]).astype(np.float32)
    got = O.e4m3_round(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref), np.nonzero(got != ref)[0][:10]


def test_e4m3_saturates():
    x = np.array([448.0, 464.0, 500.0, 1e6, 3.0e38], dtype=np.float32)
    assert np.all(O.e4m3_round(x) == 0x7E)


def test_e2m1_rounding_ties_and_saturation():
    # midpoints of the E2M1 grid go to the even code
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, c in ties.items():
        assert O.e2m1_round(np.array([v]))[0] == c
        assert O.e2m1_round(np.array([-v]))[0] == c | 8
    assert np.all(O.e2m1_round(np.array([6.0, 7.0, 1e9])) == 7)
    assert O.e2m1_round(np.array([-0.1]))[0] == 8          # negative values keep the sign


def test_e2m1_rounding_is_nearest(golden):
    table = {}
    for row in golden("e2m1_grid.txt"):
        c, v = row[0].split()
        table[int(c)] = float(v)
    mags = np.array([table[c] for c in range(8)])
    rng = np.random.default_rng(2)
    x = rng.uniform(-8, 8, 50000).astype(np.float32)
    codes = O.e2m1_round(x)
    got = np.array([table[int(c)] for c in codes])
    err = np.abs(got - x)
    best = np.min(np.abs(np.abs(x)[:, None] - mags[None, :]), axis=1)
    assert np.all(err <= best + 0.0)
    assert np.all(np.sign(got[got != 0]) == np.sign(x[got != 0]))


def test_fp16_rounding_matches_numpy():
    rng = np.random.default_rng(3)
    L = O.lib()
    codes = np.arange(0, 0x7C00, dtype=np.uint16)
    vals = codes.view(np.float16).astype(np.float64)
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)  # exact in fp32
    x = np.concatenate([
        np.exp(rng.uniform(np.log(1e-8), np.log(6e4), 50000)).astype(np.float32), mids[::7],
        vals[::5].astype(np.float32), np.nextafter(mids[::11], np.float32(0)),
    ]).astype(np.float32)
    got = O.fp16_round(x)
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)
    dec = np.array([L.oracle_fp16_decode(int(c)) for c in codes[::97]], dtype=np.float32)
    assert np.array_equal(dec, codes[::97].view(np.float16).astype(np.float32))


def test_fp16_saturates():
    assert np.all(O.fp16_round(np.array([65504.0, 65520.0, 1e9], dtype=np.float32)) == 0x7BFF)


def test_bf16_rounding_matches_torch_for_fp32_inputs():
    rng = np.random.default_rng(4)
    x = np.concatenate([rng.standard_normal(50000) * 10.0 ** rng.integers(-30, 30, 50000),
                        rng.standard_normal(1000)]).astype(np.float32)
    # exact midpoints between neighbouring bf16 values
    b = torch.from_numpy(x[:2000]).to(torch.bfloat16).float().numpy().astype(np.float64)
    mid = (b * (1 + 2.0 ** -8)).astype(np.float32)
    x = np.concatenate([x, mid])
    got = O.bf16_round(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_rounding_double_inputs_hand_cases():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1); a hair above -> up;
    # 1 + 3*2^-8 is a tie between significands 129 and 130 -> 130.
    cases = {1 + 2.0 ** -8: 1.0, 1 + 2.0 ** -8 + 2.0 ** -40: 1 + 2.0 ** -7,
             1 + 3 * 2.0 ** -8: 1 + 2.0 ** -6, -(1 + 2.0 ** -8 - 2.0 ** -40): -1.0,
             7.734375: 7.75, 11.234375: 11.25, 0.0: 0.0}
    for x, want in cases.items():
        got = O.bf16_decode(O.bf16_round(np.array([x])))[0]
        assert got == want, (x, got, want)
