"""Pins of the oracle's group quantizer (SVDQuant Sec. 3) and of its activation path.

Hand-worked groups from the golden fixtures, a brute-force search over every
scale and code on random groups, and the packing/XL1 conventions of the
fused quantize + down-projection step (SVDQuant Sec. 4.3).
"""
from fractions import Fraction

import numpy as np
import torch

import oracle as O
import workloads as WL


def _hex_list(s):
    return [int(t, 16) for t in s.split()]


def test_nvfp4_hand_worked_groups(golden):
    for name, vals, scale, codes in golden("nvfp4_groups.txt"):
        v = np.array([float(t) for t in vals.split()], dtype=np.float32)
        c, s = O.quant_group("nvfp4", v)
        assert s == int(scale, 16), (name, hex(s))
        assert list(c) == _hex_list(codes), (name, [hex(t) for t in c])


def test_int4_hand_worked_groups(golden):
    for name, vals, scale, codes in golden("int4_groups.txt"):
        head = np.array([float(t) for t in vals.split()], dtype=np.float32)
        v = np.zeros(64, dtype=np.float32)
        v[:head.size] = head
        c, s = O.quant_group("int4", v)
        assert s == int(scale, 16), (name, hex(s))
        want = _hex_list(codes)
        assert list(c[:len(want)]) == want and not np.any(c[len(want):]), name


def _e2m1_table(golden):
    t = {}
    for row in golden("e2m1_grid.txt"):
        c, v = row[0].split()
        t[int(c)] = float(v)
    return t


# The division of Sec. 3, Q = round(v / s), is taken in fp32 as v * fp32(1/s).
# That product is within about one fp32 ulp of the exact quotient, so the two
# readings can part only where v / s lies at or within ~2^-22 (relative) of a
# rounding midpoint.  Away from that window the oracle's code must be the
# nearest grid point to the exact rational quotient; inside it, the code the
# fp32 product gives.
_WINDOW = Fraction(1, 1 << 22)


def _nearest_even(q: Fraction, grid):
    """Index of the grid value nearest to q >= 0, ties to the even index,
    saturating at the last point."""
    best, best_i = None, 0
    for i, g in enumerate(grid):
        d = abs(q - Fraction(g))
        if best is None or d < best or (d == best and i % 2 == 0):
            best, best_i = d, i
    return best_i


def _near_midpoint(q: Fraction, grid):
    return any(abs(q - (Fraction(a) + Fraction(b)) / 2) <= _WINDOW * (Fraction(a) + Fraction(b)) / 2
               for a, b in zip(grid[:-1], grid[1:]))


def _nearest_scale(s32, table):
    d = np.abs(table.astype(np.float64) - float(s32))
    cands = np.nonzero(d == d.min())[0]
    return int(cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0])


def _tie_group(rng, size, qmax, scales, mids):
    """A group whose scale is a value of `scales` that is not a power of two and
    whose entries sit exactly on rounding midpoints (t * s), one fp32 ulp beside
    them, or at random: amax = qmax * s makes the group's scale s exactly."""
    while True:
        s = float(scales[rng.integers(len(scales))])
        m, _ = np.frexp(s)
        if m != 0.5 and 1e-3 < s < 50:
            break
    v = np.zeros(size, dtype=np.float32)
    v[0] = np.float32(qmax * s)
    for i in range(1, size):
        t = np.float32(float(mids[rng.integers(len(mids))]) * s)
        step = int(rng.integers(-2, 3))
        for _ in range(abs(step)):
            t = np.nextafter(t, np.float32(np.inf if step > 0 else -np.inf), dtype=np.float32)
        v[i] = -t if rng.integers(2) else t
    rng.shuffle(v)
    return v


def test_nvfp4_groups_brute_force(golden):
    """Scale = nearest E4M3 to amax/6 by exhaustive search over all 127 finite
    scales; each code = nearest E2M1 point to the exact rational quotient v/s,
    except within the documented window around a midpoint, where it is the
    code of v * fp32(1/s).  Random groups, plus groups built on midpoints at
    scales that are not powers of two, so the window is exercised."""
    e2m1 = _e2m1_table(golden)
    grid = [e2m1[c] for c in range(8)]
    e4m3 = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    mids = [(a + b) / 2 for a, b in zip(grid[:-1], grid[1:])]
    rng = np.random.default_rng(5)
    in_window = differ = 0
    for trial in range(600):
        if trial % 2:
            v = _tie_group(rng, 16, 6, e4m3[8:], mids)
        else:
            v = (rng.standard_normal(16) * 10.0 ** rng.uniform(-4, 3.5)).astype(np.float32)
            if trial % 7 == 0:
                v[rng.integers(16)] *= 40
        codes, s = O.quant_group("nvfp4", v)
        assert s == _nearest_scale(np.float32(np.max(np.abs(v))) / np.float32(6), e4m3)
        sd = np.float32(e4m3[s])
        if sd == 0:
            assert not np.any(codes)
            continue
        for vi, ci in zip(v, codes):
            q = Fraction(float(abs(vi))) / Fraction(float(sd))
            exact = _nearest_even(q, grid)
            if _near_midpoint(q, grid):
                in_window += 1
                p = np.float32(vi) * (np.float32(1) / sd)
                want = _nearest_even(Fraction(float(abs(p))), grid)
                differ += want != exact
            else:
                want = exact
            assert (ci & 7) == want, (vi, sd, ci)
            assert (ci >> 3) == (1 if np.signbit(vi) else 0)
    assert in_window > 500 and differ > 10, (in_window, differ)


def test_int4_groups_brute_force():
    """As above for INT4: nearest fp16 to amax/7; codes from the exact quotient
    (ties to even, clamped to [-7, 7]) outside the window, from v * fp32(1/s)
    inside it."""
    rng = np.random.default_rng(6)
    fp16_vals = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    grid = list(range(0, 8))
    mids = [k + 0.5 for k in range(7)]
    in_window = differ = 0
    for trial in range(400):
        if trial % 2:
            v = _tie_group(rng, 64, 7, fp16_vals[0x2000:0x5000], mids)
        else:
            v = (rng.standard_normal(64) * 10.0 ** rng.uniform(-3, 2)).astype(np.float32)
        codes, s = O.quant_group("int4", v)
        assert s == _nearest_scale(np.float32(np.max(np.abs(v))) / np.float32(7), fp16_vals)
        sd = np.float32(fp16_vals[s])
        for vi, ci in zip(v, codes):
            q = Fraction(float(abs(vi))) / Fraction(float(sd))
            exact = _nearest_even(q, grid)
            if _near_midpoint(q, grid):
                in_window += 1
                p = np.float32(vi) * (np.float32(1) / sd)
                want = _nearest_even(Fraction(float(abs(p))), grid)
                differ += want != exact
            else:
                want = exact
            signed = int(ci) - 16 if ci >= 8 else int(ci)
            assert abs(signed) == want and (signed == 0 or (signed < 0) == bool(np.signbit(vi))), (vi, sd, ci)
    assert in_window > 2000 and differ > 20, (in_window, differ)


def test_quantization_error_bound():
    """|v - s*Q(v)| <= s * (half the local E2M1 spacing) away from saturation: a
    dropped or swapped scale index in the row quantizer would break this."""
    d = WL.make_small(64, 512, 64)
    Xb = WL.bf16_bits(d["X"])
    codes, scales, _ = O.act_quant("nvfp4", Xb, None, None)
    deq = O.dequant("nvfp4", codes, scales)
    X = O.bf16_decode(Xb)
    s = O.e4m3_decode(scales).repeat(16, axis=1)
    # largest gap of the E2M1 grid is 2 (between 4 and 6) -> error <= 1 * s, plus the
    # scale's own rounding, which can push |v|/s up to 6 * (1 + 2^-4)
    assert np.all(np.abs(X - deq) <= 1.0 * s + np.abs(X) * 0.07 + 1e-30)
    g = np.abs(X).reshape(64, -1, 16).max(axis=2)
    rel = np.abs(X - deq).reshape(64, -1, 16).max(axis=2) / np.maximum(g, 1e-30)
    assert rel.mean() < 0.1


def test_act_quant_packing_and_xl1():
    """Element 2i sits in the low nibble; XL1 is the branch X_hat L1 of Sec. 4.2
    with x_hat = fp32(x) * inv_lambda (the quantizer's own value) against the
    unfolded bf16 L1, summed in fp32: it must lie within the worst-case bound
    of an fp32 sequential sum of K rounded products, (K + 1) 2^-24 sum|x_hat L1|,
    of the fp64 value.  A down-projection that rounds the smoothing into its
    factor once, bf16(inv_lambda L1), misses that bound by orders of magnitude."""
    rng = np.random.default_rng(7)
    for fmt, (M, K, r) in (("nvfp4", (3, 32, 4)), ("int4", (5, 256, 8)), ("w8a8", (4, 192, 16))):
        X = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
        Xb = WL.bf16_bits(X)
        inv = (np.float32(1) / rng.uniform(0.5, 2, K).astype(np.float32)).astype(np.float32)
        L1 = O.bf16_round(rng.standard_normal((K, r)) * 0.1)
        codes, scales, XL1 = O.act_quant(fmt, Xb, inv, L1)
        xh = O.bf16_decode(Xb) * inv
        assert xh.dtype == np.float32 and XL1.dtype == np.float32 and XL1.shape == (M, r)
        if fmt == "nvfp4":
            for m in range(M):
                for g in range(K // 16):
                    c, s = O.quant_group("nvfp4", xh[m, 16 * g:16 * g + 16])
                    assert s == scales[m, g]
                    packed = codes[m, 8 * g:8 * g + 8]
                    assert np.array_equal(packed & 0xF, c[0::2]) and np.array_equal(packed >> 4, c[1::2])
        l1 = O.bf16_decode(L1).astype(np.float64)
        exact = xh.astype(np.float64) @ l1
        S = np.abs(xh.astype(np.float64)) @ np.abs(l1)
        bound = (K + 1) * 2.0 ** -24 * S
        got = XL1.astype(np.float64)
        assert np.all(np.abs(got - exact) <= bound), (fmt, float(np.max(np.abs(got - exact) / S)))
        # the folded factor (one bf16 rounding of inv_lambda * L1, fp64 here) is
        # not X_hat L1 to this accuracy
        folded = O.bf16_decode(O.bf16_round(inv.astype(np.float64)[:, None] * l1)).astype(np.float64)
        x = O.bf16_decode(Xb).astype(np.float64)
        assert np.any(np.abs(x @ folded - exact) > bound), fmt
