"""Pins of the oracle's group quantizer (SVDQuant Sec. 3) and of its activation path.

Hand-worked groups from the golden fixtures, a brute-force search over every
scale and code on random groups, and the packing/XL1 conventions of the
fused quantize + down-projection step (SVDQuant Sec. 4.3).
"""
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


def test_nvfp4_groups_brute_force(golden):
    """Scale = nearest E4M3 to amax/6 and each code = nearest grid point to v*(1/s),
    found by exhaustive search over all 127 finite scales and 16 codes."""
    e2m1 = _e2m1_table(golden)
    e4m3 = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    rng = np.random.default_rng(5)
    for trial in range(300):
        mag = 10.0 ** rng.uniform(-4, 3.5)
        v = (rng.standard_normal(16) * mag).astype(np.float32)
        if trial % 7 == 0:
            v[rng.integers(16)] *= 40
        codes, s = O.quant_group("nvfp4", v)
        s32 = np.float32(np.max(np.abs(v))) / np.float32(6)
        d = np.abs(e4m3.astype(np.float64) - float(s32))
        cands = np.nonzero(d == d.min())[0]
        want_s = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
        assert s == want_s
        sd = np.float32(e4m3[s])
        if sd == 0:
            assert not np.any(codes)
            continue
        q = v * (np.float32(1) / sd)
        for qi, ci in zip(q, codes):
            dist = {c: abs(abs(float(qi)) - abs(e2m1[c])) for c in range(8)}
            best = min(dist.values())
            allowed = [c for c in range(8) if dist[c] == best]
            mag_code = allowed[0] if len(allowed) == 1 else [c for c in allowed if c % 2 == 0][0]
            assert (ci & 7) == mag_code and (ci >> 3) == (1 if np.signbit(qi) else 0)


def test_int4_groups_brute_force():
    rng = np.random.default_rng(6)
    fp16_vals = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    for trial in range(200):
        v = (rng.standard_normal(64) * 10.0 ** rng.uniform(-3, 2)).astype(np.float32)
        codes, s = O.quant_group("int4", v)
        s32 = np.float32(np.max(np.abs(v))) / np.float32(7)
        d = np.abs(fp16_vals - float(s32))
        cands = np.nonzero(d == d.min())[0]
        want_s = cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
        assert s == want_s
        inv = np.float32(1) / np.float32(fp16_vals[s])
        for vi, ci in zip(v, codes):
            q = float(np.float32(vi) * inv)
            signed = int(ci) - 16 if ci >= 8 else int(ci)
            best = min(abs(q - k) for k in range(-7, 8))
            allowed = [k for k in range(-7, 8) if abs(q - k) == best]
            want = allowed[0] if len(allowed) == 1 else [k for k in allowed if k % 2 == 0][0]
            assert signed == want


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
    """Element 2i sits in the low nibble; XL1 = X @ bf16(diag(1/lambda) L1) in fp32,
    which equals X_hat L1 up to the rounding of the folded factor."""
    M, K, r = 3, 32, 4
    rng = np.random.default_rng(7)
    X = torch.from_numpy(rng.standard_normal((M, K)).astype(np.float32)).to(torch.bfloat16)
    Xb = WL.bf16_bits(X)
    inv = (np.float32(1) / rng.uniform(0.5, 2, K).astype(np.float32)).astype(np.float32)
    L1 = O.bf16_round(rng.standard_normal((K, r)) * 0.1)
    codes, scales, XL1 = O.act_quant("nvfp4", Xb, inv, L1)
    xh = O.bf16_decode(Xb) * inv
    for m in range(M):
        for g in range(K // 16):
            c, s = O.quant_group("nvfp4", xh[m, 16 * g:16 * g + 16])
            assert s == scales[m, g]
            packed = codes[m, 8 * g:8 * g + 8]
            assert np.array_equal(packed & 0xF, c[0::2]) and np.array_equal(packed >> 4, c[1::2])
    # the folded factor is one nearest rounding of the exact product inv * L1
    L1s = O.fold_l1(L1, inv)
    prod = inv.astype(np.float64)[:, None] * O.bf16_decode(L1).astype(np.float64)
    assert np.all(np.abs(O.bf16_decode(L1s) - prod) <= np.abs(prod) * 2.0 ** -8)
    x = O.bf16_decode(Xb).astype(np.float64)
    ref = x @ O.bf16_decode(L1s).astype(np.float64)
    got = XL1.astype(np.float64)
    assert XL1.dtype == np.float32
    assert np.all(np.abs(got - ref) <= 1e-5 * np.abs(x) @ np.abs(O.bf16_decode(L1s)).astype(np.float64))
    # and it is X_hat L1 up to the rounding of the folded factor
    exact = xh.astype(np.float64) @ O.bf16_decode(L1).astype(np.float64)
    assert np.all(np.abs(got - exact) <= np.abs(xh) @ np.abs(O.bf16_decode(L1)) * 2.0 ** -8 + 1e-6)
