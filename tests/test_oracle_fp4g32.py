"""Pins of the oracle's FP4 group-32 format (E2M1 codes, one E4M3 scale per 32
values along K): the paper's own FP4 setting (SVDQuant paper, Sec. 5.1: FP4
groups of 32 with an FP8 scale, read here as E4M3)."""
import numpy as np
import torch

import oracle as O
import workloads as WL


def _e2m1_table(golden):
    t = {}
    for row in golden("e2m1_grid.txt"):
        c, v = row[0].split()
        t[int(c)] = float(v)
    return t


def test_fp4g32_groups_brute_force(golden):
    """Scale = nearest E4M3 to amax/6 over all 32 values; each code = nearest
    E2M1 value of v * (1/s), by exhaustive search over scales and codes."""
    e2m1 = _e2m1_table(golden)
    e4m3 = torch.arange(0, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    rng = np.random.default_rng(32)
    for trial in range(200):
        v = (rng.standard_normal(32) * 10.0 ** rng.uniform(-4, 3.5)).astype(np.float32)
        if trial % 5 == 0:
            v[rng.integers(32)] *= 40        # an outlier in either half sets the shared scale
        codes, s = O.quant_group("fp4g32", v)
        s32 = np.float32(np.max(np.abs(v))) / np.float32(6)
        d = np.abs(e4m3.astype(np.float64) - float(s32))
        cands = np.nonzero(d == d.min())[0]
        assert s == (cands[0] if len(cands) == 1 else [c for c in cands if c % 2 == 0][0])
        sd = np.float32(e4m3[s])
        if sd == 0:
            assert not np.any(codes)
            continue
        q = v * (np.float32(1) / sd)
        for qi, ci in zip(q, codes):
            dist = {c: abs(abs(float(qi)) - abs(e2m1[c])) for c in range(8)}
            best = min(dist.values())
            allowed = [c for c in range(8) if dist[c] == best]
            mag = allowed[0] if len(allowed) == 1 else [c for c in allowed if c % 2 == 0][0]
            assert (ci & 7) == mag and (ci >> 3) == (1 if np.signbit(qi) else 0)


def test_fp4g32_equals_nvfp4_when_both_halves_share_the_scale():
    """With equal amax in both 16-value halves, one scale per 32 equals one per 16."""
    rng = np.random.default_rng(3)
    for _ in range(50):
        v = rng.standard_normal(32).astype(np.float32)
        a = np.float32(np.max(np.abs(v)) * 1.5)
        v[0], v[16] = a, -a
        c32, s32 = O.quant_group("fp4g32", v)
        c0, s0 = O.quant_group("nvfp4", v[:16])
        c1, s1 = O.quant_group("nvfp4", v[16:])
        assert s32 == s0 == s1
        assert np.array_equal(c32, np.concatenate([c0, c1]))


def test_fp4g32_row_layout_and_gemm_reduce_to_dequantized_product():
    """Row quantizer: one scale per 32 columns, codes packed low nibble first;
    the GEMM with r = 0 equals the fp64 product of the dequantized operands."""
    d = WL.make_small(8, 128, 16, seed=4)
    Xb = WL.bf16_bits(d["X"])
    codes, scales, _ = O.act_quant("fp4g32", Xb, None, None)
    assert codes.shape == (8, 64) and scales.shape == (8, 4) and scales.dtype == np.uint8
    x = O.bf16_decode(Xb)
    for m in range(8):
        for g in range(4):
            c, s = O.quant_group("fp4g32", x[m, 32 * g:32 * g + 32])
            assert s == scales[m, g]
            packed = codes[m, 16 * g:16 * g + 16]
            assert np.array_equal(packed & 0xF, c[0::2]) and np.array_equal(packed >> 4, c[1::2])
    R = (np.random.default_rng(5).standard_normal((128, 16)) * 0.05).astype(np.float32)
    wq = O.weight_quant("fp4g32", R)
    Y = O.bf16_decode(O.linear("fp4g32", (codes, scales, np.zeros((8, 0), np.float32)), wq, None, None, 16))
    ref = O.dequant("fp4g32", codes, scales).astype(np.float64) @ O.dequant("fp4g32", *wq).astype(np.float64).T
    assert np.all(np.abs(Y - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6 * np.abs(ref).max())
