"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Codes and scales must be bit-exact; Y must be within |d| <= 2^-7 |y| +
1e-3 rms(Y) and X_hat L1 within the bound of gpu_common.xl1_within_bound.  Both sides get the same seeded inputs; the
library gets the oracle's prepared factors (so both quantize the same R),
except in the tests of the library's own preparation, which are checked
against invariants of the SVD instead.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL
from gpu_common import (bits, xl1_within_bound, load_from_oracle, oracle_layer, require_gpu, svdq,
                        to_dev_bits, to_dev_f32, y_within_tol)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def S():
    require_gpu()
    return svdq()


def _run_layer(S, w, X_bits):
    X = to_dev_bits(X_bits)
    M = X.shape[0]
    ws = S.alloc_workspace(w, M)
    Y = torch.empty(M, w.N, dtype=torch.bfloat16, device="cuda")
    S.svdq_quantize_act(w, X, ws)
    S.svdq_linear(w, ws, M, Y)
    torch.cuda.synchronize()
    assert S.svdq_get_error() == 0
    return ws, Y


def _golden_groups(golden, name):
    return {r[0]: np.array([float(t) for t in r[1].split()], dtype=np.float32) for r in golden(name)}


@pytest.mark.parametrize("fmt", ["nvfp4", "fp4g32", "int4"])
def test_quantizer_ties_at_non_power_of_two_scales(S, fmt, golden):
    """The hand-worked tie groups (scales 0x27 and 0x23; fp16 0x2e80), whose
    entries sit exactly on rounding midpoints where v * fp32(1/s) and the exact
    quotient v / s part, through the GPU's activation quantizer (as bf16 rows,
    lambda = 1) and its weight quantizer (as fp32 residual columns, with some
    entries moved one fp32 ulp off the midpoint): codes and scales bit-exact
    against the oracle, Y within tolerance."""
    rng = np.random.default_rng(11)
    if fmt == "int4":
        base = [_golden_groups(golden, "int4_groups.txt")["C"]]
        g = 64
    else:
        gg = _golden_groups(golden, "nvfp4_groups.txt")
        base = [gg["G"], gg["H"]]
        g = 16 if fmt == "nvfp4" else 32
    base = [np.concatenate([b, np.zeros(g - b.size, np.float32)]) for b in base]
    M, K, N = 130, 256, 272

    def group(nudge):
        v = base[rng.integers(len(base))][rng.permutation(g)] * (-1 if rng.integers(2) else 1)
        if nudge:   # one fp32 ulp off some midpoints, never the group maximum
            amax = np.max(np.abs(v))
            for i in np.nonzero((np.abs(v) < amax) & (v != 0) & (rng.random(g) < 0.5))[0]:
                v[i] = np.nextafter(v[i], np.float32(np.inf if rng.integers(2) else -np.inf), dtype=np.float32)
        return v.astype(np.float32)

    X = np.stack([np.concatenate([group(False) for _ in range(K // g)]) for _ in range(M)])
    Xb = WL.bf16_bits(torch.from_numpy(X).to(torch.bfloat16))
    assert np.array_equal(O.bf16_decode(Xb), X)     # every tie value is bf16-exact
    R = np.stack([np.concatenate([group(n % 2 == 1) for _ in range(K // g)]) for n in range(N)], axis=1)
    R = np.ascontiguousarray(R, dtype=np.float32)
    ones = np.ones(K, np.float32)
    w = S.svdq_load_weights(to_dev_f32(R), fmt=fmt, inv_lambda=to_dev_f32(ones), lam=to_dev_f32(ones))
    try:
        wq = O.weight_quant(fmt, R)
        e = S.svdq_export_weights(w)
        assert np.array_equal(e["scales"], wq[1]), "weight scales differ"
        assert np.array_equal(e["codes"], wq[0]), "weight codes differ"
        act = O.act_quant(fmt, Xb, ones, None)
        ws, Y = _run_layer(S, w, Xb)
        codes, scales, _ = S.svdq_export_act(w, ws, M)
        assert np.array_equal(scales, act[1]), "activation scales differ"
        assert np.array_equal(codes, act[0]), "activation codes differ"
        ok, info = y_within_tol(bits(Y), O.linear(fmt, act, wq, None, None, N))
        assert ok, ("Y", info)
    finally:
        w.close()


def test_weight_quantizer_edge_values(S):
    """Ties, subnormal and saturating scales, negative values rounding to zero."""
    groups = [
        [6, 3, -1.5, 0.25] + [0] * 12,
        [1, 0.75, -0.5, 0.1] + [0] * 12,
        [6, 5, 2.5, 0.75, 1.25, 1.75, 3.5, -5, -0.25, 0.5] + [0] * 6,
        [0.003, -0.002, 0.001] + [0] * 13,
        [0.006, -0.0012] + [0] * 14,
        [3000, 2300, 2200, -1000] + [0] * 12,
        [-0.01, 1, -0.2, 0.12] + [0] * 12,
        [0.0] * 16,
    ]
    rng = np.random.default_rng(11)
    K = 256
    cols = []
    for g in groups:
        c = np.zeros(K, dtype=np.float32)
        c[:16] = g
        c[16:] = rng.standard_normal(K - 16) * 10.0 ** rng.uniform(-3, 3)
        cols.append(c)
    while len(cols) < 32:
        cols.append((rng.standard_normal(K) * 10.0 ** rng.uniform(-4, 3)).astype(np.float32))
    R = np.stack(cols, axis=1).astype(np.float32)     # K x 32
    for fmt in ("nvfp4", "int4", "fp4g32"):
        w = S.svdq_load_weights(to_dev_f32(R), fmt=fmt)
        got = S.svdq_export_weights(w)
        codes, scales = O.weight_quant(fmt, R)
        assert np.array_equal(got["scales"], scales), fmt
        assert np.array_equal(got["codes"], codes), (fmt, np.argwhere(got["codes"] != codes)[:8])


def test_weight_quantizer_edge_values_w8a8(S):
    """W8A8 per-channel int8: exact ties at scale 1 and 1/2 (round half to
    even), an all-zero channel, tiny and large channels."""
    K = 256
    rng = np.random.default_rng(12)
    cols = []
    c = np.zeros(K, dtype=np.float32)
    c[:8] = [127, 2.5, -0.5, 3.5, 1.5, -126.5, 0.5, -2.5]          # s = 1
    cols.append(c)
    c = np.zeros(K, dtype=np.float32)
    c[:6] = [63.5, 0.25, 0.75, -0.25, -63.25, 1.25]                 # s = 1/2
    cols.append(c)
    cols.append(np.zeros(K, dtype=np.float32))
    cols.append((rng.standard_normal(K) * 1e-3).astype(np.float32))
    cols.append((rng.standard_normal(K) * 3000).astype(np.float32))
    while len(cols) < 32:
        cols.append((rng.standard_normal(K) * 10.0 ** rng.uniform(-4, 3)).astype(np.float32))
    R = np.stack(cols, axis=1).astype(np.float32)     # K x 32
    w = S.svdq_load_weights(to_dev_f32(R), fmt="w8a8")
    got = S.svdq_export_weights(w)
    codes, scales = O.weight_quant("w8a8", R)
    assert np.array_equal(got["scales"], scales)
    assert np.array_equal(got["codes"], codes), np.argwhere(got["codes"] != codes)[:8]
    assert list(got["codes"][0, :8]) == [127, 2, 0, 4, 2, -126, 0, -2]
    assert list(got["codes"][1, :6]) == [127, 0, 2, 0, -126, 2]
    assert got["scales"][2] == 0 and not got["codes"][2].any()


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "fp4g32", "w8a8"])
def test_act_quantizer_edge_rows(S, fmt):
    """Activation rows with exact ties, an all-zero row, huge and tiny rows,
    through svdq_quantize_act with lambda = 1; codes and scales bit-exact."""
    K, N, M = 256, 64, 40
    rng = np.random.default_rng(13)
    X = (rng.standard_normal((M, K)) * 10.0 ** rng.uniform(-2, 2, size=(M, 1))).astype(np.float32)
    X[0] = 0
    X[0, :8] = [127, 2.5, -0.5, 3.5, 1.5, -126.5, 0.5, -2.5]
    X[1] = 0
    X[2] *= 1e4
    X[3] *= 1e-30
    X[4, :16] = [6, 3, -1.5, 0.25, 5, 2.5, 0.75, 1.25, 1.75, 3.5, -5, -0.25, 0.5, 0, 0, 0]
    Xb = WL.bf16_bits(torch.from_numpy(X).to(torch.bfloat16))
    R = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    ones = np.ones(K, dtype=np.float32)
    w = S.svdq_load_weights(to_dev_f32(R), fmt=fmt, inv_lambda=to_dev_f32(ones), lam=to_dev_f32(ones))
    ws, Y = _run_layer(S, w, Xb)
    codes, scales, _ = S.svdq_export_act(w, ws, M)
    want = O.act_quant(fmt, Xb, ones, None)
    assert np.array_equal(scales, want[1]), np.argwhere(scales != want[1])[:8]
    assert np.array_equal(codes, want[0]), np.argwhere(codes != want[0])[:8]
    w.close()


SHAPES = [
    # M, K, N, rank, fmt, bias
    (1, 256, 256, 32, "nvfp4", False),
    (77, 512, 384, 32, "nvfp4", True),
    (200, 1024, 512, 16, "nvfp4", False),
    (256, 320, 272, 32, "nvfp4", True),      # K % 256 != 0, N % 256 != 0
    (300, 768, 256, 64, "nvfp4", False),
    (129, 512, 256, 0, "nvfp4", True),       # plain W4A4
    (130, 512, 256, 48, "nvfp4", False),     # rank padded to 64
    (96, 512, 256, 32, "int4", True),
    (200, 1024, 512, 48, "int4", False),
    (64, 256, 272, 0, "int4", False),
    (130, 320, 256, 32, "int4", True),       # five groups of 64: the last stage holds one
    (77, 512, 384, 32, "fp4g32", True),      # one E4M3 scale per 32 values, stored per 16
    (300, 320, 272, 48, "fp4g32", False),
    (77, 512, 384, 16, "w8a8", True),        # int8, per-token / per-channel scales
    (300, 320, 272, 16, "w8a8", False),      # K % 128 != 0: the last K step is half padding
    (129, 512, 256, 0, "w8a8", True),        # plain W8A8
    (200, 1024, 512, 64, "w8a8", False),
]


@pytest.mark.parametrize("M,K,N,rank,fmt,bias", SHAPES)
def test_layer_parity_small(S, M, K, N, rank, fmt, bias):
    data = WL.make_small(M, K, N, rank=rank, fmt=fmt, bias=bias, seed=M + K + N)
    ref = oracle_layer(fmt, data, rank)
    prep = ref["prep"]
    bias_bits = WL.bf16_bits(data["bias"]) if bias else None
    w = load_from_oracle(S, fmt, prep, bias_bits)
    wexp = S.svdq_export_weights(w)
    assert np.array_equal(wexp["codes"], ref["wq"][0]) and np.array_equal(wexp["scales"], ref["wq"][1])
    ws, Y = _run_layer(S, w, WL.bf16_bits(data["X"]))
    codes, scales, xl1 = S.svdq_export_act(w, ws, M)
    assert np.array_equal(scales, ref["act"][1]), "activation scales differ"
    assert np.array_equal(codes, ref["act"][0]), "activation codes differ"
    if rank:
        ok, info = xl1_within_bound(xl1, ref["act"][2], WL.bf16_bits(data["X"]), prep["inv_lambda"], prep["L1"])
        assert ok, ("XL1", info)
    ok, info = y_within_tol(bits(Y), ref["Y"])
    assert ok, ("Y", info)


@pytest.mark.parametrize("M,K,N,rank,fmt", [
    (300, 320, 272, 48, "nvfp4"),    # 5 sub-tiles: clusters of 4 leave one CTA without a K range
    (200, 512, 256, 32, "int4"),
    (130, 1024, 256, 16, "fp4g32"),
    (77, 512, 384, 16, "w8a8"),
])
def test_forced_launch_shapes(S, M, K, N, rank, fmt):
    """Every launch shape of the activation kernel (stacked sub-tiles x CTAs per
    cluster) gives the oracle's codes and scales bit for bit and X_hat L1, Y
    within tolerance; shapes a layer cannot use fall back to the automatic one."""
    data = WL.make_small(M, K, N, rank=rank, fmt=fmt, seed=M + K + 1)
    ref = oracle_layer(fmt, data, rank)
    w = load_from_oracle(S, fmt, ref["prep"])
    try:
        for st in (1, 2, 4, 8):
            for cl in (1, 2, 4, 8):
                S.svdq_set_quant_split(st, cl)
                ws, Y = _run_layer(S, w, WL.bf16_bits(data["X"]))
                codes, scales, xl1 = S.svdq_export_act(w, ws, M)
                assert np.array_equal(scales, ref["act"][1]), (st, cl, "scales")
                assert np.array_equal(codes, ref["act"][0]), (st, cl, "codes")
                ok, info = xl1_within_bound(xl1, ref["act"][2], WL.bf16_bits(data["X"]),
                                            ref["prep"]["inv_lambda"], ref["prep"]["L1"])
                assert ok, (st, cl, "XL1", info)
                ok, info = y_within_tol(bits(Y), ref["Y"])
                assert ok, (st, cl, "Y", info)
    finally:
        S.svdq_set_quant_split(0, 0)
        w.close()


@pytest.mark.parametrize("M,K,N,rank,fmt", [
    (600, 512, 784, 16, "nvfp4"),    # odd number of 128-row blocks: the last pair's second CTA has no rows
    (130, 1024, 256, 32, "fp4g32"),
    (256, 256, 512, 0, "nvfp4"),     # no low-rank tail
    (1000, 768, 272, 48, "nvfp4"),   # ragged last column block, 3 tail chunks
    (384, 320, 1024, 32, "nvfp4"),   # K below two K steps
    (520, 512, 208, 32, "nvfp4"),    # one 192-column tile and a 16-column one
    (1792, 512, 3072, 32, "nvfp4"),  # 84 tiles of 256 x 256: a full round of the pairs, then halves
])
def test_forced_gemm_kernel(S, M, K, N, rank, fmt):
    """The FP4 GEMM on single CTAs (128 x 256 tiles), on CTA pairs with 256 x 256
    tiles (at these sizes every tile as two 256 x 128 halves, kind 2, or whole,
    kind 4) and on CTA pairs with 256 x 192 tiles and two accumulators
    (cta_group::2 MMAs) sums the same products in the same order: Y bit for bit
    the same, within tolerance of the oracle."""
    data = WL.make_small(M, K, N, rank=rank, fmt=fmt, seed=M + K)
    ref = oracle_layer(fmt, data, rank)
    w = load_from_oracle(S, fmt, ref["prep"])
    try:
        Ys = {}
        for kind in (1, 2, 3, 4):
            S.svdq_set_gemm_kernel(kind)
            _, Y = _run_layer(S, w, WL.bf16_bits(data["X"]))
            ok, info = y_within_tol(bits(Y), ref["Y"])
            assert ok, (kind, info)
            Ys[kind] = bits(Y)
        for kind in (2, 3, 4):
            assert np.array_equal(Ys[1], Ys[kind]), kind
    finally:
        S.svdq_set_gemm_kernel(0)
        w.close()


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "w8a8"])
def test_forced_gemm_raster(S, fmt):
    """The GEMM's tile order changes which CTA computes a tile and when, not what
    it computes: every order gives the same Y bit for bit, within tolerance of
    the oracle (5 row blocks, 4 column blocks with a ragged last one)."""
    M, K, N, rank = 600, 512, 784, 16
    data = WL.make_small(M, K, N, rank=rank, fmt=fmt, seed=91)
    ref = oracle_layer(fmt, data, rank)
    w = load_from_oracle(S, fmt, ref["prep"])
    try:
        S.svdq_set_gemm_raster(0)
        _, Y0 = _run_layer(S, w, WL.bf16_bits(data["X"]))
        ok, info = y_within_tol(bits(Y0), ref["Y"])
        assert ok, ("auto", info)
        for g in (1, 2, 3, 5, 64):
            S.svdq_set_gemm_raster(g)
            _, Y = _run_layer(S, w, WL.bf16_bits(data["X"]))
            assert np.array_equal(bits(Y), bits(Y0)), g
    finally:
        S.svdq_set_gemm_raster(0)
        w.close()


@pytest.mark.parametrize("fmt", ["nvfp4", "fp4g32"])
def test_pow2_prescale_parity(S, fmt):
    """Small weights with the power-of-two prescale: the library's exponent, weight
    codes and scales are the oracle's for R * 2^e, and Y (also after a LoRA is
    appended, which rebuilds the scaled tail operand) is within tolerance of the
    oracle's layer that scales the group sum back by 2^-e."""
    M, K, N, r, rl = 150, 512, 384, 32, 16
    d = WL.make_small(M, K, N, rank=r, fmt=fmt, bias=True, lora_rank=rl, seed=31)
    Xb = WL.bf16_bits(d["X"])
    Wb = WL.bf16_bits((d["W"].float() * 0.01).to(torch.bfloat16))
    bb = WL.bf16_bits(d["bias"])
    prep = O.prepare(Wb, O.calib_absmax(Xb), r)
    e = O.prescale_exponent(fmt, prep["R"])
    assert e > 0
    wq = O.weight_quant(fmt, prep["R"], e)
    w = S.svdq_load_weights(to_dev_f32(prep["R"]), fmt=fmt, L1=to_dev_bits(prep["L1"]),
                            L2=to_dev_bits(prep["L2"]), inv_lambda=to_dev_f32(prep["inv_lambda"]),
                            lam=to_dev_f32(prep["lam"]), bias=to_dev_bits(bb), pow2_prescale=True)
    try:
        assert S.svdq_weights_scale_exponent(w) == e
        ex = S.svdq_export_weights(w)
        assert np.array_equal(ex["scales"], wq[1]) and np.array_equal(ex["codes"], wq[0])
        assert np.array_equal(ex["L2"], prep["L2"])          # the exported factor is unscaled
        act = O.act_quant(fmt, Xb, prep["inv_lambda"], prep["L1"])
        y_ref = O.linear(fmt, act, wq, prep["L2"], bb, N, w_exp=e)
        ws, Y = _run_layer(S, w, Xb)
        ok, info = y_within_tol(bits(Y), y_ref)
        assert ok, ("Y", info)
        # LoRA folded into the branch of the prescaled handle
        S.svdq_append_lora(w, d["lora_A"].cuda(), d["lora_B"].cuda())
        ref = O.prepare(Wb, O.calib_absmax(Xb), r, WL.bf16_bits(d["lora_A"]), WL.bf16_bits(d["lora_B"]))
        act = O.act_quant(fmt, Xb, ref["inv_lambda"], ref["L1"])
        y_ref = O.linear(fmt, act, wq, ref["L2"], bb, N, w_exp=e)
        ws, Y = _run_layer(S, w, Xb)
        ok, info = y_within_tol(bits(Y), y_ref)
        assert ok, ("Y after LoRA", info)
    finally:
        w.close()


def test_pow2_prescale_in_preparation(S):
    """svdq_prepare_weights with the prescale: the codes are the oracle quantizer's
    of R * 2^e for the library's own residual, and on a weight whose scales would
    sit in the E4M3 subnormal range the layer is much closer to X W."""
    M, K, N = 128, 512, 256
    d = WL.make_small(M, K, N, rank=0, seed=32, x_outliers=0)
    Wt = (d["W"].float() * 0.02).to(torch.bfloat16)
    Xb, Wb = WL.bf16_bits(d["X"]), WL.bf16_bits(Wt)
    exact = O.bf16_decode(Xb).astype(np.float64) @ O.bf16_decode(Wb).astype(np.float64)
    err = {}
    for pre in (False, True):
        w = S.svdq_prepare_weights(Wt.cuda(), 0, "nvfp4", pow2_prescale=pre)
        try:
            e = S.svdq_weights_scale_exponent(w)
            R = O.bf16_decode(Wb).astype(np.float32)        # rank 0, lambda = 1: R = W
            assert e == (O.prescale_exponent("nvfp4", R) if pre else 0)
            ex = S.svdq_export_weights(w)
            codes, scales = O.weight_quant("nvfp4", R, e)
            assert np.array_equal(ex["scales"], scales) and np.array_equal(ex["codes"], codes)
            ws, Y = _run_layer(S, w, Xb)
            err[pre] = np.linalg.norm(O.bf16_decode(bits(Y)) - exact) / np.linalg.norm(exact)
        finally:
            w.close()
    assert err[True] < 0.25 and err[False] > 0.9, err


def test_prepare_weights_invariants(S):
    """The library's own preparation (cuSOLVER on the fp64 Gram matrix):
    1/lambda bit-exact, the branch spans the oracle's optimal rank-r subspace,
    and the residual carries the Eckart-Young energy."""
    M, K, N, r = 256, 512, 384, 32
    data = WL.make_small(M, K, N, w_outlier_rows=4, seed=5)
    Xb, Wb = WL.bf16_bits(data["X"]), WL.bf16_bits(data["W"])
    xm = O.calib_absmax(Xb)
    prep = O.prepare(Wb, xm, r)
    X = data["X"].cuda()
    W = data["W"].cuda()
    xabs = S.svdq_calib_absmax(X)
    torch.cuda.synchronize()
    assert np.array_equal(xabs.cpu().numpy(), xm)
    w = S.svdq_prepare_weights(W, r, "nvfp4", x_absmax=xabs)
    e = S.svdq_export_weights(w)
    assert np.array_equal(e["inv_lambda"], prep["inv_lambda"])
    assert np.array_equal(e["lambda"], prep["lam"])
    L1L2_lib = O.bf16_decode(e["L1"]).astype(np.float64) @ O.bf16_decode(e["L2"]).astype(np.float64)
    L1L2_ora = prep["L1_exact"] @ prep["L2_exact"]
    assert np.linalg.norm(L1L2_lib - L1L2_ora) <= 0.02 * np.linalg.norm(L1L2_ora)
    resid = np.linalg.norm(prep["W_hat"] - L1L2_lib) ** 2
    eym = np.sum(prep["sigma"][r:] ** 2)
    assert eym <= resid <= eym * 1.02 + 1e-4 * np.linalg.norm(prep["W_hat"]) ** 2
    # the whole library path approximates X W as well as the oracle's layer does
    ws, Y = _run_layer(S, w, Xb)
    ref = O.layer("nvfp4", Xb, Wb, r)
    exact = O.bf16_decode(Xb).astype(np.float64) @ O.bf16_decode(Wb).astype(np.float64)
    e_lib = np.linalg.norm(O.bf16_decode(bits(Y)) - exact) / np.linalg.norm(exact)
    e_ora = np.linalg.norm(O.bf16_decode(ref["Y"]) - exact) / np.linalg.norm(exact)
    assert e_lib <= 1.1 * e_ora + 1e-3, (e_lib, e_ora)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "fp4g32", "w8a8"])
def test_lora_fold_parity(S, fmt):
    M, K, N, r, rl = 160, 512, 384, 32, 16
    data = WL.make_small(M, K, N, rank=r, fmt=fmt, lora_rank=rl, seed=9)
    ref = oracle_layer(fmt, data, r, lora=True)
    base = O.prepare(WL.bf16_bits(data["W"]), O.calib_absmax(WL.bf16_bits(data["X"])), r)
    w = load_from_oracle(S, fmt, base)
    before = S.svdq_export_weights(w)
    S.svdq_append_lora(w, data["lora_A"].cuda(), data["lora_B"].cuda())
    assert w.rank == r + rl
    after = S.svdq_export_weights(w)
    assert np.array_equal(before["codes"], after["codes"]) and np.array_equal(before["scales"], after["scales"])
    assert np.array_equal(after["L1"], ref["prep"]["L1"]) and np.array_equal(after["L2"], ref["prep"]["L2"])
    ws, Y = _run_layer(S, w, WL.bf16_bits(data["X"]))
    codes, scales, xl1 = S.svdq_export_act(w, ws, M)
    assert np.array_equal(codes, ref["act"][0]) and np.array_equal(scales, ref["act"][1])
    ok, info = y_within_tol(bits(Y), ref["Y"])
    assert ok, info


def test_forward_matches_two_calls_and_is_deterministic(S):
    data = WL.make_small(333, 512, 256, seed=3)
    prep = O.prepare(WL.bf16_bits(data["W"]), O.calib_absmax(WL.bf16_bits(data["X"])), 32)
    w = load_from_oracle(S, "nvfp4", prep)
    X = data["X"].cuda()
    Y1 = S.svdq_forward(w, X)
    Y2 = S.svdq_forward(w, X)
    ws, Y3 = _run_layer(S, w, WL.bf16_bits(data["X"]))
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2) and torch.equal(Y1, Y3)


def test_empty_batch_is_a_noop(S):
    data = WL.make_small(16, 256, 256, seed=1)
    prep = O.prepare(WL.bf16_bits(data["W"]), None, 16)
    w = load_from_oracle(S, "nvfp4", prep)
    X = torch.empty(0, 256, dtype=torch.bfloat16, device="cuda")
    Y = S.svdq_forward(w, X)
    assert Y.shape == (0, 256)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "fp4g32", "w8a8"])
def test_prepare_refinement(S, fmt):
    """Iterative refinement of the branch in svdq_prepare_weights: the kept
    error is what the exported parts give, it drops below the SVD start, and
    both ends agree with the oracle's refinement of the same layer."""
    M, K, N, r = 128, 256, 192, 16
    data = WL.make_small(M, K, N, w_outlier_rows=6, seed=11)
    Xb, Wb = WL.bf16_bits(data["X"]), WL.bf16_bits(data["W"])
    xm = O.calib_absmax(Xb)
    ora = O.prepare(Wb, xm, r, refine_fmt=fmt, refine_iters=4)
    w = S.svdq_prepare_weights(data["W"].cuda(), r, fmt, x_absmax=S.svdq_calib_absmax(data["X"].cuda()),
                               refine_iters=4)
    e0, kept = S.svdq_weights_refine_error(w)
    e = S.svdq_export_weights(w)
    What = ora["W_hat"]
    LL = O.bf16_decode(e["L1"]).astype(np.float64) @ O.bf16_decode(e["L2"]).astype(np.float64)
    Rq = O.dequant(fmt, e["codes"], e["scales"]).T.astype(np.float64)
    assert np.linalg.norm(What - LL - Rq) == pytest.approx(kept, rel=1e-9)
    assert kept <= e0 and kept < 0.97 * e0
    errs = ora["refine_errors"]
    assert e0 == pytest.approx(errs[0], rel=0.02)
    assert kept == pytest.approx(min(errs), rel=0.03)
    # the exported codes are the oracle quantizer's codes of the kept residual
    R = (What - LL).astype(np.float32)
    codes, scales = O.weight_quant(fmt, R)
    assert np.array_equal(scales, e["scales"]) and np.array_equal(codes, e["codes"])
    w.close()


@pytest.mark.parametrize("fmt,pre", [("nvfp4", False), ("nvfp4", True), ("fp4g32", False), ("int4", False)])
def test_refined_weights_through_the_gemm(S, fmt, pre):
    """After a refinement that may keep an earlier iterate, every GEMM kernel reads
    the kept codes and scales (and the layouts derived from them): Y from each
    kernel is the oracle's layer of the exported parts, bit for bit the same
    across the FP4 kernels.  With the prescale, the kept iterate's exponent."""
    M, K, N, r = 300, 512, 400, 16
    data = WL.make_small(M, K, N, w_outlier_rows=6, seed=13)
    Xb = WL.bf16_bits(data["X"])
    W = data["W"]
    if pre:
        W = (W.float() * 0.02).to(torch.bfloat16)   # residual scales in the E4M3 subnormal range
    w = S.svdq_prepare_weights(W.cuda(), r, fmt, x_absmax=S.svdq_calib_absmax(data["X"].cuda()),
                               refine_iters=4, pow2_prescale=pre)
    try:
        e = S.svdq_export_weights(w)
        exp = S.svdq_weights_scale_exponent(w)
        act = O.act_quant(fmt, Xb, e["inv_lambda"], e["L1"])
        Y_ora = O.linear(fmt, act, (e["codes"], e["scales"]), e["L2"], None, N, w_exp=exp)
        kinds = (1, 2, 3) if fmt != "int4" else (0,)
        Ys = []
        for kind in kinds:
            S.svdq_set_gemm_kernel(kind)
            _, Y = _run_layer(S, w, Xb)
            ok, info = y_within_tol(bits(Y), Y_ora)
            assert ok, (kind, info)
            Ys.append(bits(Y))
        for y in Ys[1:]:
            assert np.array_equal(y, Ys[0])
    finally:
        S.svdq_set_gemm_kernel(0)
        w.close()

