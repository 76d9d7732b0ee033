"""Pins of the oracle's preparation (SVDQuant Sec. 4.2, Sec. 5.2) and layer (Eq. 5).

What the paper fixes and these tests check:
  * smoothing balances the channel maxima of X_hat and W_hat;
  * the SVD factors are the optimal rank-r approximation (Eckart-Young-Mirsky):
    ||W_hat - L1 L2||_F^2 = sum of the discarded sigma_i^2, the same as the sum of
    the smallest eigenvalues of W_hat^T W_hat (an independent LAPACK routine);
  * full rank leaves a zero residual and gives Y = X W up to 16-bit rounding;
  * with lambda = 1 and r = 0 the layer is plain W4A4, equal to a float64
    matmul of the dequantized operands (decoded here from the published
    E2M1 table and torch's float8 decoder, not from the oracle);
  * Proposition 4.1's error bound holds;
  * the ablation ordering of Sec. 5.2 (SVDQuant < smoothing only < naive) and
    the error falling with the rank (Fig. 11) hold on outlier-heavy inputs;
  * a LoRA folds into the branch exactly and leaves R untouched;
  * the hand-worked tiny layer.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL


def _f64(bits):
    return O.bf16_decode(bits).astype(np.float64)


def _deq_independent(fmt, codes, scales, golden):
    """Dequantize with the published E2M1 table / integer codes and torch's scale decoders."""
    rows, K = codes.shape[0], codes.shape[1] * 2
    nib = np.empty((rows, K), dtype=np.uint8)
    nib[:, 0::2] = codes & 0xF
    nib[:, 1::2] = codes >> 4
    if fmt == "nvfp4":
        table = {}
        for row in golden("e2m1_grid.txt"):
            c, v = row[0].split()
            table[int(c)] = float(v)
        q = np.vectorize(table.get)(nib).astype(np.float64)
        s = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).double().numpy()
        g = 16
    else:
        q = np.where(nib >= 8, nib.astype(np.int64) - 16, nib).astype(np.float64)
        s = scales.view(np.float16).astype(np.float64)
        g = 64
    return q * np.repeat(s, g, axis=1)


def test_smoothing_balances_channel_maxima():
    d = WL.make_small(128, 256, 192, x_outliers=6)
    Xb, Wb = WL.bf16_bits(d["X"]), WL.bf16_bits(d["W"])
    xm = O.calib_absmax(Xb)
    lam, inv = O.smoothing(xm, Wb)
    wm = np.max(np.abs(_f64(Wb)), axis=1)
    x_hat_max = xm.astype(np.float64) * inv.astype(np.float64)
    w_hat_max = lam.astype(np.float64) * wm
    assert np.allclose(x_hat_max, w_hat_max, rtol=1e-6)
    assert np.allclose(x_hat_max, np.sqrt(xm * wm), rtol=1e-6)
    # the outlier channels get the largest lambda
    top = np.argsort(-xm)[:6]
    assert set(top) == set(np.argsort(-lam)[:6])


def test_smoothing_degenerate_channels():
    W = torch.zeros(32, 16, dtype=torch.bfloat16)
    W[1:] = 0.5
    xm = np.ones(32, dtype=np.float32)
    xm[2] = 0.0
    lam, inv = O.smoothing(xm, WL.bf16_bits(W))
    assert lam[0] == 1.0 and lam[2] == 1.0 and inv[0] == 1.0
    lam, inv = O.smoothing(None, WL.bf16_bits(W))
    assert np.all(lam == 1.0) and np.all(inv == 1.0)


@pytest.mark.parametrize("K,N,r", [(128, 96, 16), (96, 160, 32), (64, 64, 8)])
def test_eckart_young_optimal_rank_r(K, N, r):
    d = WL.make_small(64, K, N, w_outlier_rows=3)
    Xb, Wb = WL.bf16_bits(d["X"]), WL.bf16_bits(d["W"])
    p = O.prepare(Wb, O.calib_absmax(Xb), r)
    W_hat = p["W_hat"]
    resid = np.linalg.norm(W_hat - p["L1_exact"] @ p["L2_exact"]) ** 2
    ev = np.linalg.eigvalsh(W_hat.T @ W_hat if N <= K else W_hat @ W_hat.T)  # ascending
    discarded = np.sum(ev[: len(ev) - r])
    assert abs(resid - discarded) <= 1e-9 * np.linalg.norm(W_hat) ** 2
    assert abs(resid - np.sum(p["sigma"][r:] ** 2)) <= 1e-10 * np.linalg.norm(W_hat) ** 2
    # orthonormal right factor, L1 columns orthogonal with norms sigma
    assert np.allclose(p["L2_exact"] @ p["L2_exact"].T, np.eye(r), atol=1e-12)
    G = p["L1_exact"].T @ p["L1_exact"]
    assert np.allclose(G, np.diag(p["sigma"][:r] ** 2), atol=1e-9 * p["sigma"][0] ** 2)
    # no other rank-r factorization does better: a random subspace and a perturbed one
    rng = np.random.default_rng(8)
    Q, _ = np.linalg.qr(rng.standard_normal((N, r)))
    assert np.linalg.norm(W_hat - W_hat @ Q @ Q.T) ** 2 > resid
    V = p["L2_exact"].T + 1e-3 * rng.standard_normal((N, r))
    Q2, _ = np.linalg.qr(V)
    assert np.linalg.norm(W_hat - W_hat @ Q2 @ Q2.T) ** 2 >= resid * (1 - 1e-12)
    # the fp32 residual is taken against the bf16 factors and sits near the EYM norm
    R_norm2 = np.linalg.norm(p["R"].astype(np.float64)) ** 2
    assert abs(R_norm2 - discarded) <= 0.05 * discarded + 1e-3 * np.linalg.norm(W_hat) ** 2


def test_full_rank_zero_residual_and_exact_product():
    M, K, N = 32, 64, 48
    d = WL.make_small(M, K, N)
    Xb, Wb = WL.bf16_bits(d["X"]), WL.bf16_bits(d["W"])
    res = O.layer("nvfp4", Xb, Wb, rank=min(K, N))
    p = res["prep"]
    exact_resid = p["W_hat"] - p["L1_exact"] @ p["L2_exact"]
    assert np.linalg.norm(exact_resid) <= 1e-12 * np.linalg.norm(p["W_hat"])
    Y = _f64(res["Y"])
    ref = _f64(Xb) @ _f64(Wb)
    # only the 16-bit rounding of x_hat, L1, L2, XL1 and Y remains
    assert np.linalg.norm(Y - ref) <= 0.01 * np.linalg.norm(ref)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_plain_w4a4_reduction(fmt, golden):
    """lambda = 1, r = 0: the layer is Q(X) Q(W), equal to a float64 matmul of the
    independently dequantized operands (differences: fp32 accumulation only)."""
    M, K, N = 24, 256, 40
    d = WL.make_small(M, K, N, bias=True)
    Xb, Wb = WL.bf16_bits(d["X"]), WL.bf16_bits(d["W"])
    res = O.layer(fmt, Xb, Wb, rank=0, bias_bits=WL.bf16_bits(d["bias"]), smooth=False)
    cx, sx, _ = res["act"]
    cw, sw = res["wq"]
    # the residual at r = 0 is W itself (lambda = 1)
    assert np.array_equal(res["prep"]["R"], O.bf16_decode(Wb))
    qx = _deq_independent(fmt, cx, sx, golden)
    qw = _deq_independent(fmt, cw, sw, golden)
    ref = qx @ qw.T + _f64(WL.bf16_bits(d["bias"]))[None, :]
    Y = _f64(res["Y"])
    tol = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.sqrt(np.mean(ref ** 2))
    assert np.all(np.abs(Y - ref) <= tol)
    # Q(X) is a quantization of X itself (lambda = 1): per-group relative error is small
    X = _f64(Xb)
    assert np.linalg.norm(qx - X) < 0.2 * np.linalg.norm(X)


def test_proposition_4_1_error_bound(golden):
    M, K, N = 64, 256, 96
    d = WL.make_small(M, K, N)
    Xb, Wb = WL.bf16_bits(d["X"]), WL.bf16_bits(d["W"])
    res = O.layer("nvfp4", Xb, Wb, rank=0, smooth=False)
    X, W = _f64(Xb), _f64(Wb)
    QX = _deq_independent("nvfp4", *res["act"][:2], golden)
    QW = _deq_independent("nvfp4", *res["wq"], golden).T
    E = np.linalg.norm(X @ W - QX @ QW)
    bound = (np.linalg.norm(X) * np.linalg.norm(W - QW)
             + np.linalg.norm(X - QX) * (np.linalg.norm(W) + np.linalg.norm(W - QW)))
    assert E <= bound


def test_ablation_ordering_and_rank_trend():
    """Sec. 5.2 ablation: smoothing + low-rank branch beats smoothing alone and
    naive W4A4 on outlier-heavy data; Fig. 11: error falls as the rank grows."""
    M, K, N = 128, 512, 256
    d = WL.make_small(M, K, N, x_outliers=8, w_outlier_rows=4)
    Xb, Wb = WL.bf16_bits(d["X"]), WL.bf16_bits(d["W"])
    ref = _f64(Xb) @ _f64(Wb)

    def err(rank, smooth):
        Y = _f64(O.layer("nvfp4", Xb, Wb, rank=rank, smooth=smooth)["Y"])
        return np.linalg.norm(Y - ref) / np.linalg.norm(ref)

    naive, smooth_only, svdq = err(0, False), err(0, True), err(32, True)
    assert svdq < smooth_only < naive
    errs = [err(r, True) for r in (0, 16, 32, 64)]
    assert all(b < a for a, b in zip(errs, errs[1:])), errs


def test_lora_fold_exact_without_requantization():
    M, K, N, r, rl = 16, 128, 64, 16, 8
    d = WL.make_small(M, K, N, lora_rank=rl)
    Xb, Wb = WL.bf16_bits(d["X"]), WL.bf16_bits(d["W"])
    A, B = WL.bf16_bits(d["lora_A"]), WL.bf16_bits(d["lora_B"])
    xm = O.calib_absmax(Xb)
    p0 = O.prepare(Wb, xm, r)
    p1 = O.prepare(Wb, xm, r, A, B)
    assert p1["rank"] == r + rl
    assert np.array_equal(p0["R"], p1["R"])                  # R untouched
    assert np.array_equal(p1["L1"][:, :r], p0["L1"]) and np.array_equal(p1["L2"][:r], p0["L2"])
    wq0, wq1 = O.weight_quant("nvfp4", p0["R"]), O.weight_quant("nvfp4", p1["R"])
    assert all(np.array_equal(a, b) for a, b in zip(wq0, wq1))
    X = _f64(Xb)
    x_hat = X * p1["inv_lambda"].astype(np.float64)
    lhs = x_hat @ _f64(p1["L1"]) @ _f64(p1["L2"])
    rhs = x_hat @ _f64(p0["L1"]) @ _f64(p0["L2"]) + X @ _f64(A) @ _f64(B)
    # exact up to the bf16 rounding of diag(lambda) A
    assert np.linalg.norm(lhs - rhs) <= 2.0 ** -8 * np.linalg.norm(X @ _f64(A) @ _f64(B))


def test_hand_worked_tiny_layer(golden):
    rows = {r[0]: r[1] for r in golden("layer_tiny.txt")}
    vec = lambda k: np.array([float(t) for t in rows[k].split()])
    hexv = lambda k: np.array([int(t, 16) for t in rows[k].split()])
    K, N = 16, 2
    X = torch.from_numpy(vec("x")[None, :].astype(np.float32)).to(torch.bfloat16)
    Xb = WL.bf16_bits(X)
    R = np.stack([vec("r0"), vec("r1")], axis=1).astype(np.float32)
    cw, sw = O.weight_quant("nvfp4", R)
    for n in range(N):
        c = hexv(f"w_codes{n}")
        assert np.array_equal(cw[n] & 0xF, c[0::2]) and np.array_equal(cw[n] >> 4, c[1::2])
        assert sw[n, 0] == hexv(f"w_scale{n}")[0]
    # plain: r = 0, no bias
    act = O.act_quant("nvfp4", Xb, np.ones(K, np.float32), None)
    c = hexv("x_codes")
    assert np.array_equal(act[0][0] & 0xF, c[0::2]) and act[1][0, 0] == hexv("x_scale")[0]
    Y = O.bf16_decode(O.linear("nvfp4", act, (cw, sw), None, None, N))
    assert np.array_equal(Y[0], vec("y_plain").astype(np.float32))
    # full: r = 1, L1[0,0] = 0.5, L2 = [1, -1], bias [0.5, -0.25]
    L1 = O.bf16_round(np.eye(K, 1) * 0.5)
    L2 = O.bf16_round(np.array([[1.0, -1.0]]))
    bias = O.bf16_round(np.array([0.5, -0.25]))
    act = O.act_quant("nvfp4", Xb, np.ones(K, np.float32), L1)
    assert act[2][0, 0] == 3.0
    Y = O.bf16_decode(O.linear("nvfp4", act, (cw, sw), L2, bias, N))
    assert np.array_equal(Y[0], vec("y_full").astype(np.float32))
    # smooth: 1/lambda = 0.75 on channel 0 reaches both the quantizer and the branch
    act = O.act_quant("nvfp4", Xb, vec("inv_l").astype(np.float32), L1)
    c = hexv("xs_codes")
    assert np.array_equal(act[0][0] & 0xF, c[0::2]) and np.array_equal(act[0][0] >> 4, c[1::2])
    assert act[1][0, 0] == hexv("xs_scale")[0]
    assert act[2][0, 0] == vec("xs_xl1")[0]
    Y = O.bf16_decode(O.linear("nvfp4", act, (cw, sw), L2, bias, N))
    assert np.array_equal(Y[0], vec("y_smooth").astype(np.float32))


def test_row_subset_matches_full():
    d = WL.make_small(40, 128, 48, bias=True)
    Xb, Wb = WL.bf16_bits(d["X"]), WL.bf16_bits(d["W"])
    full = O.layer("nvfp4", Xb, Wb, 16, bias_bits=WL.bf16_bits(d["bias"]))
    rows = np.array([39, 0, 17, 5])
    Ys = O.linear("nvfp4", full["act"], full["wq"], full["prep"]["L2"], WL.bf16_bits(d["bias"]),
                  48, rows=rows)
    assert np.array_equal(Ys, full["Y"][rows])


@pytest.mark.parametrize("K,N", [(96, 160), (160, 96)])
def test_gram_route_spans_the_svd_subspace(K, N):
    """prepare(svd="gram") (top-r factors from the smaller Gram matrix, used for
    the full-size GPU parity tests) gives the same rank-r product, singular
    values and, where the bf16 rounding of the factors agrees, the same residual
    as the full SVD; a dropped Sigma or a transposed Gram matrix would not."""
    d = WL.make_small(32, K, N, w_outlier_rows=3, seed=K + N)
    Wb = WL.bf16_bits(d["W"])
    xm = O.calib_absmax(WL.bf16_bits(d["X"]))
    a = O.prepare(Wb, xm, 24)
    b = O.prepare(Wb, xm, 24, svd="gram")
    pa = a["L1_exact"] @ a["L2_exact"]
    pb = b["L1_exact"] @ b["L2_exact"]
    assert np.linalg.norm(pa - pb) <= 1e-9 * np.linalg.norm(pa)
    assert np.allclose(a["sigma"][:24], b["sigma"][:24], rtol=1e-9)
    assert np.array_equal(a["lam"], b["lam"]) and np.array_equal(a["inv_lambda"], b["inv_lambda"])
    # the residuals differ only through the bf16 rounding of sign-flipped factors
    Ra = a["R"].astype(np.float64)
    Rb = b["R"].astype(np.float64)
    assert np.linalg.norm(Ra - Rb) <= 2.0 ** -7 * np.linalg.norm(pa)


@pytest.mark.parametrize("fmt", ["nvfp4", "int4", "fp4g32"])
def test_iterative_refinement_keeps_the_best_iterate(fmt):
    """Sec. 4.2, last paragraph: re-decomposing W_hat - deq(Q(R)) and requantizing
    lowers the weight error on outlier-heavy weights; the returned parts are the
    iterate with the smallest error, and they keep the residual convention."""
    d = WL.make_small(64, 256, 192, w_outlier_rows=6, seed=11)
    Wb = WL.bf16_bits(d["W"])
    xm = O.calib_absmax(WL.bf16_bits(d["X"]))
    plain = O.prepare(Wb, xm, 16)
    none = O.prepare(Wb, xm, 16, refine_fmt=fmt, refine_iters=0)
    assert none["refine_errors"] is None
    assert np.array_equal(none["L1"], plain["L1"]) and np.array_equal(none["R"], plain["R"])
    ref = O.prepare(Wb, xm, 16, refine_fmt=fmt, refine_iters=4)
    errs = ref["refine_errors"]
    assert len(errs) == 5
    e0, _ = O.weight_error(fmt, plain["W_hat"], plain["L1"], plain["L2"], plain["R"])
    assert errs[0] == pytest.approx(e0, rel=1e-12)
    got, _ = O.weight_error(fmt, ref["W_hat"], ref["L1"], ref["L2"], ref["R"])
    assert got == pytest.approx(min(errs), rel=1e-12)
    assert min(errs) < 0.97 * errs[0]
    R64 = ref["W_hat"] - O.bf16_decode(ref["L1"]).astype(np.float64) @ O.bf16_decode(ref["L2"]).astype(np.float64)
    assert np.array_equal(ref["R"], R64.astype(np.float32))
