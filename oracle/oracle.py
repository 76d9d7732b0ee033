"""Python side of the CPU oracle for the SVDQuant W4A4 + low-rank linear layer.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It never imports the CUDA package and the CUDA package never imports
it.

The arithmetic lives in two places, both written from the SVDQuant paper
("SVDQuant: Absorbing Outliers by Low-Rank Components for 4-Bit Diffusion
Models", arXiv 2411.05007):
  * ``svdq_oracle.c`` (plain C, fp32 where the decision is fp32): number
    formats, the per-group quantizer (Sec. 3), the activation path and the
    fp32-accumulated GEMM;
  * this file (numpy fp64): the smoothing factor (Sec. 4.2, "migrate outliers
    from activations to weights"), the truncated SVD of the smoothed weight
    (Sec. 4.2, Eckart-Young-Mirsky), the residual and the LoRA fold
    (Sec. 5.2, "Integrate LoRA into Nunchaku").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

NVFP4, INT4, FP4G32, W8A8 = 0, 1, 2, 3
_FMT = {"nvfp4": NVFP4, "int4": INT4, "fp4g32": FP4G32, "w8a8": W8A8,
        NVFP4: NVFP4, INT4: INT4, FP4G32: FP4G32, W8A8: W8A8}
GROUP = {NVFP4: 16, INT4: 64, FP4G32: 32}   # W8A8: one scale per row over all of K

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "svdq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libsvdq_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (IEEE fp32, no contraction, no fast-math)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=gnu11",
           "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        L = ctypes.c_long
        _lib.oracle_bf16_decode.restype = ctypes.c_float
        _lib.oracle_bf16_decode.argtypes = [ctypes.c_uint16]
        _lib.oracle_bf16_round.restype = ctypes.c_uint16
        _lib.oracle_bf16_round.argtypes = [ctypes.c_double]
        _lib.oracle_e2m1_decode.restype = ctypes.c_float
        _lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        _lib.oracle_e2m1_round.restype = ctypes.c_uint8
        _lib.oracle_e2m1_round.argtypes = [ctypes.c_float]
        _lib.oracle_e4m3_decode.restype = ctypes.c_float
        _lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        _lib.oracle_e4m3_round_sat.restype = ctypes.c_uint8
        _lib.oracle_e4m3_round_sat.argtypes = [ctypes.c_float]
        _lib.oracle_fp16_decode.restype = ctypes.c_float
        _lib.oracle_fp16_decode.argtypes = [ctypes.c_uint16]
        _lib.oracle_fp16_round_sat.restype = ctypes.c_uint16
        _lib.oracle_fp16_round_sat.argtypes = [ctypes.c_float]
        _lib.oracle_quant_group_nvfp4.argtypes = [P, P, P]
        _lib.oracle_quant_group_fp4g32.argtypes = [P, P, P]
        _lib.oracle_act_quant_w8.argtypes = [I, I, I, P, P, P, P, P, P]
        _lib.oracle_weight_quant_w8.argtypes = [I, I, P, P, P]
        _lib.oracle_linear_rows_w8.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P, I, P]
        _lib.oracle_quant_group_int4.argtypes = [P, P, P]
        for name in ("oracle_bf16_round_array", "oracle_e4m3_round_array",
                     "oracle_e2m1_round_array", "oracle_fp16_round_array"):
            getattr(_lib, name).argtypes = [P, L, P]
            getattr(_lib, name).restype = None
        _lib.oracle_act_quant.argtypes = [I, I, I, I, P, P, P, P, P, P]
        _lib.oracle_weight_quant.argtypes = [I, I, I, P, P, P]
        _lib.oracle_linear_rows.argtypes = [I, I, I, I, I, P, P, P, P, P, P, P, P, I, I, P]
        _lib.oracle_dequant.argtypes = [I, I, I, P, P, P]
    return _lib


def _ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------

def bf16_round(x) -> np.ndarray:
    """Nearest bf16 (ties to even) of each element, as uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().oracle_bf16_round_array(_ptr(x), x.size, _ptr(out))
    return out


def bf16_decode(bits) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def e4m3_round(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().oracle_e4m3_round_array(_ptr(x), x.size, _ptr(out))
    return out


def e2m1_round(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().oracle_e2m1_round_array(_ptr(x), x.size, _ptr(out))
    return out


def fp16_round(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().oracle_fp16_round_array(_ptr(x), x.size, _ptr(out))
    return out


def e4m3_decode(codes) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_e4m3_decode(int(c)) for c in np.ravel(codes)],
                    dtype=np.float32).reshape(np.shape(codes))


def e2m1_decode(codes) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_e2m1_decode(int(c)) for c in np.ravel(codes)],
                    dtype=np.float32).reshape(np.shape(codes))


def fp16_decode(codes) -> np.ndarray:
    L = lib()
    return np.array([L.oracle_fp16_decode(int(c)) for c in np.ravel(codes)],
                    dtype=np.float32).reshape(np.shape(codes))


def quant_group(fmt, v) -> tuple:
    """One group (16 values NVFP4 / 32 FP4 g32 / 64 INT4) -> (codes one per byte, scale code)."""
    fmt = _FMT[fmt]
    v = np.ascontiguousarray(v, dtype=np.float32)
    assert v.size == GROUP[fmt]
    codes = np.zeros(v.size, dtype=np.uint8)
    if fmt == NVFP4:
        sc = np.zeros(1, dtype=np.uint8)
        lib().oracle_quant_group_nvfp4(_ptr(v), _ptr(codes), _ptr(sc))
    elif fmt == FP4G32:
        sc = np.zeros(1, dtype=np.uint8)
        lib().oracle_quant_group_fp4g32(_ptr(v), _ptr(codes), _ptr(sc))
    else:
        sc = np.zeros(1, dtype=np.uint16)
        lib().oracle_quant_group_int4(_ptr(v), _ptr(codes), _ptr(sc))
    return codes, int(sc[0])


# --------------------------------------------------------------------------
# preparation (offline, Sec. 4.2 and Sec. 5.2)
# --------------------------------------------------------------------------

def smoothing(x_absmax: Optional[np.ndarray], W_bits: np.ndarray):
    """Per-input-channel smoothing factor lambda and its fp32 reciprocal.

    lambda_j = sqrt(max|X_j| / max|W_j|) in fp64, rounded to fp32 (the
    square-root balance of SmoothQuant, which SVDQuant Sec. 4.2 cites for
    migrating outliers); lambda_j = 1 where either maximum is 0 or no
    calibration maximum is given.  inv_lambda = fp32(1) / lambda (fp32 IEEE).
    """
    W = bf16_decode(W_bits).astype(np.float64)
    K = W.shape[0]
    if x_absmax is None:
        lam = np.ones(K, dtype=np.float32)
    else:
        xm = np.asarray(x_absmax, dtype=np.float32).astype(np.float64)
        wm = np.max(np.abs(W), axis=1)
        ok = (xm > 0) & (wm > 0)
        lam64 = np.ones(K, dtype=np.float64)
        lam64[ok] = np.sqrt(xm[ok] / wm[ok])
        lam = lam64.astype(np.float32)
    inv = (np.float32(1.0) / lam).astype(np.float32)
    return lam, inv


def calib_absmax(X_bits: np.ndarray) -> np.ndarray:
    """max_m |X[m, j]| per input channel (exact; the calibration statistic)."""
    return np.max(np.abs(bf16_decode(X_bits)), axis=0).astype(np.float32)


def _top_factors_gram(W_hat: np.ndarray, r: int):
    """The top-r singular triplets of W_hat from the fp64 eigendecomposition of
    its smaller Gram matrix (W_hat W_hat^T or W_hat^T W_hat): the same rank-r
    subspace as the SVD, at O(min(K, N)^3) instead of a full SVD."""
    K, N = W_hat.shape
    if K <= N:
        ev, U = np.linalg.eigh(W_hat @ W_hat.T)
        order = np.argsort(ev)[::-1]
        S = np.sqrt(np.maximum(ev[order], 0.0))
        U = U[:, order]
        L1 = U[:, :r] * S[:r]
        L2 = np.divide(U[:, :r].T @ W_hat, S[:r, None], out=np.zeros((r, N)), where=S[:r, None] > 0)
    else:
        ev, V = np.linalg.eigh(W_hat.T @ W_hat)
        order = np.argsort(ev)[::-1]
        S = np.sqrt(np.maximum(ev[order], 0.0))
        V = V[:, order]
        L2 = V[:, :r].T
        L1 = W_hat @ V[:, :r]
    return L1, L2, S


def weight_error(fmt, W_hat: np.ndarray, L1_bits: np.ndarray, L2_bits: np.ndarray, R: np.ndarray):
    """||W_hat - L1 L2 - deq(Q(R))||_F in fp64 for bf16 factors and the fp32
    residual R (K x N), and the dequantized Q(R) (K x N)."""
    codes, scales = weight_quant(fmt, R)
    Rq = dequant(fmt, codes, scales).T.astype(np.float64)
    LL = bf16_decode(L1_bits).astype(np.float64) @ bf16_decode(L2_bits).astype(np.float64)
    return float(np.linalg.norm(W_hat - LL - Rq)), Rq


def prepare(W_bits: np.ndarray, x_absmax: Optional[np.ndarray], rank: int,
            lora_A_bits: Optional[np.ndarray] = None,
            lora_B_bits: Optional[np.ndarray] = None, svd: str = "full",
            refine_fmt=None, refine_iters: int = 0) -> dict:
    """Smoothing, truncated SVD, residual and optional LoRA fold, in fp64.

    W_hat = diag(lambda) W; W_hat = U S V^T (numpy/LAPACK fp64);
    L1 = U[:, :r] S[:r] and L2 = V^T[:r, :] (the optimal rank-r factors),
    rounded to bf16; R = fp32(W_hat - L1_bf16 L2_bf16), so the residual is
    taken against the factors the layer actually uses.  A LoRA (A: K x rl,
    B: rl x N) joins the branch as L1' = [L1 | bf16(diag(lambda) A)],
    L2' = [L2 ; B] without touching R (no requantization).

    svd="gram" takes the top-r factors from the Gram matrix instead of a full
    SVD (for layers of FLUX size, where the full SVD takes minutes); "sigma"
    then holds the square roots of the Gram eigenvalues.

    refine_iters > 0 runs the iterative update of the low-rank branch (Sec. 4.2,
    last paragraph): decompose the part of W_hat the quantized residual misses,
    E = W_hat - deq(Q(R)), into its rank-r factors, take R = W_hat - L1 L2 again,
    quantize it in `refine_fmt`, repeat, and keep the iterate (the SVD start
    included) with the smallest ||W_hat - L1 L2 - deq(Q(R))||_F; the errors of
    all iterates are returned in "refine_errors".
    """
    W = bf16_decode(W_bits).astype(np.float64)
    K, N = W.shape
    lam, inv = smoothing(x_absmax, W_bits)
    W_hat = lam.astype(np.float64)[:, None] * W
    r = int(rank)
    if svd == "gram":
        L1_exact, L2_exact, S = _top_factors_gram(W_hat, r)
    else:
        U, S, Vt = np.linalg.svd(W_hat, full_matrices=False)
        L1_exact = U[:, :r] * S[:r]
        L2_exact = Vt[:r, :]
    L1 = bf16_round(L1_exact)
    L2 = bf16_round(L2_exact)
    R64 = W_hat - bf16_decode(L1).astype(np.float64) @ bf16_decode(L2).astype(np.float64)
    R = R64.astype(np.float32)
    refine_errors = None
    if refine_iters and r:
        err, Rq = weight_error(refine_fmt, W_hat, L1, L2, R)
        refine_errors = [err]
        best = (err, L1, L2, R, L1_exact, L2_exact)
        for _ in range(int(refine_iters)):
            E = W_hat - Rq
            if svd == "gram":
                L1_exact, L2_exact, _ = _top_factors_gram(E, r)
            else:
                U, Se, Vt = np.linalg.svd(E, full_matrices=False)
                L1_exact, L2_exact = U[:, :r] * Se[:r], Vt[:r, :]
            L1, L2 = bf16_round(L1_exact), bf16_round(L2_exact)
            R = (W_hat - bf16_decode(L1).astype(np.float64) @ bf16_decode(L2).astype(np.float64)).astype(np.float32)
            err, Rq = weight_error(refine_fmt, W_hat, L1, L2, R)
            refine_errors.append(err)
            if err < best[0]:
                best = (err, L1, L2, R, L1_exact, L2_exact)
        _, L1, L2, R, L1_exact, L2_exact = best
    out = {"lam": lam, "inv_lambda": inv, "W_hat": W_hat, "sigma": S,
           "L1_exact": L1_exact, "L2_exact": L2_exact, "L1": L1, "L2": L2, "R": R,
           "rank": r, "refine_errors": refine_errors}
    if lora_A_bits is not None:
        A = bf16_decode(lora_A_bits).astype(np.float64)
        L1_lora = bf16_round(lam.astype(np.float64)[:, None] * A)
        out["L1"] = np.ascontiguousarray(np.concatenate([L1, L1_lora], axis=1))
        out["L2"] = np.ascontiguousarray(np.concatenate([L2, lora_B_bits], axis=0))
        out["rank"] = r + A.shape[1]
    return out


# --------------------------------------------------------------------------
# quantization and the layer (C oracle)
# --------------------------------------------------------------------------

def prescale_exponent(fmt, R: np.ndarray) -> int:
    """The optional power-of-two prescale of the weight residual (FP4 formats):
    the largest integer e with 2^e * s_max <= 448, the top of the E4M3 range,
    where s_max = fp32(max|R| / 6) is the largest group scale before rounding;
    0 when R is zero or the format's scales are not E4M3.  The E4M3 scale
    bottoms out at subnormals near 2^-9; multiplying R by 2^e (exact) lifts
    small residuals' scales back into the normal range.  The paper has no
    global scale for its FP4 groups; this is an opt-in reading."""
    fmt = _FMT[fmt]
    if fmt not in (NVFP4, FP4G32):
        return 0
    amax = np.float32(np.max(np.abs(np.asarray(R, dtype=np.float32)))) if np.size(R) else np.float32(0)
    s_max = np.float32(amax) / np.float32(6.0)
    if s_max == 0:
        return 0
    f, q = np.frexp(np.float64(s_max))   # s_max = f 2^q, 0.5 <= f < 1; 448 = 0.875 * 2^9
    e = (9 - int(q)) if f <= 0.875 else (8 - int(q))
    return max(-64, min(64, e))


def weight_quant(fmt, R: np.ndarray, exp: int = 0):
    """Quantize R (K x N fp32) along K per output column -> codes (N x K/2), scales (N x K/g);
    W8A8: codes N x K int8, scales N fp32 (one per output channel).  exp != 0
    quantizes R * 2^exp (the prescale, exact in fp32)."""
    fmt = _FMT[fmt]
    R = np.ascontiguousarray(R, dtype=np.float32)
    if exp:
        R = np.ldexp(R, np.int32(exp)).astype(np.float32)
    K, N = R.shape
    if fmt == W8A8:
        codes = np.zeros((N, K), dtype=np.int8)
        scales = np.zeros(N, dtype=np.float32)
        assert lib().oracle_weight_quant_w8(K, N, _ptr(R), _ptr(codes), _ptr(scales)) == 0
        return codes, scales
    g = GROUP[fmt]
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros((N, K // g), dtype=np.uint16 if fmt == INT4 else np.uint8)
    rc = lib().oracle_weight_quant(fmt, K, N, _ptr(R), _ptr(codes), _ptr(scales))
    assert rc == 0
    return codes, scales


def act_quant(fmt, X_bits: np.ndarray, inv_lambda: Optional[np.ndarray], L1_bits: Optional[np.ndarray]):
    """Smooth and quantize X (M x K bf16) -> codes, scales, and the down-projection
    XL1 = X_hat L1 (M x r fp32): x_hat = fp32(x) * inv_lambda, the value the
    quantizer sees, times the bf16 factor L1, fp32 products and sums in
    increasing k (Sec. 4.2: X_hat = X diag(lambda)^-1; the branch X_hat L1)."""
    fmt = _FMT[fmt]
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    M, K = X_bits.shape
    r = 0 if L1_bits is None else L1_bits.shape[1]
    inv = None if inv_lambda is None else np.ascontiguousarray(inv_lambda, dtype=np.float32)
    if fmt == W8A8:
        # per-token: codes M x K int8, scales M fp32
        codes = np.zeros((M, K), dtype=np.int8)
        scales = np.zeros(M, dtype=np.float32)
        XL1 = np.zeros((M, r), dtype=np.float32)
        L1 = None if L1_bits is None else np.ascontiguousarray(L1_bits, dtype=np.uint16)
        assert lib().oracle_act_quant_w8(M, K, r, _ptr(X_bits), _ptr(inv), _ptr(L1), _ptr(codes),
                                         _ptr(scales), _ptr(XL1)) == 0
        return codes, scales, XL1
    g = GROUP[fmt]
    codes = np.zeros((M, K // 2), dtype=np.uint8)
    scales = np.zeros((M, K // g), dtype=np.uint16 if fmt == INT4 else np.uint8)
    XL1 = np.zeros((M, r), dtype=np.float32)
    L1 = None if L1_bits is None else np.ascontiguousarray(L1_bits, dtype=np.uint16)
    rc = lib().oracle_act_quant(fmt, M, K, r, _ptr(X_bits), _ptr(inv), _ptr(L1),
                                _ptr(codes), _ptr(scales), _ptr(XL1))
    assert rc == 0
    return codes, scales, XL1


def linear(fmt, act, wq, L2_bits: Optional[np.ndarray], bias_bits: Optional[np.ndarray],
           N: int, rows: Optional[np.ndarray] = None, w_exp: int = 0) -> np.ndarray:
    """Y rows (bf16 bits): 4-bit GEMM over groups + XL1 L2 + bias, fp32 accumulation.
    w_exp: the weights were quantized with the prescale 2^w_exp; the group sum is
    scaled back by 2^-w_exp before the branch and the bias are added."""
    fmt = _FMT[fmt]
    cx, sx, XL1 = act
    cw, sw = wq
    M = cx.shape[0]
    K = cx.shape[1] * (1 if fmt == W8A8 else 2)
    r = XL1.shape[1]
    if r:
        assert L2_bits is not None and L2_bits.shape == (r, N)
    rows_arr = None if rows is None else np.ascontiguousarray(rows, dtype=np.int32)
    n_rows = M if rows is None else len(rows_arr)
    Y = np.zeros((n_rows, N), dtype=np.uint16)
    L2 = None if not r else np.ascontiguousarray(L2_bits, dtype=np.uint16)
    bias = None if bias_bits is None else np.ascontiguousarray(bias_bits, dtype=np.uint16)
    if fmt == W8A8:
        rc = lib().oracle_linear_rows_w8(M, N, K, r, _ptr(cx), _ptr(sx), _ptr(XL1), _ptr(cw), _ptr(sw),
                                         _ptr(L2), _ptr(bias), _ptr(rows_arr), n_rows, _ptr(Y))
    else:
        rc = lib().oracle_linear_rows(fmt, M, N, K, r, _ptr(cx), _ptr(sx), _ptr(XL1), _ptr(cw),
                                      _ptr(sw), _ptr(L2), _ptr(bias), _ptr(rows_arr), n_rows, int(w_exp),
                                      _ptr(Y))
    assert rc == 0
    return Y


def dequant(fmt, codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """s * deq(q) for packed codes (rows x K/2) -> fp32 rows x K; W8A8: int8 codes
    rows x K times the row's fp32 scale."""
    fmt = _FMT[fmt]
    if fmt == W8A8:
        return (np.asarray(codes, dtype=np.float32) * np.asarray(scales, dtype=np.float32)[:, None])
    rows, K = codes.shape[0], codes.shape[1] * 2
    out = np.zeros((rows, K), dtype=np.float32)
    rc = lib().oracle_dequant(fmt, rows, K, _ptr(np.ascontiguousarray(codes)),
                              _ptr(np.ascontiguousarray(scales)), _ptr(out))
    assert rc == 0
    return out


def layer(fmt, X_bits, W_bits, rank: int, bias_bits=None, lora_A_bits=None, lora_B_bits=None,
          x_absmax=None, smooth: bool = True, rows=None, pow2_prescale: bool = False) -> dict:
    """The whole layer: prepare (fp64), quantize W and X, GEMM; returns every intermediate."""
    if smooth and x_absmax is None:
        x_absmax = calib_absmax(X_bits)
    prep = prepare(W_bits, x_absmax if smooth else None, rank, lora_A_bits, lora_B_bits)
    w_exp = prescale_exponent(fmt, prep["R"]) if pow2_prescale else 0
    wq = weight_quant(fmt, prep["R"], w_exp)
    r = prep["rank"]
    act = act_quant(fmt, X_bits, prep["inv_lambda"], prep["L1"] if r else None)
    Y = linear(fmt, act, wq, prep["L2"] if r else None, bias_bits, W_bits.shape[1], rows, w_exp)
    return {"prep": prep, "wq": wq, "act": act, "Y": Y, "w_exp": w_exp}
