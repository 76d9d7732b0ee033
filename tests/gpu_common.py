"""Shared helpers of the GPU parity tests: build/load the library, run the
oracle on the same seeded inputs, and the tolerance the layer output must meet.

Tolerance (per element): |y_gpu - y_oracle| <= 2^-7 |y_oracle| + 1e-3 rms(Y_oracle).
Codes and scales: bit-exact.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL

REL_TOL = 2.0 ** -7
ABS_TOL_RMS = 1e-3


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if major != 10:
        pytest.skip(f"needs sm_100 (B200), found sm_{major}{minor}")


def svdq():
    """The CUDA package, with its library built if the sources are newer."""
    from w4a4_gemm_b200 import build as B
    B.build()
    import w4a4_gemm_b200 as S
    S.lib()
    return S


def y_within_tol(y_gpu_bits, y_ora_bits):
    g = O.bf16_decode(y_gpu_bits).astype(np.float64)
    o = O.bf16_decode(y_ora_bits).astype(np.float64)
    rms = np.sqrt(np.mean(o ** 2)) if o.size else 0.0
    err = np.abs(g - o)
    tol = REL_TOL * np.abs(o) + ABS_TOL_RMS * rms
    bad = err > tol
    return (not bad.any()), {"max_err_over_tol": float(np.max(err / np.maximum(tol, 1e-30))) if o.size else 0.0,
                             "n_bad": int(bad.sum()), "n": int(o.size)}


# X_hat L1 (fp32 on both sides) against the oracle's, per element, relative to
# S[m,j] = sum_k |x_hat[m,k]| |L1[k,j]|:
#   2^-16  the library's factor, inv_lambda L1 carried as a bf16 pair hi + lo
#          (|hi + lo - inv_lambda L1| <= 2^-16 |inv_lambda L1| per term);
#   2^-16  the result carried to the GEMM as a bf16 pair hi + lo;
#   2^-15  fp32 products and sums in different orders on the two sides
#          (about sqrt(K) 2^-24 with random signs; 4 sigma at K = 12288);
# together 2^-14.  One bf16 rounding of the factor alone (2^-8 per term) reads
# 2^-10 to 2^-9 S on the FLUX-shaped layers and fails it.
XL1_REL = 2.0 ** -14


def xl1_within_bound(got, want, X_bits, inv_lambda, L1_bits, rows=None, rel=XL1_REL):
    """|XL1_gpu - XL1_oracle| <= rel * S elementwise (S as above, fp64 from the
    inputs; computed in row blocks to bound the memory)."""
    l1 = np.abs(O.bf16_decode(L1_bits).astype(np.float64))
    inv = np.ones(X_bits.shape[1], np.float32) if inv_lambda is None else np.asarray(inv_lambda, np.float32)
    worst = 0.0
    M = got.shape[0]
    for r0 in range(0, M, 2048):
        xr = O.bf16_decode(X_bits[r0:r0 + 2048])
        S = np.abs((xr * inv[None, :]).astype(np.float32)).astype(np.float64) @ l1
        err = np.abs(got[r0:r0 + 2048].astype(np.float64) - want[r0:r0 + 2048].astype(np.float64))
        worst = max(worst, float(np.max(err / np.maximum(rel * S, 1e-30))) if err.size else 0.0)
    return worst <= 1.0, {"max_err_over_tol": worst}


def to_dev_bits(a: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> device bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_layer(fmt, data, rank, smooth=True, lora=False):
    """Oracle prepare + quantize + layer on a workloads dict (all rows)."""
    Xb = WL.bf16_bits(data["X"])
    Wb = WL.bf16_bits(data["W"])
    bias = WL.bf16_bits(data["bias"]) if data["bias"] is not None else None
    A = WL.bf16_bits(data["lora_A"]) if lora else None
    B = WL.bf16_bits(data["lora_B"]) if lora else None
    return O.layer(fmt, Xb, Wb, rank, bias_bits=bias, lora_A_bits=A, lora_B_bits=B, smooth=smooth)


def load_from_oracle(S, fmt, prep, bias_bits=None, with_lowrank=True):
    """Library handle from the oracle's prepared parts (same R -> same codes)."""
    r = prep["rank"] if with_lowrank else 0
    return S.svdq_load_weights(
        to_dev_f32(prep["R"]), fmt=fmt,
        L1=to_dev_bits(prep["L1"]) if r else None, L2=to_dev_bits(prep["L2"]) if r else None,
        inv_lambda=to_dev_f32(prep["inv_lambda"]), lam=to_dev_f32(prep["lam"]),
        bias=to_dev_bits(bias_bits) if bias_bits is not None else None)
