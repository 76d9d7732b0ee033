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


def close_f32(got: np.ndarray, want: np.ndarray, rel=2.0 ** -12):
    """fp32 intermediates (X_hat L1): |d| <= rel |want| + rel rms(want)."""
    g, o = got.astype(np.float64), want.astype(np.float64)
    rms = np.sqrt(np.mean(o ** 2)) if o.size else 0.0
    err = np.abs(g - o)
    tol = rel * np.abs(o) + rel * rms
    return bool(np.all(err <= tol)), {"max_err_over_tol": float(np.max(err / np.maximum(tol, 1e-30))) if o.size else 0.0}


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
