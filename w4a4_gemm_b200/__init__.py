"""Python binding of the B200 SVDQuant W4A4 + low-rank linear layer (``libsvdq.so``).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels; torch supplies device memory and the current stream.  The functions
carry the names of the C entry points in ``include/svdq.h``.

Importing this package never builds anything; if ``libsvdq.so`` has not been
built (``python -m w4a4_gemm_b200.build``) every call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvdq.so")

NVFP4, INT4, FP4G32, W8A8 = 0, 1, 2, 3
_FMT = {"nvfp4": NVFP4, "int4": INT4, "fp4g32": FP4G32, "w8a8": W8A8,
        NVFP4: NVFP4, INT4: INT4, FP4G32: FP4G32, W8A8: W8A8}
GROUP = {NVFP4: 16, INT4: 64, FP4G32: 32}   # W8A8: one scale per row over all of K


def _code_scale_arrays(fmt: int, rows: int, K: int):
    """Host arrays for exported codes and scales of `rows` rows: 4-bit formats
    give packed nibble pairs (rows x K/2) and per-group scales; W8A8 gives int8
    codes (rows x K) and one fp32 scale per row."""
    if fmt == W8A8:
        return np.zeros((rows, K), dtype=np.int8), np.zeros(rows, dtype=np.float32)
    return (np.zeros((rows, K // 2), dtype=np.uint8),
            np.zeros((rows, K // GROUP[fmt]), dtype=np.uint16 if fmt == INT4 else np.uint8))

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "device allocation failed",
          4: "CUDA error", 5: "device wait timed out", 6: "cuSOLVER/cuBLAS error"}

EXPORTED = ("svdq_calib_absmax", "svdq_prepare_weights", "svdq_load_weights", "svdq_append_lora",
            "svdq_weights_info", "svdq_weights_refine_error", "svdq_weights_scale_exponent", "svdq_act_workspace_bytes", "svdq_quantize_act", "svdq_linear",
            "svdq_forward", "svdq_forward_noalloc", "svdq_export_act", "svdq_export_weights", "svdq_get_error",
            "svdq_set_wait_budget", "svdq_set_quant_split", "svdq_set_gemm_raster", "svdq_set_gemm_kernel", "svdq_status_string", "svdq_tensor_peak",
            "svdq_weights_destroy")


class SvdqError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)} (status {status})")
        self.status = status


class _PrepareDesc(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int), ("K", ctypes.c_int), ("N", ctypes.c_int),
                ("rank", ctypes.c_int), ("W", ctypes.c_void_p), ("x_absmax", ctypes.c_void_p),
                ("bias", ctypes.c_void_p), ("lora_A", ctypes.c_void_p),
                ("lora_B", ctypes.c_void_p), ("lora_rank", ctypes.c_int),
                ("refine_iters", ctypes.c_int), ("flags", ctypes.c_uint)]


class _PartsDesc(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int), ("K", ctypes.c_int), ("N", ctypes.c_int),
                ("rank", ctypes.c_int), ("inv_lambda", ctypes.c_void_p),
                ("lambda_", ctypes.c_void_p), ("L1", ctypes.c_void_p), ("L2", ctypes.c_void_p),
                ("R", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("flags", ctypes.c_uint)]


WEIGHT_POW2_PRESCALE = 1   # svdq_prepare_desc / svdq_parts_desc flag (see include/svdq.h)


_lib = None


def lib() -> ctypes.CDLL:
    """Load ``libsvdq.so``; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m w4a4_gemm_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, I, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
    L.svdq_calib_absmax.argtypes = [P, I, I, P, I, P]
    L.svdq_prepare_weights.argtypes = [ctypes.POINTER(_PrepareDesc), P, ctypes.POINTER(P)]
    L.svdq_load_weights.argtypes = [ctypes.POINTER(_PartsDesc), P, ctypes.POINTER(P)]
    L.svdq_append_lora.argtypes = [P, P, P, I, P]
    L.svdq_weights_info.argtypes = [P] + [ctypes.POINTER(I)] * 5
    L.svdq_weights_refine_error.argtypes = [P, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]
    L.svdq_weights_scale_exponent.argtypes = [P, ctypes.POINTER(ctypes.c_int)]
    L.svdq_act_workspace_bytes.argtypes = [P, I, ctypes.POINTER(ctypes.c_size_t)]
    L.svdq_quantize_act.argtypes = [P, P, I, P, P]
    L.svdq_linear.argtypes = [P, P, I, P, P]
    L.svdq_forward.argtypes = [P, P, I, P, P, P]
    L.svdq_forward_noalloc.argtypes = [P, P, I, P, P]
    L.svdq_export_act.argtypes = [P, P, I, P, P, P]
    L.svdq_export_weights.argtypes = [P, P, P, P, P, P, P]
    L.svdq_get_error.argtypes = []
    L.svdq_set_wait_budget.argtypes = [LL]
    L.svdq_set_quant_split.argtypes = [I, I]
    L.svdq_set_gemm_raster.argtypes = [I]
    L.svdq_set_gemm_kernel.argtypes = [I]
    L.svdq_status_string.argtypes = [I]
    L.svdq_status_string.restype = ctypes.c_char_p
    L.svdq_tensor_peak.argtypes = [I, LL, P]
    L.svdq_weights_destroy.argtypes = [P]
    L.svdq_weights_destroy.restype = None
    _lib = L
    return L


def _check(rc: int, what: str):
    if rc != 0:
        raise SvdqError(rc, what)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t: torch.Tensor, dtype, name: str, shape=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


class Weights:
    """A prepared layer (owns the library handle)."""

    def __init__(self, handle: ctypes.c_void_p):
        self._h = handle
        fmt, K, N, r, rp = (ctypes.c_int() for _ in range(5))
        _check(lib().svdq_weights_info(handle, ctypes.byref(fmt), ctypes.byref(K), ctypes.byref(N),
                                       ctypes.byref(r), ctypes.byref(rp)), "svdq_weights_info")
        self.fmt, self.K, self.N, self.rank, self.rank_padded = fmt.value, K.value, N.value, r.value, rp.value

    @property
    def handle(self):
        return self._h

    def _refresh(self):
        fmt, K, N, r, rp = (ctypes.c_int() for _ in range(5))
        lib().svdq_weights_info(self._h, ctypes.byref(fmt), ctypes.byref(K), ctypes.byref(N),
                                ctypes.byref(r), ctypes.byref(rp))
        self.rank, self.rank_padded = r.value, rp.value

    def close(self):
        if self._h:
            lib().svdq_weights_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def svdq_calib_absmax(X: torch.Tensor, out: Optional[torch.Tensor] = None, accumulate: bool = False,
                      stream=None) -> torch.Tensor:
    _dev(X, torch.bfloat16, "X")
    M, K = X.shape
    if out is None:
        out = torch.zeros(K, dtype=torch.float32, device=X.device)
    _dev(out, torch.float32, "absmax", (K,))
    _check(lib().svdq_calib_absmax(_ptr(X), M, K, _ptr(out), int(accumulate), _stream(stream)),
           "svdq_calib_absmax")
    return out


def svdq_prepare_weights(W: torch.Tensor, rank: int, fmt="nvfp4", x_absmax: Optional[torch.Tensor] = None,
                         bias: Optional[torch.Tensor] = None, lora_A: Optional[torch.Tensor] = None,
                         lora_B: Optional[torch.Tensor] = None, refine_iters: int = 0,
                         pow2_prescale: bool = False, stream=None) -> Weights:
    _dev(W, torch.bfloat16, "W")
    K, N = W.shape
    if x_absmax is not None:
        _dev(x_absmax, torch.float32, "x_absmax", (K,))
    if bias is not None:
        _dev(bias, torch.bfloat16, "bias", (N,))
    rl = 0
    if lora_A is not None:
        rl = lora_A.shape[1]
        _dev(lora_A, torch.bfloat16, "lora_A", (K, rl))
        _dev(lora_B, torch.bfloat16, "lora_B", (rl, N))
    d = _PrepareDesc(_FMT[fmt], K, N, int(rank), W.data_ptr(),
                     x_absmax.data_ptr() if x_absmax is not None else None,
                     bias.data_ptr() if bias is not None else None,
                     lora_A.data_ptr() if lora_A is not None else None,
                     lora_B.data_ptr() if lora_B is not None else None, rl, int(refine_iters),
                     WEIGHT_POW2_PRESCALE if pow2_prescale else 0)
    h = ctypes.c_void_p()
    _check(lib().svdq_prepare_weights(ctypes.byref(d), _stream(stream), ctypes.byref(h)),
           "svdq_prepare_weights")
    return Weights(h)


def svdq_load_weights(R: torch.Tensor, fmt="nvfp4", L1: Optional[torch.Tensor] = None,
                      L2: Optional[torch.Tensor] = None, inv_lambda: Optional[torch.Tensor] = None,
                      lam: Optional[torch.Tensor] = None, bias: Optional[torch.Tensor] = None,
                      pow2_prescale: bool = False, stream=None) -> Weights:
    _dev(R, torch.float32, "R")
    K, N = R.shape
    r = 0 if L1 is None else L1.shape[1]
    if r:
        _dev(L1, torch.bfloat16, "L1", (K, r))
        _dev(L2, torch.bfloat16, "L2", (r, N))
    for t, n in ((inv_lambda, "inv_lambda"), (lam, "lambda")):
        if t is not None:
            _dev(t, torch.float32, n, (K,))
    if bias is not None:
        _dev(bias, torch.bfloat16, "bias", (N,))
    d = _PartsDesc(_FMT[fmt], K, N, r, inv_lambda.data_ptr() if inv_lambda is not None else None,
                   lam.data_ptr() if lam is not None else None,
                   L1.data_ptr() if r else None, L2.data_ptr() if r else None, R.data_ptr(),
                   bias.data_ptr() if bias is not None else None,
                   WEIGHT_POW2_PRESCALE if pow2_prescale else 0)
    h = ctypes.c_void_p()
    _check(lib().svdq_load_weights(ctypes.byref(d), _stream(stream), ctypes.byref(h)), "svdq_load_weights")
    return Weights(h)


def svdq_append_lora(w: Weights, A: torch.Tensor, B: torch.Tensor, stream=None) -> Weights:
    rl = A.shape[1]
    _dev(A, torch.bfloat16, "lora_A", (w.K, rl))
    _dev(B, torch.bfloat16, "lora_B", (rl, w.N))
    _check(lib().svdq_append_lora(w.handle, _ptr(A), _ptr(B), rl, _stream(stream)), "svdq_append_lora")
    w._refresh()
    return w


def svdq_act_workspace_bytes(w: Weights, M: int) -> int:
    n = ctypes.c_size_t()
    _check(lib().svdq_act_workspace_bytes(w.handle, int(M), ctypes.byref(n)), "svdq_act_workspace_bytes")
    return n.value


def alloc_workspace(w: Weights, M: int, device=None) -> torch.Tensor:
    """A device byte buffer large enough for svdq_quantize_act at M tokens."""
    return torch.empty(max(svdq_act_workspace_bytes(w, M), 256), dtype=torch.uint8,
                       device=device or torch.device("cuda", torch.cuda.current_device()))


def svdq_quantize_act(w: Weights, X: torch.Tensor, workspace: torch.Tensor, stream=None):
    _dev(X, torch.bfloat16, "X")
    M, K = X.shape
    if K != w.K:
        raise ValueError(f"X has K={K}, layer has K={w.K}")
    if workspace.numel() < svdq_act_workspace_bytes(w, M):
        raise ValueError("workspace too small")
    _check(lib().svdq_quantize_act(w.handle, _ptr(X), M, _ptr(workspace), _stream(stream)),
           "svdq_quantize_act")


def svdq_linear(w: Weights, workspace: torch.Tensor, M: int, Y: torch.Tensor, stream=None):
    _dev(Y, torch.bfloat16, "Y", (M, w.N))
    _check(lib().svdq_linear(w.handle, _ptr(workspace), int(M), _ptr(Y), _stream(stream)), "svdq_linear")


def svdq_forward(w: Weights, X: torch.Tensor, Y: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _dev(X, torch.bfloat16, "X")
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, w.N, dtype=torch.bfloat16, device=X.device)
    _dev(Y, torch.bfloat16, "Y", (M, w.N))
    if workspace is None:
        workspace = alloc_workspace(w, M, X.device)
    _check(lib().svdq_forward(w.handle, _ptr(X), M, _ptr(Y), _ptr(workspace), _stream(stream)),
           "svdq_forward")
    return Y


def svdq_forward_noalloc(w: Weights, X: torch.Tensor, Y: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """svdq_forward with the library's fixed device workspace (no allocation
    inside the call; see include/svdq.h for the size limit and the sharing rule)."""
    _dev(X, torch.bfloat16, "X")
    M = X.shape[0]
    if Y is None:
        Y = torch.empty(M, w.N, dtype=torch.bfloat16, device=X.device)
    _dev(Y, torch.bfloat16, "Y", (M, w.N))
    _check(lib().svdq_forward_noalloc(w.handle, _ptr(X), M, _ptr(Y), _stream(stream)),
           "svdq_forward_noalloc")
    return Y


def svdq_export_act(w: Weights, workspace: torch.Tensor, M: int):
    """(codes, scales, xl1 M x rank float32) on the host: codes M x K/2 uint8 and
    scales M x K/g for the 4-bit formats, int8 M x K and fp32 M for W8A8."""
    codes, scales = _code_scale_arrays(w.fmt, M, w.K)
    xl1 = np.zeros((M, w.rank), dtype=np.float32)
    _check(lib().svdq_export_act(w.handle, _ptr(workspace), int(M), codes.ctypes.data_as(ctypes.c_void_p),
                                 scales.ctypes.data_as(ctypes.c_void_p),
                                 xl1.ctypes.data_as(ctypes.c_void_p) if w.rank else None),
           "svdq_export_act")
    return codes, scales, xl1


def svdq_export_weights(w: Weights) -> dict:
    codes, scales = _code_scale_arrays(w.fmt, w.N, w.K)
    L1 = np.zeros((w.K, w.rank), dtype=np.uint16)
    L2 = np.zeros((w.rank, w.N), dtype=np.uint16)
    inv = np.zeros(w.K, dtype=np.float32)
    lam = np.zeros(w.K, dtype=np.float32)
    vp = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    _check(lib().svdq_export_weights(w.handle, vp(codes), vp(scales), vp(L1) if w.rank else None,
                                     vp(L2) if w.rank else None, vp(inv), vp(lam)), "svdq_export_weights")
    return {"codes": codes, "scales": scales, "L1": L1, "L2": L2, "inv_lambda": inv, "lambda": lam}


def svdq_get_error() -> int:
    return int(lib().svdq_get_error())


def svdq_weights_scale_exponent(w: "Weights") -> int:
    """e of the weight prescale: the stored codes and scales are those of R * 2^e."""
    e = ctypes.c_int()
    _check(lib().svdq_weights_scale_exponent(w.handle, ctypes.byref(e)), "svdq_weights_scale_exponent")
    return e.value


def svdq_weights_refine_error(w: "Weights"):
    """(initial, kept) weight error of the refinement, -1 where none ran."""
    a, b = ctypes.c_double(), ctypes.c_double()
    _check(lib().svdq_weights_refine_error(w.handle, ctypes.byref(a), ctypes.byref(b)),
           "svdq_weights_refine_error")
    return a.value, b.value


def svdq_tensor_peak(fmt: str, steps: int, stream=None):
    """Launch the tensor-core ceiling kernel (see include/svdq.h); time it with
    CUDA events.  FLOP = SMs * steps * 4 * 2 * 128 * 256 * (64 NVFP4 / FP4 g32 | 32 INT4, W8A8)."""
    _check(lib().svdq_tensor_peak(_FMT[fmt], int(steps), _stream(stream)), "svdq_tensor_peak")


def svdq_set_wait_budget(cycles: int):
    _check(lib().svdq_set_wait_budget(int(cycles)), "svdq_set_wait_budget")


def svdq_set_quant_split(S: int = 0, C: int = 0):
    """Force the activation kernel's launch shape (see include/svdq.h); 0, 0 = automatic."""
    _check(lib().svdq_set_quant_split(int(S), int(C)), "svdq_set_quant_split")


def svdq_set_gemm_kernel(kind: int = 0):
    """Force the FP4 GEMM kernel: 1 = one CTA per tile, 2 = CTA pairs on 256 x 256 tiles (the
    tiles of a short last round as 256 x 128 halves), 3 = CTA pairs on 256 x 192 tiles with two
    accumulators, 4 = as 2 with whole tiles only; 0 = automatic (see include/svdq.h)."""
    _check(lib().svdq_set_gemm_kernel(int(kind)), "svdq_set_gemm_kernel")


def svdq_set_gemm_raster(group_m: int = 0):
    """Force the GEMM's tile order (row blocks per group, see include/svdq.h); 0 = automatic."""
    _check(lib().svdq_set_gemm_raster(int(group_m)), "svdq_set_gemm_raster")
