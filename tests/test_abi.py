"""The C-ABI library builds for sm_100a, loads without a GPU, exports every
entry point include/svdq.h declares, and rejects bad arguments on the host
before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "svdq.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SVDQ_API\s+[\w\s\*]+?\b(svdq_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def L():
    from w4a4_gemm_b200 import build as B
    B.build()
    import w4a4_gemm_b200 as S
    return S.lib()


def test_header_declares_the_layer_calls():
    syms = declared_symbols()
    for name in ("svdq_prepare_weights", "svdq_quantize_act", "svdq_linear", "svdq_load_weights",
                 "svdq_append_lora", "svdq_calib_absmax", "svdq_export_act", "svdq_export_weights"):
        assert name in syms


def test_every_declared_symbol_is_exported(L):
    import w4a4_gemm_b200 as S
    for name in declared_symbols():
        assert hasattr(L, name), name
    assert set(declared_symbols()) == set(S.EXPORTED)


def test_host_side_argument_rejection(L):
    import w4a4_gemm_b200 as S
    assert L.svdq_status_string(2) == b"unsupported shape"
    h = ctypes.c_void_p()
    assert L.svdq_prepare_weights(None, None, ctypes.byref(h)) == 1
    fake = ctypes.c_void_p(0x1000)
    for K, N, rank, fmt, want in [(100, 256, 16, 0, 2), (256, 250, 16, 0, 2), (256, 256, 300, 0, 2),
                                  (256, 256, 16, 7, 1), (0, 256, 16, 0, 2), (128, 64, 65, 1, 2)]:
        d = S._PrepareDesc(fmt, K, N, rank, fake.value, None, None, None, None, 0)
        assert L.svdq_prepare_weights(ctypes.byref(d), None, ctypes.byref(h)) == want, (K, N, rank, fmt)
    d = S._PrepareDesc(0, 256, 256, 16, fake.value, None, None, fake.value, None, 8)
    assert L.svdq_prepare_weights(ctypes.byref(d), None, ctypes.byref(h)) == 1   # LoRA B missing
    d = S._PrepareDesc(0, 256, 256, 16, fake.value, None, None, None, None, 0, 0, 6)
    assert L.svdq_prepare_weights(ctypes.byref(d), None, ctypes.byref(h)) == 1   # unknown flag bits
    e = ctypes.c_int()
    assert L.svdq_weights_scale_exponent(None, ctypes.byref(e)) == 1
    n = ctypes.c_size_t()
    assert L.svdq_act_workspace_bytes(None, 16, ctypes.byref(n)) == 1
    assert L.svdq_quantize_act(None, fake, 16, fake, None) == 1
    assert L.svdq_linear(None, fake, 16, fake, None) == 1
    assert L.svdq_set_wait_budget(0) == 1
    assert L.svdq_set_quant_split(3, 1) == 1 and L.svdq_set_quant_split(1, 16) == 1
    assert L.svdq_set_quant_split(0, 0) == 0
    assert L.svdq_set_gemm_raster(-1) == 1 and L.svdq_set_gemm_raster(0) == 0
    assert L.svdq_set_gemm_kernel(5) == 1 and L.svdq_set_gemm_kernel(-1) == 1 and L.svdq_set_gemm_kernel(0) == 0
    assert L.svdq_calib_absmax(None, 4, 4, None, 0, None) == 1
