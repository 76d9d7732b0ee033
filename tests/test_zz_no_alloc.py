"""svdq_forward_noalloc: the forward call for callers that cannot allocate.

Some callers of this library may not call cudaMalloc at all, e.g. a plugin
whose host framework owns every byte of device memory, or a serving loop
that cannot afford cudaMalloc's implicit device synchronization.  For them
the library keeps the activation workspace in a fixed device array.  These
tests call the entry point through the C ABI and check its output against
svdq_forward with a caller workspace, on two calls in a row with different
inputs (the array keeps the previous call's bytes), for both formats, and
that a batch too large for the array is refused before anything runs.  The
kernels are deterministic and only the workspace address differs, so the
outputs must be bit-identical; a second layer whose K and M padding differ
from the first call's checks that no leftover byte of the array reaches Y.

This file runs last (pytest collects it after every other test file).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL
from gpu_common import bits, load_from_oracle, require_gpu, svdq, y_within_tol

pytestmark = pytest.mark.gpu


def _noalloc(S, w, X, Y):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return S.lib().svdq_forward_noalloc(w.handle, ctypes.c_void_p(X.data_ptr()), X.shape[0],
                                        ctypes.c_void_p(Y.data_ptr()), stream)


@pytest.mark.parametrize("fmt,rank", [("nvfp4", 32), ("int4", 48)])
def test_forward_noalloc_matches_forward_on_two_calls(fmt, rank):
    require_gpu()
    S = svdq()
    K, N = 1024, 768
    data = WL.make_small(1000, K, N, rank=rank, fmt=fmt, bias=True, seed=31)
    prep = O.prepare(WL.bf16_bits(data["W"]), O.calib_absmax(WL.bf16_bits(data["X"])), rank)
    w = load_from_oracle(S, fmt, prep, WL.bf16_bits(data["bias"]))
    # call 1: 1000 tokens; call 2: a different, smaller batch over the same array
    X2 = WL.make_activations(WL.LayerSpec("second", K, N, seed=77), 333)
    for X_cpu in (data["X"], X2):
        X = X_cpu.cuda()
        M = X.shape[0]
        ref = S.svdq_forward(w, X)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(S, w, X, Y) == 0
        torch.cuda.synchronize()
        assert S.svdq_get_error() == 0
        assert torch.equal(Y, ref), y_within_tol(bits(Y), bits(ref))[1]


@pytest.mark.parametrize("fmt", ["nvfp4", "int4"])
def test_forward_noalloc_after_a_call_with_other_padding(fmt):
    """A 1000 x 1024 call leaves the array full of bytes; then a layer with
    K = 320 (scale atoms padded past K) at M = 130 (a ragged last row block)
    must still equal svdq_forward bit for bit."""
    require_gpu()
    S = svdq()
    big = WL.make_small(1000, 1024, 512, rank=32, fmt=fmt, seed=41)
    wb = load_from_oracle(S, fmt, O.prepare(WL.bf16_bits(big["W"]), O.calib_absmax(WL.bf16_bits(big["X"])), 32))
    small = WL.make_small(130, 320, 272, rank=48, fmt=fmt, bias=True, seed=42)
    ws = load_from_oracle(S, fmt, O.prepare(WL.bf16_bits(small["W"]), O.calib_absmax(WL.bf16_bits(small["X"])), 48),
                          WL.bf16_bits(small["bias"]))
    try:
        Xb = big["X"].cuda()
        Yb = torch.empty(1000, 512, dtype=torch.bfloat16, device="cuda")
        assert _noalloc(S, wb, Xb, Yb) == 0
        Xs = small["X"].cuda()
        ref = S.svdq_forward(ws, Xs)
        Ys = torch.full((130, 272), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _noalloc(S, ws, Xs, Ys) == 0
        torch.cuda.synchronize()
        assert S.svdq_get_error() == 0
        assert torch.equal(Ys, ref), y_within_tol(bits(Ys), bits(ref))[1]
    finally:
        wb.close()
        ws.close()


def test_forward_noalloc_rejects_batches_beyond_the_array():
    require_gpu()
    S = svdq()
    K, N = 3072, 256
    data = WL.make_small(64, K, N, seed=4)
    prep = O.prepare(WL.bf16_bits(data["W"]), None, 32)
    w = load_from_oracle(S, "nvfp4", prep)
    limit = 16 << 20
    M = 1
    while S.svdq_act_workspace_bytes(w, M) <= limit:
        M *= 2
    X = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(M, N, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(S, w, X, Y) == 2            # SVDQ_ERR_UNSUPPORTED_SHAPE, nothing launched
    torch.cuda.synchronize()
    assert torch.count_nonzero(Y).item() == 0
