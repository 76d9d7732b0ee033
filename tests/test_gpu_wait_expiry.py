"""A bounded device wait that runs out: the kernels report it and the
library keeps working.

Every wait of the hot kernels on an mbarrier is bounded by a clock64 budget
(svdq_set_wait_budget); when it runs out the waiting role sets a bit of the
sticky device error word (bit 0: activation kernel, bit 1: GEMM), raises its
CTA's abort flag so the other roles stop waiting, and the CTA still drains
the copies and MMAs it issued, frees its TMEM and meets its cluster barriers
before it leaves.  Here the budget is cut to one cycle, so every wait that is
not satisfied on its first poll runs out: svdq_forward must come back with
the error word set (and nothing else wrong with the context), and with the
budget restored the same layer must again give bit for bit the result it
gave before.  No fault is involved: the waits end by their own limit.
"""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL
from gpu_common import load_from_oracle, require_gpu, svdq

pytestmark = pytest.mark.gpu

DEFAULT_BUDGET = 1 << 31     # the library's default (about 1 s at 1965 MHz)


@pytest.mark.parametrize("fmt,gemm_kind", [("nvfp4", 0), ("nvfp4", 1), ("int4", 0)])
def test_wait_budget_expiry_is_reported_and_recovered(fmt, gemm_kind):
    require_gpu()
    S = svdq()
    M, K, N = 1000, 3072, 1536
    data = WL.make_small(M, K, N, rank=32, fmt=fmt, seed=17)
    prep = O.prepare(WL.bf16_bits(data["W"]), O.calib_absmax(WL.bf16_bits(data["X"])), 32)
    w = load_from_oracle(S, fmt, prep)
    X = data["X"].cuda()
    try:
        S.svdq_set_gemm_kernel(gemm_kind)       # 0: the default (CTA pairs); 1: single CTAs
        ref = S.svdq_forward(w, X)
        torch.cuda.synchronize()
        assert S.svdq_get_error() == 0
        Y = torch.empty_like(ref)
        seen = 0
        try:
            S.svdq_set_wait_budget(1)
            for _ in range(3):
                S.svdq_forward(w, X, Y)
                err = S.svdq_get_error()        # synchronizes; negative if the context broke
                assert err >= 0 and (err & ~3) == 0, err
                seen |= err
        finally:
            S.svdq_set_wait_budget(DEFAULT_BUDGET)
        assert seen != 0, "no wait ran out with a one-cycle budget"
        again = S.svdq_forward(w, X)
        torch.cuda.synchronize()
        assert S.svdq_get_error() == 0
        assert torch.equal(again, ref)
    finally:
        S.svdq_set_gemm_kernel(0)
        w.close()
