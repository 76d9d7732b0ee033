"""GPU parity at the full sizes of the five workloads, through the same calls
bench.py times (svdq_quantize_act then svdq_linear on a workspace).

Both sides get the same seeded X, W, bias and LoRA of each workload and the
same prepared parts: the oracle's smoothing and its rank-r factors, taken
from the fp64 Gram matrix (oracle.prepare(svd="gram"), the same subspace as
the full SVD, which would take minutes at these sizes).  Checked:
  * weight codes and scales: every value, bit-exact;
  * activation codes and scales: every row, bit-exact;
  * X_hat L1: every row, within 2^-14 sum_k |x_hat_k| |L1_kj| (gpu_common);
  * Y: every row up to M = 512; above, the first and last row of every
    128-row block, a seeded row in each of its middle 32-row slices and 32
    seeded rows anywhere (all N columns), within |dy| <= 2^-7 |y| + 1e-3 rms(y).
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL
from gpu_common import (bits, xl1_within_bound, load_from_oracle, require_gpu, svdq, to_dev_bits,
                        y_within_tol)

pytestmark = pytest.mark.gpu

CASES = [
    ("c1_small", None, 256, None),
    ("c2_qkv", None, 4608, None),
    ("c3_mlp", "fc1", 4608, None),
    ("c3_mlp", "fc2", 4608, None),
    ("c4_int4_lora", None, 4608, None),
    ("c2_qkv", None, 4608, ("w8a8", 16)),    # the paper's 8-bit setting: W8A8 with rank 16
    ("c3_mlp", "fc2", 4608, ("w8a8", 16)),
] + [("c5_block", layer, M, None) for layer in ("qkv", "out", "fc1", "fc2") for M in (1024, 4096, 16384)]

_parts = {}


@pytest.fixture(scope="module")
def S():
    require_gpu()
    return svdq()


def _prepared(spec):
    """Oracle parts of one layer, computed once per layer for every M."""
    key = (spec.name, spec.K, spec.N, spec.seed, spec.fmt, spec.rank)
    if key not in _parts:
        W, bias, A, B = WL.make_weights(spec)
        # calibration: the layer's largest token batch of the workload
        M_cal = max(m for c in WL.CONFIGS.values() for l in c.layers
                    if dataclasses.replace(l, fmt=spec.fmt, rank=spec.rank) == spec for m in c.Ms)
        Xc = WL.bf16_bits(WL.make_activations(spec, M_cal))
        prep = O.prepare(WL.bf16_bits(W), O.calib_absmax(Xc), spec.rank,
                         WL.bf16_bits(A) if A is not None else None,
                         WL.bf16_bits(B) if B is not None else None, svd="gram")
        wq = O.weight_quant(spec.fmt, prep["R"])
        _parts.clear()   # keep one layer's weights in memory at a time
        _parts[key] = (prep, wq, WL.bf16_bits(bias) if bias is not None else None)
    return _parts[key]


def _sample_rows(M, seed):
    """Rows whose Y is checked: all of them up to 512; above, in every 128-row
    block its first and last row and one seeded row in each of its two middle
    32-row slices -- so every (row block, epilogue warp quarter) position of
    every output tile is checked -- plus 32 seeded rows anywhere."""
    if M <= 512:
        return np.arange(M, dtype=np.int32)
    rng = np.random.default_rng(seed)
    rows = [rng.integers(0, M, size=32)]
    for b in range(0, M, 128):
        last = min(b + 127, M - 1)
        rows.append(np.array([b, last]))
        for q in (1, 2):
            lo = b + 32 * q
            if lo <= last:
                rows.append(rng.integers(lo, min(lo + 32, last + 1), size=1))
    return np.unique(np.concatenate(rows)).astype(np.int32)


def _case_id(case):
    config, layer, M, override = case
    return "-".join([config] + ([layer] if layer else []) + [str(M)] +
                    ([f"{override[0]}_r{override[1]}"] if override else []))


@pytest.mark.parametrize("config,layer,M,override", CASES, ids=[_case_id(c) for c in CASES])
def test_fullsize_parity(S, config, layer, M, override):
    spec = WL.layer_spec(config, layer)
    if override is not None:
        spec = dataclasses.replace(spec, fmt=override[0], rank=override[1])
    prep, wq, bias_bits = _prepared(spec)
    w = load_from_oracle(S, spec.fmt, prep, bias_bits)
    try:
        e = S.svdq_export_weights(w)
        assert np.array_equal(e["scales"], wq[1]), "weight scales differ"
        assert np.array_equal(e["codes"], wq[0]), "weight codes differ"

        Xb = WL.bf16_bits(WL.make_activations(spec, M))
        r = prep["rank"]
        act = O.act_quant(spec.fmt, Xb, prep["inv_lambda"], prep["L1"] if r else None)

        X = to_dev_bits(Xb)
        ws = S.alloc_workspace(w, M)
        Y = torch.empty(M, spec.N, dtype=torch.bfloat16, device="cuda")
        S.svdq_quantize_act(w, X, ws)
        S.svdq_linear(w, ws, M, Y)
        torch.cuda.synchronize()
        assert S.svdq_get_error() == 0
        codes, scales, xl1 = S.svdq_export_act(w, ws, M)
        assert np.array_equal(scales, act[1]), "activation scales differ"
        assert np.array_equal(codes, act[0]), "activation codes differ"
        if r:
            ok, info = xl1_within_bound(xl1, act[2], Xb, prep["inv_lambda"], prep["L1"])
            assert ok, ("XL1", info)

        rows = _sample_rows(M, seed=M + spec.K + spec.N)
        y_ref = O.linear(spec.fmt, act, wq, prep["L2"] if r else None, bias_bits, spec.N, rows=rows)
        y_gpu = bits(Y)[rows]
        ok, info = y_within_tol(y_gpu, y_ref)
        assert ok, ("Y", info)
    finally:
        w.close()
