#!/usr/bin/env python
"""Benchmark of the SVDQuant W4A4 + low-rank linear layer on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
the fused activation kernel (smoothing + quantize + down-projection) and the
fused 4-bit GEMM (+ up-projection + bias), both through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config c5_block] [--layer fc2] [--M 16384]

Default workload: the largest FLUX-shaped GEMM of the workloads, the DiT
block's MLP fc2 layer at M = 16384 tokens, K = 12288 -> N = 3072, rank 32,
NVFP4 (bias).  The metric is the effective throughput 2*M*K*N / (layer time),
in TFLOP/s; the line also carries us/layer, the per-kernel times, the GEMM's
roofline fraction against the FP4 tensor peak and the activation kernel's
against HBM bandwidth.  Other layers: --config / --layer / --M (e.g.
--config c2_qkv for the attention QKV projection at M = 4608).

Between timed steps a 512 MiB buffer is rewritten to flush the 126 MB L2.
Under torchrun every rank runs its own batch of the same layer (token-parallel
weak scaling, no data-path collective); the time is the max over ranks.

`--impl reference` times the CPU oracle (test infrastructure: a plain C /
numpy restatement of the method) on a bounded sample of rows of the same
workload and prints the same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as WL  # noqa: E402

METRIC = "SVDQuant W4A4+low-rank linear: µs/layer, effective TFLOPS, % of FP4 peak"
UNIT = "TFLOP/s"
FLUSH_BYTES = 512 << 20


def peaks():
    """Roofline denominators: the machine's measured copy bandwidth and bf16 GEMM
    throughput; dense FP4 / INT8 = measured bf16 x the nominal ratio (4x / 2x)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return {"hbm_gbs": float(m["hbm_gbs"]), "bf16": float(m["bf16_tflops"]),
                "bf16_sustained": float(m["bf16_tflops_sustained"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture of `bench.py [--config ...] --steps 3 --warmup 3
# --no-cpu-baseline --no-extras` (the summaries under profiles/), keyed by
# kernel, workload and a fingerprint of the kernel's sources: a kernel changed
# since the capture reports null.  Part of what a kernel writes is still
# dirty in the 126 MB L2 when it ends (part of Y after a GEMM; at M = 4608 all
# of the activation kernel's outputs), so write traffic is below the bytes
# written.
# Vendor figures for one B200, for the fractions reported beside the measured
# denominators: dense FP4 and INT8 tensor peaks (NVIDIA's doubled figures are
# with 2:4 sparsity) and the HBM3e bandwidth.
DATASHEET_FP4_TFLOPS = 9000.0
DATASHEET_INT8_TOPS = 4500.0
NOMINAL_HBM_GBS = 8000.0
NCU_TRAFFIC = {
    ("gemm_nvfp4_pair_kernel", "c5_block/fc2", 16384, "nvfp4"): (222011392, "559ee5e39072da5f"),
    ("quant_act_kernel", "c5_block/fc2", 16384, "nvfp4"): (500727552, "07cf2606c82c7582"),
    ("gemm_int4_kernel", "c4_int4_lora/proj", 4608, "int4"): (21903616, "05e99fde6326be6b"),
    ("gemm_w8a8_kernel", "c2_qkv/qkv", 4608, "w8a8"): (93856256, "6fe3c9970eeb8a17"),
    ("gemm_nvfp4_pair_kernel", "c2_qkv/qkv", 4608, "nvfp4"): (63152896, "559ee5e39072da5f"),
    ("quant_act_kernel", "c2_qkv/qkv", 4608, "nvfp4"): (28758016, "07cf2606c82c7582"),
}
KERNEL_SOURCES = {
    "gemm_nvfp4_kernel": ("gemm_nvfp4.cuh", "svdq_ptx.cuh", "svdq_formats.cuh"),
    "gemm_nvfp4_pair_kernel": ("gemm_nvfp4_pair.cuh", "gemm_nvfp4.cuh", "svdq_ptx.cuh", "svdq_formats.cuh"),
    "quant_act_kernel": ("quant_act.cuh", "svdq_ptx.cuh", "svdq_formats.cuh"),
    "gemm_int4_kernel": ("gemm_int4.cuh", "gemm_nvfp4.cuh", "svdq_ptx.cuh", "svdq_formats.cuh"),
    "gemm_w8a8_kernel": ("gemm_w8a8.cuh", "gemm_nvfp4.cuh", "svdq_ptx.cuh", "svdq_formats.cuh"),
}


def kernel_fingerprint(kernel):
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "w4a4_gemm_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, workload, M, fmt):
    """Measured DRAM bytes per launch, or None if not captured for this
    workload and format or the kernel changed since."""
    entry = NCU_TRAFFIC.get((kernel, workload, M, fmt))
    if entry is None or kernel_fingerprint(kernel) != entry[1]:
        return None
    return entry[0]


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = max(mx, float(parts[2]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(nm)
        finally:
            os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# Per format: tensor-core instruction family (int8 formats run kind::i8, whose
# peak is half the FP4 one), activation code bytes per value, GEMM kernel.
INT8_KIND = ("int4", "w8a8")
GEMM_KERNEL = {"nvfp4": "gemm_nvfp4_pair_kernel", "fp4g32": "gemm_nvfp4_pair_kernel",
               "int4": "gemm_int4_kernel", "w8a8": "gemm_w8a8_kernel"}
DTYPE = {"nvfp4": "e2m1xe2m1+bf16 (fp32 acc)", "fp4g32": "e2m1xe2m1+bf16 (fp32 acc)",
         "int4": "s8xs8+bf16 (fp32 acc)", "w8a8": "s8xs8 (s32 acc)+bf16 (fp32 acc)"}


def layer_inputs(args):
    import dataclasses
    layer = args.layer
    if layer is None and args.config == "c5_block":
        layer = "fc2"      # the block's largest GEMM (K = 12288 -> N = 3072)
    spec = WL.layer_spec(args.config, layer)
    if getattr(args, "fmt", None):
        spec = dataclasses.replace(spec, fmt=args.fmt)
    if getattr(args, "rank", None) is not None:
        spec = dataclasses.replace(spec, rank=args.rank)
    M = args.M or WL.CONFIGS[args.config].Ms[-1 if args.config == "c5_block" else 0]
    return spec, M


# ----------------------------------------------------------------------------- ours
def max_over_ranks(values, world, device):
    """Element-wise maximum over all ranks (the slowest rank sets the time)."""
    if world <= 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(world, flops_per_rank_step, steps, seconds):
    """Whole-job TFLOP/s: every rank runs its own batch of the layer (weak
    scaling), so the work of all ranks over the slowest rank's time."""
    return world * flops_per_rank_step * steps / seconds / 1e12


def time_layer(S, w, X, ws, Y, M, flush, stream, steps, warmup, world, sampler=None):
    """Seconds per step, with the 126 MB L2 flushed before every step (outside
    the events), CUDA events on the launching stream:
      t_step: one event pair around the activation kernel and the GEMM, which
              the library launches back to back (the GEMM's setup overlaps the
              activation kernel's tail);
      t_q, t_g: a second pass with an event between the two kernels, which
              keeps them apart: each kernel's own time.
    The clock sampler, if given, runs over the t_step pass."""
    def run(split):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        for ev in evs:
            flush.zero_()
            ev[0].record(stream)
            S.svdq_quantize_act(w, X, ws)
            if split:
                ev[1].record(stream)
            S.svdq_linear(w, ws, M, Y)
            ev[2].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        return evs

    for _ in range(warmup):
        flush.zero_()
        S.svdq_quantize_act(w, X, ws)
        S.svdq_linear(w, ws, M, Y)
    torch.cuda.synchronize()
    if S.svdq_get_error():
        raise RuntimeError("device wait timed out during warm-up")
    if sampler:
        sampler.start()
    whole = run(False)
    clocks = sampler.stop() if sampler else None
    split = run(True)
    if S.svdq_get_error():
        raise RuntimeError("device wait timed out during timing")
    t_step = np.array([e[0].elapsed_time(e[2]) for e in whole]) * 1e-3   # s
    t_q = np.array([e[0].elapsed_time(e[1]) for e in split]) * 1e-3
    t_g = np.array([e[1].elapsed_time(e[2]) for e in split]) * 1e-3
    return t_step, t_q, t_g, clocks


def unfused_foil(S, w, w0, X, ws, Y, M, flush, stream, steps, warmup):
    """Seconds per step of the low-rank branch run unfused: the 4-bit layer at
    rank 0 (w0), then the smoothing pass X_hat = X / lambda, X_hat L1 and
    (X_hat L1) L2 as separate cuBLAS bf16 GEMMs and an addition into Y.  A
    comparison point for the fused kernels, not part of the product."""
    e = S.svdq_export_weights(w)
    dev = X.device
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    L1 = bf(e["L1"])                              # K x r
    L2 = bf(e["L2"])                              # r x N
    inv = torch.from_numpy(e["inv_lambda"]).to(dev).to(torch.bfloat16)

    def step():
        S.svdq_quantize_act(w0, X, ws)
        S.svdq_linear(w0, ws, M, Y)
        xh = X * inv                                # one bf16 pass over X
        Y.addmm_(torch.matmul(xh, L1), L2)          # Y += (X_hat L1) L2, one pass over Y

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    ts = []
    for _ in range(steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        ts.append((a, b))
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in ts])) * 1e-3


def vendor_gemm(M, K, N, flush, stream, steps, warmup):
    """Seconds per launch of cuBLAS's NVFP4 block-scaled GEMM (torch scaled_mm:
    E2M1 operands, an E4M3 scale per 16 values in the 128 x 4 swizzled layout,
    bf16 out) on random codes of the layer's M, K and N: a comparison point for
    the FP4 GEMM at rank 0 (no low-rank tail, no bias).  Not part of the
    product; None with the reason when this torch or shape cannot run it."""
    if M % 128 or (K // 16) % 4:
        return None, "needs M % 128 == 0 and K % 64 == 0"
    try:
        import torch.nn.functional as F
        from torch.nn.functional import ScalingType, SwizzleType
        dev = torch.device("cuda", torch.cuda.current_device())
        g = torch.Generator(device=dev)
        g.manual_seed(7)
        a = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g).view(torch.float4_e2m1fn_x2)
        b = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g).view(torch.float4_e2m1fn_x2)
        sa = (torch.rand(M, K // 16, device=dev, generator=g) * 1.5 + 0.25).to(torch.float8_e4m3fn)
        sb = (torch.rand(N, K // 16, device=dev, generator=g) * 1.5 + 0.25).to(torch.float8_e4m3fn)
        sw = SwizzleType.SWIZZLE_32_4_4

        def step():
            F.scaled_mm(a, b.t(), sa, ScalingType.BlockWise1x16, sb, ScalingType.BlockWise1x16,
                        swizzle_a=sw, swizzle_b=sw, output_dtype=torch.bfloat16)

        step()
        torch.cuda.synchronize()
    except Exception as e:   # an older torch or cuBLAS without NVFP4
        return None, str(e).splitlines()[0][:160]
    for _ in range(warmup):
        flush.zero_()
        step()
    ts = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        ts.append((e0, e1))
    torch.cuda.synchronize()
    return float(np.mean([x.elapsed_time(y) for x, y in ts])) * 1e-3, None


def e2e_pipelined(S, w, X, Y, ws, steps):
    """Seconds per step of the layer served end to end through svdq_forward:
    every step copies its X from pinned host memory to the device and its Y
    back, as a serving loop would, with the copies of neighbouring steps
    overlapping the compute on their own streams (double-buffered X and Y;
    copy engines run H2D and D2H at the same time).  Events on the three
    streams bracket the whole run."""
    dev = X.device
    M, N = Y.shape
    X_host = [X.cpu().pin_memory() for _ in range(2)]
    Y_host = [torch.empty(M, N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    X_dev = [torch.empty_like(X) for _ in range(2)]
    Y_dev = [Y, torch.empty_like(Y)]
    s_in, s_comp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev = lambda: torch.cuda.Event(enable_timing=False)

    def run(n):
        done_comp = [None, None]   # compute of the step that last used buffer b
        done_out = [None, None]    # D2H of the step that last used buffer b
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if done_comp[b] is not None:
                    s_in.wait_event(done_comp[b])          # X_dev[b] no longer read
                X_dev[b].copy_(X_host[b], non_blocking=True)
                e_in = ev()
                e_in.record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(e_in)
                if done_out[b] is not None:
                    s_comp.wait_event(done_out[b])         # Y_dev[b] copied out
                S.svdq_forward(w, X_dev[b], Y_dev[b], ws, stream=s_comp)
                done_comp[b] = ev()
                done_comp[b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_comp[b])
                Y_host[b].copy_(Y_dev[b], non_blocking=True)
                done_out[b] = ev()
                done_out[b].record(s_out)

    run(2)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    s_comp.wait_event(t0)
    s_out.wait_event(t0)
    run(steps)
    for s in (s_in, s_comp):
        e = ev()
        e.record(s)
        s_out.wait_event(e)
    t1.record(s_out)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) * 1e-3 / steps


def tensor_ceiling(S, fmt, stream):
    """The tensor cores' own ceiling for the GEMM's instruction (no global
    traffic): a ~5 ms burst and a ~1 s sustained run, in TFLOP/s."""
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    flop_step = sms * 4 * 2 * 128 * 256 * (32 if fmt in INT8_KIND else 64)

    def run(steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        S.svdq_tensor_peak(fmt, steps, stream)
        b.record(stream)
        torch.cuda.synchronize()
        if S.svdq_get_error():
            raise RuntimeError("device wait timed out in the tensor ceiling kernel")
        return a.elapsed_time(b) * 1e-3

    t = run(2000)
    steps_burst = max(2000, int(2000 * 0.005 / t))
    burst = max(flop_step * steps_burst / run(steps_burst) for _ in range(3)) / 1e12
    steps_long = max(2000, int(2000 * 1.0 / t))
    sustained = flop_step * steps_long / run(steps_long) / 1e12
    return {"burst": round(burst, 1), "sustained": round(sustained, 1), "unit": "TFLOP/s",
            "what": "tcgen05 " + ("kind::i8 128x256x32" if fmt in INT8_KIND else "kind::mxf4nvf4 128x256x64")
                    + " back to back from shared memory on every SM, no global loads"}


def run_ours(args):
    import w4a4_gemm_b200 as S

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    S.lib()
    spec, M = layer_inputs(args)
    K, N = spec.K, spec.N
    W, bias, A, B = WL.make_weights(spec)
    X = WL.make_activations(spec, M).to(dev)
    W = W.to(dev)
    xabs = S.svdq_calib_absmax(X)
    w = S.svdq_prepare_weights(W, spec.rank, spec.fmt, x_absmax=xabs,
                               bias=bias.to(dev) if bias is not None else None,
                               lora_A=A.to(dev) if A is not None else None,
                               lora_B=B.to(dev) if B is not None else None)
    ws = S.alloc_workspace(w, M, dev)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    # activation kernel + GEMM; FP4 formats zero the scale padding when K % 256,
    # W8A8 first computes the per-token scales
    launches_per_step = 2 + (1 if (spec.fmt in ("nvfp4", "fp4g32") and K % 256) else 0) \
        + (1 if spec.fmt == "w8a8" else 0)

    sampler = ClockSampler(local)
    t_step, t_q, t_g, clocks = time_layer(S, w, X, ws, Y, M, flush, stream, args.steps, args.warmup, world,
                                          sampler)
    total = float(t_step.sum())
    total, tq_mean, tg_mean = max_over_ranks([total, float(t_q.mean()), float(t_g.mean())], world, dev)

    # end to end through the public API: pinned host X in, host Y out, every step
    t_e2e = e2e_pipelined(S, w, X, Y, ws, max(3, min(args.steps, 10)))
    if S.svdq_get_error():
        raise RuntimeError("device wait timed out during timing")

    flops = 2.0 * M * K * N
    r = w.rank
    pk = peaks()
    fp_peak = pk["bf16"] * (2.0 if spec.fmt in INT8_KIND else 4.0)
    gemm_flops = flops + 2.0 * M * r * N
    achieved = gemm_flops / tg_mean / 1e12
    # activation kernel: algorithmic bytes (X read, codes + scales + XL1 written)
    code_bytes = M * K if spec.fmt in INT8_KIND else M * K / 2
    scale_bytes = {"nvfp4": M * K / 16, "fp4g32": M * K / 16, "int4": M * K / 64 * 2, "w8a8": M * 4}[spec.fmt]
    q_bytes = 2.0 * M * K + code_bytes + scale_bytes + 2.0 * M * w.rank_padded
    q_gbs = q_bytes / tq_mean / 1e9
    value = job_throughput(world, flops, args.steps, total)
    gemm_kernel = GEMM_KERNEL[spec.fmt]
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DTYPE[spec.fmt],
        "data": "synthetic (seeded FLUX-shaped activations and weights; no checkpoints)",
        "config": {"workload": f"{args.config}/{spec.name}: M={M} K={K} N={N} rank={r} {spec.fmt}",
                   "M": M, "K": K, "N": N, "rank": r, "format": spec.fmt,
                   "l2": "flushed between steps (512 MiB write)", "parallelism": f"dp{world} (token batches)"},
        "us_per_layer": round(total / args.steps * 1e6, 2),
        "us_quant": round(tq_mean * 1e6, 2), "us_gemm": round(tg_mean * 1e6, 2),
        "us_split_how": "us_quant, us_gemm: each kernel alone (a second pass with an event between them); "
                        "us_layer, ms_per_step: both kernels under one event pair",
        "pct_fp4_peak_layer": round(100.0 * flops / (total / args.steps) / 1e12 / fp_peak, 2),
        "roofline": {"bound": "tensor", "kernel": gemm_kernel,
                     "achieved": round(achieved, 1), "peak": round(fp_peak, 1), "unit": "TFLOP/s",
                     "frac": round(achieved / fp_peak, 4),
                     "traffic": ncu_traffic(gemm_kernel, f"{args.config}/{spec.name}", M, spec.fmt),
                     "peak_note": f"{pk['source']}: bf16 {pk['bf16']} TF/s x {'2 (INT8)' if spec.fmt in INT8_KIND else '4 (FP4)'}",
                     "datasheet_peak": DATASHEET_INT8_TOPS if spec.fmt in INT8_KIND else DATASHEET_FP4_TFLOPS,
                     "frac_of_datasheet": round(achieved / (DATASHEET_INT8_TOPS if spec.fmt in INT8_KIND
                                                            else DATASHEET_FP4_TFLOPS), 4)},
        "roofline_quant": {"bound": "hbm", "kernel": "quant_act_kernel", "achieved": round(q_gbs, 1),
                           "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(q_gbs / pk["hbm_gbs"], 4),
                           "nominal_peak": NOMINAL_HBM_GBS, "frac_of_nominal": round(q_gbs / NOMINAL_HBM_GBS, 4),
                           "algorithmic_bytes": int(q_bytes),
                           "traffic": ncu_traffic("quant_act_kernel", f"{args.config}/{spec.name}", M, spec.fmt)},
        "e2e": {"value": round(flops / t_e2e / 1e12, 3), "unit": UNIT,
                "h2d_bytes_per_step": int(X.numel() * 2), "d2h_bytes_per_step": int(Y.numel() * 2),
                "how": "svdq_forward per step with its X copied in from pinned host memory and its Y copied "
                       "out; copy-in, compute and copy-out on three streams, neighbouring steps overlapping"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_extras:
        # the same layer without the low-rank branch (plain W4A4, same smoothing)
        w0 = S.svdq_prepare_weights(W, 0, spec.fmt, x_absmax=xabs,
                                    bias=bias.to(dev) if bias is not None else None)
        s0, q0, g0, _ = time_layer(S, w0, X, ws, Y, M, flush, stream, args.steps, args.warmup, world)
        t_unf = unfused_foil(S, w, w0, X, ws, Y, M, flush, stream, args.steps, args.warmup) if r else None
        w0.close()
        l0 = float(s0.mean())
        line["lowrank_overhead"] = {
            "us_layer_r0": round(l0 * 1e6, 2), "us_quant_r0": round(float(q0.mean()) * 1e6, 2),
            "us_gemm_r0": round(float(g0.mean()) * 1e6, 2),
            "layer": round(total / args.steps / l0 - 1.0, 4),
            "gemm": round(tg_mean / float(g0.mean()) - 1.0, 4), "target": 0.15,
            "what": f"us(rank {r}) / us(rank 0) - 1, same format, shapes, smoothing and bias"}
        if t_unf is not None:
            line["lowrank_overhead"]["unfused_foil"] = {
                "us_layer": round(t_unf * 1e6, 2), "layer": round(t_unf / l0 - 1.0, 4),
                "what": "rank-0 layer, then smoothing, X_hat L1 and (X_hat L1) L2 as separate cuBLAS bf16 "
                        "GEMMs and an addition into Y (the unfused design the fused kernels replace)"}
        if spec.fmt == "nvfp4":
            t_v, why = vendor_gemm(M, spec.K, spec.N, flush, stream, args.steps, args.warmup)
            if t_v is None:
                line["vendor_gemm"] = {"unavailable": why}
            else:
                line["vendor_gemm"] = {
                    "us": round(t_v * 1e6, 2), "tflops": round(2.0 * M * spec.K * spec.N / t_v / 1e12, 1),
                    "ours_rank0_us": round(float(g0.mean()) * 1e6, 2),
                    "ours_over_vendor_time": round(float(g0.mean()) / t_v, 4),
                    "what": "cuBLAS NVFP4 block-scaled GEMM (torch scaled_mm, BlockWise1x16, swizzled E4M3 "
                            "scales) on random codes of the same M, K, N, against our FP4 GEMM at rank 0"}
        if args.rank_sweep:
            sweep = []
            for rr in args.rank_sweep:
                wr = S.svdq_prepare_weights(W, rr, spec.fmt, x_absmax=xabs,
                                            bias=bias.to(dev) if bias is not None else None)
                wsr = S.alloc_workspace(wr, M, dev)   # X_hat L1 grows with the rank
                sr, qr, gr, _ = time_layer(S, wr, X, wsr, Y, M, flush, stream, args.steps, args.warmup, world)
                del wsr
                wr.close()
                lr = float(sr.mean())
                sweep.append({"rank": rr, "us_layer": round(lr * 1e6, 2), "us_quant": round(float(qr.mean()) * 1e6, 2),
                              "us_gemm": round(float(gr.mean()) * 1e6, 2), "overhead": round(lr / l0 - 1.0, 4)})
            line["rank_sweep"] = sweep
        ceil = tensor_ceiling(S, spec.fmt, stream)
        ceil["gemm_frac_of_burst"] = round(achieved / ceil["burst"], 4)
        ceil["gemm_frac_of_sustained"] = round(achieved / ceil["sustained"], 4)
        line["tensor_ceiling"] = ceil
    del W
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(spec, M, args.cpu_rows)
    if rank == 0:
        print(json.dumps(line), flush=True)
    w.close()
    if world > 1:
        torch.distributed.destroy_process_group()


# ----------------------------------------------------------------------------- oracle
def _oracle_setup(spec, M, rows):
    import oracle as O
    W, bias, A, B = WL.make_weights(spec)
    X = WL.make_activations(spec, M)
    Xb = WL.bf16_bits(X)
    xm = O.calib_absmax(Xb)
    # the top-r factors from the Gram matrix (the same subspace as a full SVD,
    # which takes minutes at FLUX sizes); preparation is not timed
    prep = O.prepare(WL.bf16_bits(W), xm, spec.rank,
                     WL.bf16_bits(A) if A is not None else None,
                     WL.bf16_bits(B) if B is not None else None, svd="gram")
    wq = O.weight_quant(spec.fmt, prep["R"])
    sample = np.ascontiguousarray(Xb[:rows])
    return O, prep, wq, sample, (WL.bf16_bits(bias) if bias is not None else None)


def _oracle_step(O, spec, prep, wq, sample, bias):
    act = O.act_quant(spec.fmt, sample, prep["inv_lambda"], prep["L1"] if prep["rank"] else None)
    O.linear(spec.fmt, act, wq, prep["L2"] if prep["rank"] else None, bias, spec.N)


def run_block(args):
    """--layer all: the workload's layers back to back as one step (one DiT
    block's four linears at M tokens, each on its own seeded input), under one
    event pair with the L2 flushed before every step.  The activation kernel of
    each layer is launched while the previous GEMM drains (programmatic
    dependent launch).  Reports the block and each layer's share."""
    import w4a4_gemm_b200 as S

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    S.lib()
    cfg = WL.CONFIGS[args.config]
    M = args.M or cfg.Ms[-1]
    layers = []
    for spec in cfg.layers:
        W, bias, A, B = WL.make_weights(spec)
        X = WL.make_activations(spec, M).to(dev)
        w = S.svdq_prepare_weights(W.to(dev), spec.rank, spec.fmt, x_absmax=S.svdq_calib_absmax(X),
                                   bias=bias.to(dev) if bias is not None else None)
        layers.append((spec, w, X, S.alloc_workspace(w, M, dev),
                       torch.empty(M, spec.N, dtype=torch.bfloat16, device=dev)))
        del W
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def block(evs=None, split=False):
        for i, (spec, w, X, ws, Y) in enumerate(layers):
            if evs is not None and (split or i == 0):
                evs[i].record(stream)
            S.svdq_quantize_act(w, X, ws)
            S.svdq_linear(w, ws, M, Y)
        if evs is not None:
            evs[-1].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        block()
    torch.cuda.synchronize()
    if S.svdq_get_error():
        raise RuntimeError("device wait timed out during warm-up")
    n = len(layers)

    def run(split):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n + 1)] for _ in range(args.steps)]
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        for e in evs:
            flush.zero_()
            block(e, split)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        return evs

    # the block under one event pair (the layers' kernels overlap at their
    # boundaries), then a second pass with an event before every layer
    sampler = ClockSampler(local)
    sampler.start()
    whole = run(False)
    clocks = sampler.stop()
    split = run(True)
    if S.svdq_get_error():
        raise RuntimeError("device wait timed out during timing")
    t_block = np.array([e[0].elapsed_time(e[n]) for e in whole]) * 1e-3
    t_layer = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(n)] for e in split]).mean(axis=0) * 1e-3
    flops = sum(2.0 * M * spec.K * spec.N for spec, *_ in layers)
    total = float(t_block.sum())
    (total,) = max_over_ranks([total], world, dev)
    pk = peaks()
    line = {
        "metric": METRIC, "value": round(job_throughput(world, flops, args.steps, total), 2), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": DTYPE[layers[0][0].fmt],
        "data": "synthetic (seeded FLUX-shaped activations and weights; no checkpoints)",
        "config": {"workload": f"{args.config}: one block ({', '.join(s.name for s, *_ in layers)}) at M={M}",
                   "M": M, "layers": [{"name": s.name, "K": s.K, "N": s.N, "rank": s.rank} for s, *_ in layers],
                   "l2": "flushed between steps (512 MiB write)", "parallelism": f"dp{world} (token batches)"},
        "us_per_block": round(total / args.steps * 1e6, 2),
        "us_per_layer_in_block": {s.name: round(float(t) * 1e6, 2) for (s, *_), t in zip(layers, t_layer)},
        "us_split_how": "us_per_block: the block under one event pair; us_per_layer_in_block: a second pass "
                        "with an event before every layer",
        "pct_fp4_peak_block": round(100.0 * flops / (total / args.steps) / 1e12 / (pk["bf16"] * 4.0), 2),
        "gpu_launches": 2 * n * args.steps,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    for _, w, *_ in layers:
        w.close()
    if world > 1:
        torch.distributed.destroy_process_group()


def cpu_rows(spec, M, rows):
    """Rows of the oracle's timed sample: as given, else about 4 GFLOP of the
    layer (2 K N per row), at least 8 and at most M."""
    if rows is None:
        rows = max(8, int(4e9 // (2.0 * spec.K * spec.N)))
    return max(1, min(M, rows))


def cpu_baseline(spec, M, rows):
    rows = cpu_rows(spec, M, rows)
    O, prep, wq, sample, bias = _oracle_setup(spec, M, rows)
    t0 = time.perf_counter()
    _oracle_step(O, spec, prep, wq, sample, bias)
    dt = time.perf_counter() - t0
    cores = len(os.sched_getaffinity(0))
    return {"value": round(2.0 * rows * spec.K * spec.N / dt / 1e12, 6), "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"first {rows} of {M} token rows (quantize + GEMM + low-rank + bias, all N); "
                      f"OpenMP over rows; weight preparation untimed"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    spec, M = layer_inputs(args)
    rows = cpu_rows(spec, M, args.cpu_rows)
    O, prep, wq, sample, bias = _oracle_setup(spec, M, rows)
    for _ in range(args.warmup):
        _oracle_step(O, spec, prep, wq, sample, bias)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(O, spec, prep, wq, sample, bias)
    dt = (time.perf_counter() - t0) / args.steps
    value = 2.0 * rows * spec.K * spec.N / dt / 1e12
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32 (CPU oracle)",
        "data": "synthetic (seeded FLUX-shaped activations and weights; no checkpoints)",
        "config": {"workload": f"{args.config}/{spec.name}: M={M} K={spec.K} N={spec.N} rank={spec.rank} {spec.fmt}",
                   "sample_rows": rows},
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"first {rows} of {M} token rows per step"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="c5_block", choices=sorted(WL.CONFIGS))
    ap.add_argument("--layer", default=None,
                    help="a layer of the config, or 'all': the config's layers back to back as one step")
    ap.add_argument("--M", type=int, default=None)
    ap.add_argument("--fmt", choices=["nvfp4", "int4", "fp4g32", "w8a8"], default=None,
                    help="override the workload's format")
    ap.add_argument("--rank", type=int, default=None,
                    help="override the workload's low-rank branch rank (the paper pairs W8A8 with 16)")
    ap.add_argument("--cpu-rows", type=int, default=None,
                    help="token rows of the oracle's sample (default: about 4 GFLOP of the layer, >= 8 rows)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rank-sweep", type=lambda v: [int(x) for x in v.split(",")], default=None,
                    help="also time the layer at these ranks, e.g. 16,32,48,64")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the rank-0 comparison and the tensor-ceiling measurement")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.layer == "all":
        run_block(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
