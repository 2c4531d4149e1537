#!/usr/bin/env python3
"""Benchmark: block-scaled FP4 quantization throughput on B200.

Metric: GB/s = (algorithmic bytes in + out) / kernel time, and % of the
measured HBM copy bandwidth.  One "step" is one pass of the whole hot path
over the benchmark workloads (each kernel with the tensor amax already on the
device, as with delayed scaling or a fused producer):

  activation 8192x4096 BF16   NVFP4 1x16 row + col from one read
  activation 8192x4096 BF16   MXFP4 1x32 row + col
  weight    14336x4096 FP32   NVFP4 16x16 2D, W and W^T codes
  gradient   8192x5120 BF16   RHT-16 / RHT-128 + NVFP4 of dY^T, SR and RNE
  if4       16384x8192 BF16   IF4 quantize, and IF4 -> BF16 dequantize

Each kernel is timed with CUDA events on the launching stream; the L2 is
flushed before every kernel, outside the timed events: a 256 MiB buffer is
written and then read back, so the kernel starts with none of its own data
in L2 and without the flush's dirty lines still waiting to be written back
(which would charge the flush's DRAM writes to the kernel).  A short
device-side sleep before each flush keeps the GPU busy while the host
enqueues the flush, the start event and the kernel, so the events bracket the
kernel itself rather than the host's launch latency (which the e2e figure
includes).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (torchrun): every rank runs the suite on its own tensors (the work
shards into independent tensors; no collective on the data path), the step
time is the max over ranks and ``value`` is all ranks' bytes over that time.
``--impl reference`` times the CPU oracle on a bounded sample instead (rank 0
only).  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "quantize throughput GB/s (bytes in+out) and % of B200 HBM peak per config"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20
# the workload both arms name in their "config"
SUITE_WORKLOAD = ("fp4 quantization suite: activation 8192x4096 nvfp4 row+col and mxfp4 "
                  "row+col; weight 14336x4096 fp32 2d16x16; gradient 8192x5120 rht16/rht128 x "
                  "sr/rne; if4 16384x8192 quant + bf16 dequant")
LEAD_SLEEP_CYCLES = 200_000  # ~0.1 ms at 1.965 GHz, untimed
FIRST_LEAD_CYCLES = 4_000_000  # ~2 ms, untimed, before the first timed job


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# jobs: one kernel launch each, with its algorithmic byte count
# ---------------------------------------------------------------------------

class Job:
    def __init__(self, name, src, bytes_moved, launches, run, e2e=None, oracle=None,
                 run_amax=None):
        self.name = name            # workload / variant
        self.src = src              # CUDA source file of the kernel
        self.bytes = bytes_moved    # algorithmic bytes (input once + outputs)
        self.launches = launches    # our kernels per call
        self.run = run              # device call (inputs resident, tensor amax given)
        self.e2e = e2e              # E2E: host inputs -> public API -> host outputs
        self.oracle = oracle        # CPU oracle on a row fraction: returns bytes done
        self.run_amax = run_amax    # the same call computing the tensor amax first


class E2E:
    """One job end to end: pinned host inputs are copied into the job's own
    device buffers, the public API call runs on them (computing the tensor
    amax itself), and every output is copied back to pinned host memory.
    The three steps run on three streams so that the copies of neighbouring
    jobs overlap (host-to-device and device-to-host run at the same time);
    events order each job's steps and keep a buffer from being refilled
    while an earlier step still uses it."""

    def __init__(self, host_in, dev_in, compute, dev_out):
        import torch
        self.host_in, self.dev_in, self.compute_fn = host_in, dev_in, compute
        self.dev_out = dev_out
        self.host_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                         for k, v in dev_out.items()}
        self.h2d_bytes = sum(t.numel() * t.element_size() for t in host_in)
        self.d2h_bytes = sum(t.numel() * t.element_size() for t in dev_out.values())
        self.ev_in = torch.cuda.Event()      # inputs on the device
        self.ev_comp = torch.cuda.Event()    # outputs written, inputs free
        self.ev_out = torch.cuda.Event()     # outputs copied out

    def step(self, s_in, s_comp, s_out, first):
        import torch
        with torch.cuda.stream(s_in):
            if not first:
                s_in.wait_event(self.ev_comp)          # the last call has read the inputs
            for h, d in zip(self.host_in, self.dev_in):
                d.copy_(h, non_blocking=True)
            self.ev_in.record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(self.ev_in)
            if not first:
                s_comp.wait_event(self.ev_out)         # the last outputs are out
            self.compute_fn()
            self.ev_comp.record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(self.ev_comp)
            for k, v in self.dev_out.items():
                self.host_out[k].copy_(v, non_blocking=True)
            self.ev_out.record(s_out)
        return self.h2d_bytes, self.d2h_bytes


def build_jobs(device, fq, inputs):
    """The benchmark suite on `device`.  Inputs and outputs are allocated once."""
    import torch

    jobs = []
    SW = fq.SCALE_SWIZZLED

    def pinned_like(t):
        return torch.empty(t.shape, dtype=t.dtype, pin_memory=True)

    def dev_like(t):
        return torch.empty(t.shape, dtype=t.dtype, device=device)

    # ---- activation: NVFP4 row + col, MXFP4 row + col -------------------
    xa_cpu = inputs["activation"]
    xa = xa_cpu.to(device)
    amax_a = fq.fp4q_amax(xa)
    out_nv = fq.fp4q_quantize_nvfp4(xa, layouts=3, amax=amax_a, scale_layout=SW)
    out_mx = fq.fp4q_quantize_mxfp4(xa, layouts=3, scale_layout=SW)
    R, C = xa.shape
    nb_nv = R * C * 2 + 2 * (R * C // 2) + 2 * (R * C // 16) + 4
    nb_mx = R * C * 2 + 2 * (R * C // 2) + 2 * (R * C // 32)
    xa_h = pinned_like(xa_cpu).copy_(xa_cpu)
    xe_nv, xe_mx = dev_like(xa), dev_like(xa)
    oe_nv = {k: dev_like(v) for k, v in out_nv.items()}
    oe_mx = {k: dev_like(v) for k, v in out_mx.items()}
    e2e_nv = E2E([xa_h], [xe_nv], lambda: fq.fp4q_quantize_nvfp4(
        xe_nv, layouts=3, scale_layout=SW, out=oe_nv), oe_nv)
    e2e_mx = E2E([xa_h], [xe_mx], lambda: fq.fp4q_quantize_mxfp4(
        xe_mx, layouts=3, scale_layout=SW, out=oe_mx), oe_mx)

    jobs.append(Job("activation 8192x4096 bf16 nvfp4 row+col", "nvfp4.cu", nb_nv, 1,
                    lambda: fq.fp4q_quantize_nvfp4(xa, layouts=3, amax=amax_a, scale_layout=SW,
                                                   out=out_nv), e2e_nv,
                    run_amax=lambda: fq.fp4q_quantize_nvfp4(xa, layouts=3, scale_layout=SW,
                                                            out=out_nv)))
    jobs.append(Job("activation 8192x4096 bf16 mxfp4 row+col", "nvfp4.cu", nb_mx, 1,
                    lambda: fq.fp4q_quantize_mxfp4(xa, layouts=3, scale_layout=SW, out=out_mx),
                    e2e_mx))

    # ---- weight: 2D 16x16 ------------------------------------------------
    w_cpu = inputs["weight"]
    w = w_cpu.to(device)
    amax_w = fq.fp4q_amax(w)
    out_w = fq.fp4q_quantize_2d(w, amax=amax_w)
    R, C = w.shape
    nb_w = R * C * 4 + 2 * (R * C // 2) + (R // 16) * (C // 16) + 4
    w_h = pinned_like(w_cpu).copy_(w_cpu)
    we = dev_like(w)
    oe_w = {k: dev_like(v) for k, v in out_w.items()}
    e2e_w = E2E([w_h], [we], lambda: fq.fp4q_quantize_2d(we, out=oe_w), oe_w)

    jobs.append(Job("weight 14336x4096 fp32 2d16x16 w+wt", "quant2d.cu", nb_w, 1,
                    lambda: fq.fp4q_quantize_2d(w, amax=amax_w, out=out_w), e2e_w,
                    run_amax=lambda: fq.fp4q_quantize_2d(w, out=out_w)))

    # ---- gradient: RHT + NVFP4 of dY^T ----------------------------------
    g_cpu = inputs["gradient"]
    g = g_cpu.to(device)
    T, C = g.shape
    nb_g = T * C * 2 + (T * C // 2) + (T * C // 16) + 4
    g_h = pinned_like(g_cpu).copy_(g_cpu)
    for n in (16, 128):
        amax_g = fq.fp4q_rht_amax(g, n, seed=0)
        for rnd, rname in ((fq.SR, "sr"), (fq.RNE, "rne")):
            out_g = fq.fp4q_quantize_rht_sr(g, n, round=rnd, seed=0, amax_rht=amax_g,
                                            scale_layout=SW)
            ge = dev_like(g)
            oe_g = {k: dev_like(v) for k, v in out_g.items()}
            e2e_g = E2E([g_h], [ge], lambda n=n, rnd=rnd, ge=ge, oe_g=oe_g: fq.fp4q_quantize_rht_sr(
                ge, n, round=rnd, seed=0, scale_layout=SW, out=oe_g), oe_g)

            jobs.append(Job(f"gradient 8192x5120 bf16 rht{n}+{rname}", "rht.cu", nb_g, 1,
                            lambda n=n, rnd=rnd, a=amax_g, o=out_g: fq.fp4q_quantize_rht_sr(
                                g, n, round=rnd, seed=0, amax_rht=a, scale_layout=SW, out=o),
                            e2e_g,
                            run_amax=lambda n=n, rnd=rnd, o=out_g: fq.fp4q_quantize_rht_sr(
                                g, n, round=rnd, seed=0, scale_layout=SW, out=o)))

    # ---- IF4: quantize and dequantize -----------------------------------
    x5_cpu = inputs["if4"]
    x5 = x5_cpu.to(device)
    amax5 = fq.fp4q_amax(x5)
    out5 = fq.fp4q_quantize_if4(x5, amax=amax5, scale_layout=SW)
    R, C = x5.shape
    nb_q5 = R * C * 2 + R * C // 2 + R * C // 16 + 4
    # the dequant reads its own copy of the codes so it never sees them in L2
    q5 = out5["q"].clone()
    sf5 = out5["sf"].clone()
    s5 = out5["s_dec"].clone()
    y5 = torch.empty((R, C), dtype=torch.bfloat16, device=device)
    nb_d5 = R * C // 2 + R * C // 16 + 4 + R * C * 2
    x5_h = pinned_like(x5_cpu).copy_(x5_cpu)
    x5e = dev_like(x5)
    oe5 = {k: dev_like(v) for k, v in out5.items()}
    e2e_q5 = E2E([x5_h], [x5e], lambda: fq.fp4q_quantize_if4(x5e, scale_layout=SW, out=oe5), oe5)
    q5_h, sf5_h, s5_h = q5.cpu().pin_memory(), sf5.cpu().pin_memory(), s5.cpu().pin_memory()
    q5e, sf5e, s5e, y5e = dev_like(q5), dev_like(sf5), dev_like(s5), dev_like(y5)
    e2e_d5 = E2E([q5_h, sf5_h, s5_h], [q5e, sf5e, s5e], lambda: fq.fp4q_dequantize(
        fq.FMT_IF4, q5e, sf5e, R, C, tensor_scale=s5e, scale_layout=SW, out=y5e), {"y": y5e})

    jobs.append(Job("if4 16384x8192 bf16 quantize", "if4.cu", nb_q5, 1,
                    lambda: fq.fp4q_quantize_if4(x5, amax=amax5, scale_layout=SW, out=out5),
                    e2e_q5,
                    run_amax=lambda: fq.fp4q_quantize_if4(x5, scale_layout=SW, out=out5)))
    jobs.append(Job("if4 16384x8192 dequantize to bf16", "dequant.cu", nb_d5, 1,
                    lambda: fq.fp4q_dequantize(fq.FMT_IF4, q5, sf5, R, C, tensor_scale=s5,
                                               scale_layout=SW, out=y5), e2e_d5))
    torch.cuda.synchronize(device)
    return jobs


def time_consumer_gemm(fq, device, stream, args, M=8192, N=8192, K=8192):
    """NVFP4 GEMM X W^T on operands this library quantized with swizzled
    scales, by this library's tensor-core GEMM (fp4q_gemm_nvfp4) and by the
    vendor's block-scaled GEMM (torch.nn.functional.scaled_mm): TFLOP/s
    against the FP4 peak (the measured BF16 peak x 4, the nominal FP4 / BF16
    ratio).  The vendor entry says "unavailable" where the installed library
    has no such GEMM."""
    import torch
    import torch.nn.functional as F
    g = torch.Generator().manual_seed(5)
    x = torch.randn(M, K, generator=g).to(torch.bfloat16).to(device)
    w = (torch.randn(N, K, generator=g) * 0.05).to(torch.bfloat16).to(device)
    sw = fq.SCALE_SWIZZLED
    ox = fq.fp4q_quantize_nvfp4(x, layouts=fq.ROWWISE, scale_layout=sw)
    ow = fq.fp4q_quantize_nvfp4(w, layouts=fq.ROWWISE, scale_layout=sw)
    del x, w
    try:
        bf16 = float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"])
        peak, kind = 4.0 * bf16, "measured bf16 x 4"
    except Exception:
        peak, kind = 4.0 * 1590.0, "fallback bf16 x 4"

    def timed(run):
        for _ in range(max(3, args.warmup)):
            run()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = max(5, args.steps)
        e0.record(stream)
        for _ in range(reps):
            run()
        e1.record(stream)
        torch.cuda.synchronize(device)
        s = e0.elapsed_time(e1) * 1e-3 / reps
        tflops = 2.0 * M * N * K / s / 1e12
        return {"us": round(s * 1e6, 1), "tflops": round(tflops, 1), "frac": round(tflops / peak, 4)}

    out = {"shape": [M, N, K], "format": "nvfp4 1x16, swizzled scales from fp4q, bf16 out",
           "peak_tflops": round(peak, 1), "peak_kind": kind,
           "note": "back-to-back launches; the 64 MB of codes may stay in the 126 MB L2"}
    c = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    out["fp4q"] = timed(lambda: fq.fp4q_gemm_nvfp4(
        ox["q_row"], ox["sf_row"], ow["q_row"], ow["sf_row"], K, tensor_scale_a=ox["s_dec"],
        tensor_scale_b=ow["s_dec"], out=c))
    out["fp4q"]["kernel"] = ("gemm_nvfp4_kernel (tcgen05.mma kind::mxf4nvf4, persistent, "
                             "128x256 tiles)")
    # the same product with an IF4 activation operand (split pass + one two-accumulator GEMM)
    g5 = torch.Generator().manual_seed(6)
    xi = torch.randn(M, K, generator=g5).to(torch.bfloat16).to(device)
    oi = fq.fp4q_quantize_if4(xi, scale_layout=sw)
    del xi
    ci = torch.empty((M, N), dtype=torch.float32, device=device)
    wsi = torch.empty(int(fq.lib().fp4q_gemm_if4_workspace_bytes(M, K)), dtype=torch.uint8,
                      device=device)
    out["fp4q_if4"] = timed(lambda: fq.fp4q_gemm_if4_nvfp4(
        oi["q"], oi["sf"], ow["q_row"], ow["sf_row"], K, tensor_scale_a=oi["s_dec"],
        tensor_scale_b=ow["s_dec"], out=ci, workspace=wsi))
    out["fp4q_if4"]["kernel"] = ("if4_split_kernel + gemm_nvfp4_kernel with three A operands "
                                 "and two accumulators (IF4 x NVFP4, FP32 out)")
    del wsi, ci
    A = ox["q_row"].view(torch.float4_e2m1fn_x2)
    B = ow["q_row"].view(torch.float4_e2m1fn_x2).t()
    sa, sb = ox["sf_row"].view(torch.float8_e4m3fn), ow["sf_row"].view(torch.float8_e4m3fn)
    try:
        out["vendor"] = timed(lambda: F.scaled_mm(
            A, B, sa, F.ScalingType.BlockWise1x16, sb, F.ScalingType.BlockWise1x16,
            swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
            output_dtype=torch.bfloat16))
    except Exception as e:  # the installed library has no block-scaled FP4 GEMM
        out["vendor"] = {"unavailable": str(e)[:200]}
    return out


def build_extra_jobs(device, fq, inputs):
    """Calls outside the headline suite, timed like it but reported apart from
    its value: the fused backward call and the row-wise operand alone on the
    gradient workload, and the IF4 explainer's comparison formats
    (four-over-six on the activation workload, NVINT4 on the IF4 workload),
    the tensor amax of the activation workload (which the suite takes as given),
    IF6 and IF3 on the IF4 workload and MXFP6 E2M3 on the activation workload."""
    import torch
    SW = fq.SCALE_SWIZZLED
    xa = inputs["activation"].to(device)
    amax_a = fq.fp4q_amax(xa)
    o46 = fq.fp4q_quantize_four_over_six(xa, layouts=3, amax=amax_a, scale_layout=SW)
    R, C = xa.shape
    nb46 = R * C * 2 + 2 * (R * C // 2) + 2 * (R * C // 16) + 4
    x5 = inputs["if4"].to(device)
    amax5 = fq.fp4q_amax(x5)
    oi4 = fq.fp4q_quantize_nvint4(x5, amax=amax5, scale_layout=SW)
    R5, C5 = x5.shape
    nbi4 = R5 * C5 * 2 + R5 * C5 // 2 + R5 * C5 // 16 + 4
    # the fused backward call on the gradient workload, and the row-wise
    # operand alone (the column-wise operand alone is in the suite)
    g = inputs["gradient"].to(device)
    T, Cg = g.shape
    amax_g = fq.fp4q_amax(g)
    amax_r16 = fq.fp4q_rht_amax(g, 16, seed=0)
    obw = fq.fp4q_quantize_backward(g, 16, round=fq.SR, seed_row=1, seed_col=0, amax_row=amax_g,
                                    amax_rht=amax_r16, scale_layout=SW)
    orow = fq.fp4q_quantize_nvfp4(g, layouts=fq.ROWWISE, round=fq.SR, seed=1, amax=amax_g,
                                  scale_layout=SW)
    obw_n = fq.fp4q_quantize_backward(g, 16, round=fq.RNE, amax_row=amax_g, amax_rht=amax_r16,
                                      scale_layout=SW)
    orow_n = fq.fp4q_quantize_nvfp4(g, layouts=fq.ROWWISE, amax=amax_g, scale_layout=SW)
    nb_row = T * Cg * 2 + T * Cg // 2 + T * Cg // 16 + 4
    nb_bw = T * Cg * 2 + 2 * (T * Cg // 2 + T * Cg // 16 + 4)
    # IF6 of the IF4 workload: 2 bytes in, 0.75 + 1/16 out
    oi6 = fq.fp4q_quantize_if6(x5, amax=amax5, scale_layout=SW)
    nbi6 = R5 * C5 * 2 + R5 * C5 * 3 // 4 + R5 * C5 // 16 + 4
    # IF3 of the IF4 workload: 2 bytes in, 0.375 + 1/16 out
    oi3 = fq.fp4q_quantize_if3(x5, amax=amax5, scale_layout=SW)
    nbi3 = R5 * C5 * 2 + R5 * C5 * 3 // 8 + R5 * C5 // 16 + 4
    # MXFP6 (E2M3) of the activation workload: 2 bytes in, 0.75 + 1/32 out
    o6 = fq.fp4q_quantize_mxfp6(xa, fq.FP6_E2M3, scale_layout=SW)
    nb6 = R * C * 2 + R * C * 3 // 4 + R * C // 32
    # the small parity workload: NVFP4 1x16 of a 256x256 BF16 matrix (codes,
    # scales, s_dec) and its FP32 dequantization; launch-latency bound
    xs = inputs["small"].to(device)
    amax_s = fq.fp4q_amax(xs)
    osm = fq.fp4q_quantize_nvfp4(xs, layouts=fq.ROWWISE, amax=amax_s)
    ysm = torch.empty((256, 256), dtype=torch.float32, device=device)
    nb_sq = 256 * 256 * 2 + 256 * 128 + 256 * 16 + 4
    nb_sd = 256 * 128 + 256 * 16 + 4 + 256 * 256 * 4
    torch.cuda.synchronize(device)
    return [
        Job("small 256x256 bf16 nvfp4 quantize (row-wise, rne)", "nvfp4.cu", nb_sq, 1,
            lambda: fq.fp4q_quantize_nvfp4(xs, layouts=fq.ROWWISE, amax=amax_s, out=osm),
            run_amax=lambda: fq.fp4q_quantize_nvfp4(xs, layouts=fq.ROWWISE, out=osm)),
        Job("small 256x256 nvfp4 dequantize to fp32", "dequant.cu", nb_sd, 1,
            lambda: fq.fp4q_dequantize(fq.FMT_NVFP4, osm["q_row"], osm["sf_row"], 256, 256,
                                       tensor_scale=osm["s_dec"], out=ysm)),
        Job("gradient 8192x5120 bf16 backward: row-wise sr + rht16+sr from one read", "rht.cu",
            nb_bw, 1, lambda: fq.fp4q_quantize_backward(
                g, 16, round=fq.SR, seed_row=1, seed_col=0, amax_row=amax_g, amax_rht=amax_r16,
                scale_layout=SW, out=obw)),
        Job("gradient 8192x5120 bf16 row-wise nvfp4 sr", "nvfp4.cu", nb_row, 1,
            lambda: fq.fp4q_quantize_nvfp4(g, layouts=fq.ROWWISE, round=fq.SR, seed=1,
                                           amax=amax_g, scale_layout=SW, out=orow)),
        Job("gradient 8192x5120 bf16 backward: row-wise rne + rht16+rne from one read", "rht.cu",
            nb_bw, 1, lambda: fq.fp4q_quantize_backward(
                g, 16, round=fq.RNE, amax_row=amax_g, amax_rht=amax_r16, scale_layout=SW,
                out=obw_n)),
        Job("gradient 8192x5120 bf16 row-wise nvfp4 rne", "nvfp4.cu", nb_row, 1,
            lambda: fq.fp4q_quantize_nvfp4(g, layouts=fq.ROWWISE, amax=amax_g, scale_layout=SW,
                                           out=orow_n)),
        Job("activation 8192x4096 bf16 four-over-six row+col", "nvfp4.cu", nb46, 1,
            lambda: fq.fp4q_quantize_four_over_six(xa, layouts=3, amax=amax_a, scale_layout=SW,
                                                   out=o46)),
        Job("if4 16384x8192 bf16 nvint4", "if4.cu", nbi4, 1,
            lambda: fq.fp4q_quantize_nvint4(x5, amax=amax5, scale_layout=SW, out=oi4)),
        Job("activation 8192x4096 bf16 tensor amax", "amax.cu", R * C * 2 + 4, 1,
            lambda: fq.fp4q_amax(xa, out=amax_a)),
        Job("if4 16384x8192 bf16 if6", "if6.cu", nbi6, 1,
            lambda: fq.fp4q_quantize_if6(x5, amax=amax5, scale_layout=SW, out=oi6)),
        Job("if4 16384x8192 bf16 if3", "if3.cu", nbi3, 1,
            lambda: fq.fp4q_quantize_if3(x5, amax=amax5, scale_layout=SW, out=oi3)),
        Job("activation 8192x4096 bf16 mxfp6 e2m3 row-wise", "mxfp6.cu", nb6, 1,
            lambda: fq.fp4q_quantize_mxfp6(xa, fq.FP6_E2M3, scale_layout=SW, out=o6)),
    ]


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read only)
# ---------------------------------------------------------------------------

_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x2: "applications_clocks_setting", 0x1: "gpu_idle"}


class ClockSampler:
    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _handle(self, idx):
        import torch
        nv = self._nv
        try:
            p = torch.cuda.get_device_properties(idx)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                try:
                    return nv.nvmlDeviceGetHandleByIndex(int(vis.split(",")[idx]))
                except Exception:
                    pass
            return nv.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        nv = self._nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = get_r(self._h)
                for bit, name in _REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.005)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# the CPU oracle on a bounded sample (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def suite_inputs():
    """CPU copies of the suite's inputs (activation, weight, gradient, if4)
    and of the small parity workload."""
    from fp4_block_scaled_04_b200 import workloads
    return {"activation": workloads.activation(), "weight": workloads.weight(),
            "gradient": workloads.gradient(), "if4": workloads.if4_blocks(),
            "small": workloads.small_matrix()}


def input_digests(inputs):
    """First 16 hex digits of the SHA-256 of each input's bytes, for the log."""
    out = {}
    for k, t in inputs.items():
        b = t.contiguous().view(-1).view(torch_uint8()).numpy().tobytes()
        out[k] = hashlib.sha256(b).hexdigest()[:16]
    return out


def torch_uint8():
    import torch
    return torch.uint8


def oracle_sample(rows_fraction: float, inputs=None, parts=None):
    """Run the oracle over the first rows_fraction of every workload of the
    suite; returns (algorithmic bytes of the sample, seconds, description).
    If ``parts`` is a dict, each call's (bytes, seconds) is stored in it under
    the call's workload name."""
    import numpy as np
    import torch
    import oracle as orc

    def bits(t):
        t = t.contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        return t.numpy()

    def rows_of(n, align):
        return max(align, int(n * rows_fraction) // align * align)

    total = [0, 0.0]

    def timed(name, nbytes, fn):
        t0 = time.perf_counter()
        out = fn()
        sec = time.perf_counter() - t0
        total[0] += nbytes
        total[1] += sec
        if parts is not None:
            parts[name] = (nbytes, sec)
        return out

    inputs = inputs or suite_inputs()
    xa, w, g, x5 = inputs["activation"], inputs["weight"], inputs["gradient"], inputs["if4"]
    ra = rows_of(xa.shape[0], 32)
    a = np.ascontiguousarray(bits(xa[:ra]))
    C = xa.shape[1]
    sl = orc.SCALE_SWIZZLED if ra % 128 == 0 else 0
    timed("activation nvfp4 row+col", ra * C * 2 + 2 * (ra * C // 2) + 2 * (ra * C // 16) + 4,
          lambda: orc.quantize_nvfp4(a, layouts=3, scale_layout=sl))
    timed("activation mxfp4 row+col", ra * C * 2 + 2 * (ra * C // 2) + 2 * (ra * C // 32),
          lambda: orc.quantize_mxfp4(a, layouts=3))
    rw = rows_of(w.shape[0], 16)
    ww = np.ascontiguousarray(bits(w[:rw]))
    C = w.shape[1]
    timed("weight 2d16x16 w+wt", rw * C * 4 + 2 * (rw * C // 2) + (rw // 16) * (C // 16) + 4,
          lambda: orc.quantize_2d(ww))
    rg = rows_of(g.shape[0], 128)
    gg = np.ascontiguousarray(bits(g[:rg]))
    C = g.shape[1]
    for n in (16, 128):
        for rnd, rname in ((orc.SR, "sr"), (orc.RNE, "rne")):
            timed(f"gradient rht{n}+{rname}", rg * C * 2 + rg * C // 2 + rg * C // 16 + 4,
                  lambda: orc.quantize_rht(gg, n, round=rnd, seed=0))
    r5 = rows_of(x5.shape[0], 16)
    xx = np.ascontiguousarray(bits(x5[:r5]))
    C = x5.shape[1]
    nb5 = r5 * C * 2 + r5 * C // 2 + r5 * C // 16 + 4
    o = timed("if4 quantize", nb5, lambda: orc.quantize_if4(xx))
    timed("if4 dequantize to bf16", nb5,
          lambda: orc.dequantize(orc.FMT_IF4, o["q"], o["sf"], r5, C,
                                 s_dec=float(o["s_dec"][0]), out_dtype=orc.BF16))
    xs = inputs.get("small")
    if xs is not None:                    # the 256x256 parity workload, whole
        sm = np.ascontiguousarray(bits(xs))
        Rs, Cs = xs.shape
        osm = timed("small 256x256 nvfp4 quantize", Rs * Cs * 2 + Rs * Cs // 2 + Rs * Cs // 16 + 4,
                    lambda: orc.quantize_nvfp4(sm))
        timed("small 256x256 dequantize to fp32", Rs * Cs // 2 + Rs * Cs // 16 + 4 + Rs * Cs * 4,
              lambda: orc.dequantize(orc.FMT_NVFP4, osm["q_row"], osm["sf_row"], Rs, Cs,
                                     s_dec=float(osm["s_dec"][0])))
    desc = (f"oracle (plain C) on the first {rows_fraction:.4g} of the rows of every "
            f"workload of the suite: activation {ra} rows, weight {rw}, gradient {rg}, "
            f"if4 {r5}" + ("; and the whole 256x256 small workload" if xs is not None else ""))
    return total[0], total[1], desc


def host_info():
    """(usable host cores, CPU model name) of this machine."""
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:
        cores = os.cpu_count() or 1
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except Exception:
        pass
    return cores, model


def oracle_baseline(fraction: float, inputs, runs: int = 3):
    """The oracle on the same bounded sample, single-threaded and on all host
    cores (its OpenMP build, which splits only independent rows, columns and
    tile rows and gives the same bytes); the median of `runs` runs each."""
    import oracle as orc
    cores, model = host_info()
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    out, per = {}, {}
    try:
        for mode in ("single", "all"):
            orc.use_openmp(mode == "all")
            times, b, desc, runs_parts = [], 0, "", []
            for _ in range(runs):
                parts = {}
                b, sec, desc = oracle_sample(fraction, inputs, parts)
                times.append(sec)
                runs_parts.append(parts)
            out[mode] = (b, statistics.median(times), desc)
            for name in runs_parts[0]:
                nb = runs_parts[0][name][0]
                med = statistics.median(p[name][1] for p in runs_parts)
                per.setdefault(name, {})["GB/s_1_core" if mode == "single" else "GB/s_all_cores"] = \
                    round(nb / med / 1e9, 5)
    finally:
        orc.use_openmp(False)
    b1, s1, desc = out["single"]
    ba, sa, _ = out["all"]
    return {"value": round(ba / sa / 1e9, 5), "unit": "GB/s",
            "cores": int(os.environ.get("OMP_NUM_THREADS", cores)), "kind": "oracle",
            "sample": desc + "; all host cores (OpenMP build, same bytes)",
            "seconds": round(sa, 3), "runs": runs, "statistic": "median",
            "host_cores": cores, "cpu_model": model,
            "single_thread": {"value": round(b1 / s1 / 1e9, 5), "unit": "GB/s", "cores": 1,
                              "seconds": round(s1, 3)},
            "per_config": per}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return ws, int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0"))


def traffic_for(job_src: str, job_name: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernel's
    source is unchanged since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        rec = json.load(open(path))[job_name]
    except Exception:
        return None
    src = os.path.join(ROOT, "fp4_block_scaled_04_b200", "csrc", job_src)
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return rec["dram_bytes_per_launch"] if rec.get("src_sha256_16") == h else None


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle as orc
    frac = args.reference_fraction
    times, nbytes, desc = [], 0, ""
    inputs = suite_inputs()
    cores, model = host_info()
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    orc.use_openmp(True)
    for i in range(args.warmup + args.steps):
        b, s, desc = oracle_sample(frac, inputs)
        if i >= args.warmup:
            times.append(s)
            nbytes = b
    total = sum(times)
    value = nbytes * len(times) / total / 1e9
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / len(times), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": SUITE_WORKLOAD,
                   "sample": f"bounded row sample per step: the first {frac:.4g} of the rows "
                             "of every workload",
                   "rows_fraction": frac, "l2": "n/a (CPU)", "parallelism": "rank 0 only"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s",
                         "cores": int(os.environ["OMP_NUM_THREADS"]), "kind": "oracle",
                         "sample": desc + "; all host cores (OpenMP build, same bytes)",
                         "cpu_model": model},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--reference-fraction", type=float, default=1.0 / 32)
    ap.add_argument("--cpu-baseline-fraction", type=float, default=1.0 / 16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the calls outside the suite (fused backward, row-wise alone, "
                         "four-over-six, NVINT4, IF6, MXFP6) and the consumer GEMM")
    ap.add_argument("--e2e-steps", type=int, default=None)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    import fp4_block_scaled_04_b200 as fq
    from fp4_block_scaled_04_b200 import dist as fdist

    ws, rank, local = dist_env()
    if ws != args.gpus and ws > 1:
        print(f"warning: WORLD_SIZE={ws} but --gpus {args.gpus}", file=sys.stderr)
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    def barrier():
        if ws > 1:
            dist.barrier()

    fq.lib()
    inputs = suite_inputs()
    jobs = build_jobs(device, fq, inputs)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    flush_sum = torch.empty((), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step(record):
        for j, job in enumerate(jobs):
            torch.cuda._sleep(LEAD_SLEEP_CYCLES)
            flush.fill_(float(j))
            torch.sum(flush, dim=0, out=flush_sum)
            if record is not None:
                record[j][0].record(stream)
            job.run()
            if record is not None:
                record[j][1].record(stream)

    for _ in range(args.warmup):
        step(None)
    torch.cuda.synchronize(device)

    events = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
               for _ in jobs] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(device)
    wall0 = time.perf_counter()
    with ClockSampler(local) as clocks:
        # an untimed device sleep of about 2 ms first: the host then enqueues
        # the first jobs while the device waits, so neither the sampler
        # thread's start nor the loop's first host steps reach the first
        # job's events
        torch.cuda._sleep(FIRST_LEAD_CYCLES)
        for s in range(args.steps):
            step(events[s])
        torch.cuda.synchronize(device)
    barrier()
    wall = time.perf_counter() - wall0
    per_job_ms = [sum(events[s][j][0].elapsed_time(events[s][j][1]) for s in range(args.steps))
                  for j in range(len(jobs))]
    total_ms = sum(per_job_ms)
    total_ms_max = fdist.max_over_ranks(total_ms, device=device)

    step_bytes = sum(j.bytes for j in jobs)
    value = fdist.aggregate_gbs(step_bytes, ws, args.steps, total_ms_max)
    peak, peak_kind = hbm_peak()

    def time_call(run, tag):
        """Average device time (s) of one call, timed like the suite."""
        for _ in range(args.warmup):
            torch.cuda._sleep(LEAD_SLEEP_CYCLES)
            flush.fill_(tag)
            torch.sum(flush, dim=0, out=flush_sum)
            run()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        torch.cuda._sleep(FIRST_LEAD_CYCLES)
        for a, b in ev:
            torch.cuda._sleep(LEAD_SLEEP_CYCLES)
            flush.fill_(tag + 1.0)
            torch.sum(flush, dim=0, out=flush_sum)
            a.record(stream)
            run()
            b.record(stream)
        torch.cuda.synchronize(device)
        return sum(a.elapsed_time(b) for a, b in ev) * 1e-3 / args.steps

    # ---- the same calls with the tensor amax computed first (a pre-pass that
    # reads the input once more; for the gradient it is the transform's amax)
    incl_amax = {}
    for job in jobs:
        if job.run_amax is not None:
            incl_amax[job.name] = time_call(job.run_amax, 3.0)

    # ---- further calls, timed the same way, outside the headline ----------
    extra = []
    if not args.no_extra:
        xjobs = build_extra_jobs(device, fq, inputs)
        for job in xjobs:
            avg_s = time_call(job.run, 1.0)
            gbs = job.bytes / avg_s / 1e9
            entry = {"workload": job.name, "bytes": job.bytes, "us": round(avg_s * 1e6, 2),
                     "GB/s": round(gbs, 1), "pct_of_peak": round(100 * gbs / peak, 1),
                     "dram_bytes": traffic_for(job.src, job.name)}
            if job.run_amax is not None:
                entry["us_incl_amax"] = round(time_call(job.run_amax, 5.0) * 1e6, 2)
            extra.append(entry)
        del xjobs
        torch.cuda.synchronize(device)

    # ---- consumer check: the vendor's block-scaled FP4 GEMM on our operands ---
    gemm = None
    if not args.no_extra:
        gemm = time_consumer_gemm(fq, device, stream, args)

    per_config = []
    for job, ms in zip(jobs, per_job_ms):
        avg_s = ms * 1e-3 / args.steps
        gbs = job.bytes / avg_s / 1e9
        entry = {"workload": job.name, "bytes": job.bytes,
                 "us": round(avg_s * 1e6, 2), "GB/s": round(gbs, 1),
                 "pct_of_peak": round(100 * gbs / peak, 1),
                 "share": round(ms / total_ms, 4),
                 "dram_bytes": traffic_for(job.src, job.name)}
        if job.name in incl_amax:
            # the algorithmic bytes stay those of the call itself; the amax
            # pre-pass's re-read of the input is overhead, not work
            t = incl_amax[job.name]
            entry["us_incl_amax"] = round(t * 1e6, 2)
            entry["GB/s_incl_amax"] = round(job.bytes / t / 1e9, 1)
        per_config.append(entry)
    dom = max(range(len(jobs)), key=lambda j: per_job_ms[j])
    dom_avg_s = per_job_ms[dom] * 1e-3 / args.steps
    dom_achieved = jobs[dom].bytes / dom_avg_s / 1e9
    roofline = {"bound": "hbm", "achieved": round(dom_achieved, 1), "peak": peak,
                "unit": "GB/s", "frac": round(dom_achieved / peak, 4),
                "traffic": traffic_for(jobs[dom].src, jobs[dom].name),
                "kernel": jobs[dom].name, "peak_kind": f"{peak_kind} (HBM copy bandwidth)"}

    # ---- end to end through the public API with host buffers -------------
    e2e = None
    if not args.no_e2e:
        k = args.e2e_steps or max(1, min(args.steps, 10))
        s_in, s_comp, s_out = (torch.cuda.Stream(device) for _ in range(3))
        for i, job in enumerate(jobs):
            job.e2e.step(s_in, s_comp, s_out, first=True)
        torch.cuda.synchronize(device)
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        h2d = d2h = 0
        e0.record(stream)
        for st in (s_in, s_comp, s_out):
            st.wait_event(e0)
        for _ in range(k):
            h2d = d2h = 0
            for job in jobs:
                a, b = job.e2e.step(s_in, s_comp, s_out, first=False)
                h2d += a
                d2h += b
        for st in (s_in, s_comp, s_out):
            ev = torch.cuda.Event()
            ev.record(st)
            stream.wait_event(ev)
        e1.record(stream)
        torch.cuda.synchronize(device)
        e_ms = fdist.max_over_ranks(e0.elapsed_time(e1), device=device)
        e2e = {"value": round(fdist.aggregate_gbs(step_bytes, ws, k, e_ms), 3), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": k,
               "path": "pinned host -> device copy, C-ABI call (tensor amax computed inside), "
                       "device -> pinned host copy of every output; copies, calls and copies "
                       "back on three streams, so neighbouring jobs' transfers overlap"}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(args.cpu_baseline_fraction, inputs)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms_max / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": SUITE_WORKLOAD,
                       "l2": "flushed before every kernel (256 MiB written then read, untimed)",
                       "launch": "device sleep before each flush hides host launch latency",
                       "amax": "precomputed on the device (headline); per_config "
                               "us_incl_amax and e2e compute it first",
                       "parallelism": f"replicas x{ws}" if ws > 1 else "single gpu",
                       "input_sha256_16": input_digests(inputs)},
            "pct_of_peak": round(100 * value / (ws * peak), 2),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": sum(j.launches for j in jobs) * args.steps,
            "clocks": clocks.summary(), "wall_s_timed_region": round(wall, 4),
            "per_config": per_config,
            "extra_configs": extra,
            "consumer_gemm": gemm,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
