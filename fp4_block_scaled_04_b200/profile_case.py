"""Run one fp4q kernel on one seeded workload, for profilers.

    python -m fp4_block_scaled_04_b200.profile_case --op nvfp4_rowcol \\
        --rows 16384 --cols 8192 --iters 3

Inputs are generated on the host from the workload generators (same value
distributions as the benchmark, any size), copied to cuda:0, the tensor amax
is computed once, then the kernel under study runs ``--warmup`` times and
``--iters`` times more, with a device synchronize at the end.  Each of those
runs is exactly one launch of the kernel named by ``--op`` (the amax
pre-pass is outside them; ``gemm_if4`` launches the IF4 split pass before
its GEMM), so a profiler can skip the warm-up launches and capture the rest.
"""
from __future__ import annotations

import argparse
import sys

import torch

import fp4_block_scaled_04_b200 as fq
from fp4_block_scaled_04_b200 import workloads

OPS = ["amax", "nvfp4_row", "nvfp4_rowcol", "mxfp4_rowcol", "2d", "rht16_sr", "rht128_sr",
       "rht16_rne", "rht128_rne", "if4", "if4_dequant", "four_over_six_rowcol", "nvint4",
       "bwd16_sr", "bwd16_rne", "row_sr", "mxfp6_e2m3", "mxfp6_dequant", "gemm_nvfp4", "gemm_if4", "if6", "if3",
       "if3_dequant"]


def make(op: str, rows: int, cols: int, dev):
    sw = fq.SCALE_SWIZZLED if rows % 128 == 0 else fq.SCALE_LINEAR
    if op in ("bwd16_sr", "bwd16_rne", "row_sr"):
        g = workloads.gradient(tokens=rows, cols=cols).to(dev)
        a = fq.fp4q_amax(g)
        ar = fq.fp4q_rht_amax(g, 16)
        rnd = fq.RNE if op == "bwd16_rne" else fq.SR
        if op == "row_sr":
            o = fq.fp4q_quantize_nvfp4(g, layouts=fq.ROWWISE, round=fq.SR, amax=a, scale_layout=sw)
            return lambda: fq.fp4q_quantize_nvfp4(g, layouts=fq.ROWWISE, round=fq.SR, amax=a,
                                                  scale_layout=sw, out=o)
        o = fq.fp4q_quantize_backward(g, 16, round=rnd, amax_row=a, amax_rht=ar, scale_layout=sw)
        return lambda: fq.fp4q_quantize_backward(g, 16, round=rnd, amax_row=a, amax_rht=ar,
                                                 scale_layout=sw, out=o)
    if op == "four_over_six_rowcol":
        x = workloads.activation(rows=rows, cols=cols).to(dev)
        a = fq.fp4q_amax(x)
        o = fq.fp4q_quantize_four_over_six(x, layouts=3, amax=a, scale_layout=sw)
        return lambda: fq.fp4q_quantize_four_over_six(x, layouts=3, amax=a, scale_layout=sw,
                                                      out=o)
    if op == "gemm_nvfp4":              # M = N = rows, K = cols
        g = torch.Generator().manual_seed(5)
        x = torch.randn(rows, cols, generator=g).to(torch.bfloat16).to(dev)
        w = (torch.randn(rows, cols, generator=g) * 0.05).to(torch.bfloat16).to(dev)
        ox = fq.fp4q_quantize_nvfp4(x, scale_layout=fq.SCALE_SWIZZLED)
        ow = fq.fp4q_quantize_nvfp4(w, scale_layout=fq.SCALE_SWIZZLED)
        c = torch.empty((rows, rows), dtype=torch.bfloat16, device=dev)
        return lambda: fq.fp4q_gemm_nvfp4(ox["q_row"], ox["sf_row"], ow["q_row"], ow["sf_row"],
                                          cols, tensor_scale_a=ox["s_dec"],
                                          tensor_scale_b=ow["s_dec"], out=c)
    if op == "gemm_if4":                # IF4 x NVFP4, M = N = rows, K = cols, FP32 out
        g = torch.Generator().manual_seed(6)
        x = torch.randn(rows, cols, generator=g).to(torch.bfloat16).to(dev)
        w = (torch.randn(rows, cols, generator=g) * 0.05).to(torch.bfloat16).to(dev)
        ox = fq.fp4q_quantize_if4(x, scale_layout=fq.SCALE_SWIZZLED)
        ow = fq.fp4q_quantize_nvfp4(w, scale_layout=fq.SCALE_SWIZZLED)
        c = torch.empty((rows, rows), dtype=torch.float32, device=dev)
        ws = torch.empty(int(fq.lib().fp4q_gemm_if4_workspace_bytes(rows, cols)),
                         dtype=torch.uint8, device=dev)
        return lambda: fq.fp4q_gemm_if4_nvfp4(ox["q"], ox["sf"], ow["q_row"], ow["sf_row"], cols,
                                              tensor_scale_a=ox["s_dec"],
                                              tensor_scale_b=ow["s_dec"], out=c, workspace=ws)
    if op in ("mxfp6_e2m3", "mxfp6_dequant"):
        x = workloads.activation(rows=rows, cols=cols).to(dev)
        o = fq.fp4q_quantize_mxfp6(x, fq.FP6_E2M3, scale_layout=sw)
        if op == "mxfp6_e2m3":
            return lambda: fq.fp4q_quantize_mxfp6(x, fq.FP6_E2M3, scale_layout=sw, out=o)
        y = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev)
        return lambda: fq.fp4q_dequantize(fq.FMT_MXFP6_E2M3, o["q"], o["sf"], rows, cols, 1, 32,
                                          scale_layout=sw, out=y)
    if op == "if6":
        x = workloads.if4_blocks(rows=rows, cols=cols).to(dev)
        a = fq.fp4q_amax(x)
        o = fq.fp4q_quantize_if6(x, amax=a, scale_layout=sw)
        return lambda: fq.fp4q_quantize_if6(x, amax=a, scale_layout=sw, out=o)
    if op in ("if3", "if3_dequant"):
        x = workloads.if4_blocks(rows=rows, cols=cols).to(dev)
        a = fq.fp4q_amax(x)
        o = fq.fp4q_quantize_if3(x, amax=a, scale_layout=sw)
        if op == "if3":
            return lambda: fq.fp4q_quantize_if3(x, amax=a, scale_layout=sw, out=o)
        y = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev)
        return lambda: fq.fp4q_dequantize(fq.FMT_IF3, o["q"], o["sf"], rows, cols, 1, 16,
                                          tensor_scale=o["s_dec"], scale_layout=sw, out=y)
    if op == "nvint4":
        x = workloads.if4_blocks(rows=rows, cols=cols).to(dev)
        a = fq.fp4q_amax(x)
        o = fq.fp4q_quantize_nvint4(x, amax=a, scale_layout=sw)
        return lambda: fq.fp4q_quantize_nvint4(x, amax=a, scale_layout=sw, out=o)
    if op in ("amax", "nvfp4_row", "nvfp4_rowcol", "mxfp4_rowcol"):
        x = workloads.activation(rows=rows, cols=cols).to(dev)
        if op == "amax":
            out = torch.empty(1, device=dev)
            return lambda: fq.fp4q_amax(x, out=out)
        a = fq.fp4q_amax(x)
        if op == "nvfp4_row":
            o = fq.fp4q_quantize_nvfp4(x, layouts=fq.ROWWISE, amax=a, scale_layout=sw)
            return lambda: fq.fp4q_quantize_nvfp4(x, layouts=fq.ROWWISE, amax=a, scale_layout=sw, out=o)
        if op == "nvfp4_rowcol":
            o = fq.fp4q_quantize_nvfp4(x, layouts=3, amax=a, scale_layout=sw)
            return lambda: fq.fp4q_quantize_nvfp4(x, layouts=3, amax=a, scale_layout=sw, out=o)
        o = fq.fp4q_quantize_mxfp4(x, layouts=3, scale_layout=sw)
        return lambda: fq.fp4q_quantize_mxfp4(x, layouts=3, scale_layout=sw, out=o)
    if op == "2d":
        w = workloads.weight(rows=rows, cols=cols).to(dev)
        a = fq.fp4q_amax(w)
        o = fq.fp4q_quantize_2d(w, amax=a)
        return lambda: fq.fp4q_quantize_2d(w, amax=a, out=o)
    if op.startswith("rht"):
        n = 16 if op.startswith("rht16") else 128
        rnd = fq.SR if op.endswith("sr") else fq.RNE
        g = workloads.gradient(tokens=rows, cols=cols).to(dev)
        a = fq.fp4q_rht_amax(g, n)
        o = fq.fp4q_quantize_rht_sr(g, n, round=rnd, amax_rht=a, scale_layout=sw)
        return lambda: fq.fp4q_quantize_rht_sr(g, n, round=rnd, amax_rht=a, scale_layout=sw, out=o)
    if op in ("if4", "if4_dequant"):
        x = workloads.if4_blocks(rows=rows, cols=cols).to(dev)
        a = fq.fp4q_amax(x)
        o = fq.fp4q_quantize_if4(x, amax=a, scale_layout=sw)
        if op == "if4":
            return lambda: fq.fp4q_quantize_if4(x, amax=a, scale_layout=sw, out=o)
        y = torch.empty((rows, cols), dtype=torch.bfloat16, device=dev)
        return lambda: fq.fp4q_dequantize(fq.FMT_IF4, o["q"], o["sf"], rows, cols,
                                          tensor_scale=o["s_dec"], scale_layout=sw, out=y)
    raise ValueError(op)


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--op", choices=OPS, required=True)
    ap.add_argument("--rows", type=int, required=True)
    ap.add_argument("--cols", type=int, required=True)
    ap.add_argument("--warmup", type=int, default=1)
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args(argv)
    dev = torch.device("cuda", 0)
    run = make(a.op, a.rows, a.cols, dev)
    torch.cuda.synchronize(dev)
    for _ in range(a.warmup + a.iters):
        run()
    torch.cuda.synchronize(dev)
    print(f"profile_case {a.op} {a.rows}x{a.cols}: {a.warmup} warm-up + {a.iters} launches done")
    return 0


if __name__ == "__main__":
    sys.exit(main())
