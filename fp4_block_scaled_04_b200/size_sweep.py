"""Fixed cost and steady rate of the kernels: time one op over a range of
sizes, timed as the benchmark times it, and fit t = t0 + bytes / rate.

    python -m fp4_block_scaled_04_b200.size_sweep [--ops nvfp4_rowcol,if4] [--reps 25]

Every timed call sits between two CUDA events on the launching stream. A device
sleep and an L2 flush come before each call, as in ``bench.py``: 256 MiB are
written and then read back, untimed. The sweep also times the two events with
nothing between them, and a call on a 128 x 64 tensor, which is one launch
that does almost no work. Together these split a kernel's time into:

  - the floor of the timing itself (the empty event pair);
  - the cost of one launch that does almost nothing;
  - ``t0``, the intercept of the fit: the fixed cost of one full-size launch,
    including the pipeline's ramp-up at the start and its drain at the end;
  - ``rate``, the slope: the streaming rate once the kernel is running, in
    algorithmic bytes per second.

For scale, a plain device-to-device copy (``Tensor.copy_``, the operation behind
the measured HBM peak) is timed the same way at each benchmark workload's
byte count: read plus write equal to the kernel's algorithmic bytes. It shows
what the same fixed costs leave of the copy bandwidth at that size.

The fit uses the sizes from half the benchmark's shape upward. There the time
grows linearly with the bytes; smaller launches are still ramping up.
"""
from __future__ import annotations

import argparse
import json
import sys

import torch

import fp4_block_scaled_04_b200 as fq
from fp4_block_scaled_04_b200 import profile_case as pc

# op -> (row counts, columns, algorithmic bytes per element): the benchmark's
# own shape is the second row count
SWEEP = {
    "nvfp4_rowcol": ([4096, 8192, 16384, 32768], 4096, 3.125),
    "mxfp4_rowcol": ([4096, 8192, 16384, 32768], 4096, 3.0625),
    "2d": ([7168, 14336, 28672], 4096, 4 + 1.0 + 1.0 / 256),
    "rht16_rne": ([4096, 8192, 16384, 32768], 5120, 2.5625),
    "rht16_sr": ([4096, 8192, 16384, 32768], 5120, 2.5625),
    "rht128_rne": ([4096, 8192, 16384, 32768], 5120, 2.5625),
    "rht128_sr": ([4096, 8192, 16384, 32768], 5120, 2.5625),
    "if4": ([8192, 16384, 32768], 8192, 2.5625),
    "if4_dequant": ([8192, 16384, 32768], 8192, 2.5625),
}


def timer(reps: int, dev):
    flush = torch.empty((256 << 20) // 4, dtype=torch.float32, device=dev)
    fsum = torch.empty((), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def run(call) -> float:
        for _ in range(3):
            call()
        torch.cuda.synchronize(dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        torch.cuda._sleep(4_000_000)   # ~2 ms, untimed: the host gets ahead of the device
        for i, (a, b) in enumerate(ev):
            torch.cuda._sleep(200000)
            flush.fill_(float(i))
            torch.sum(flush, dim=0, out=fsum)
            a.record(stream)
            call()
            b.record(stream)
        torch.cuda.synchronize(dev)
        return sum(a.elapsed_time(b) for a, b in ev) * 1e3 / reps   # mean, µs
    return run


def fit(points):
    """Least-squares line through (bytes, µs): returns (t0 µs, rate GB/s)."""
    n = len(points)
    mx = sum(b for b, _ in points) / n
    my = sum(t for _, t in points) / n
    sxx = sum((b - mx) ** 2 for b, _ in points)
    sxy = sum((b - mx) * (t - my) for b, t in points)
    slope = sxy / sxx                        # µs per byte
    return my - slope * mx, 1e-3 / slope     # GB/s = bytes / µs / 1e3


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--ops", default=",".join(SWEEP))
    ap.add_argument("--reps", type=int, default=25)
    a = ap.parse_args(argv)
    dev = torch.device("cuda", 0)
    fq.lib()
    run = timer(a.reps, dev)
    out = {"empty_event_pair_us": round(run(lambda: None), 2)}
    tiny = pc.make("nvfp4_row", 128, 64, dev)
    out["tiny_launch_us"] = round(run(tiny), 2)
    del tiny
    print(json.dumps(out), flush=True)
    for name, nbytes in (("activation 8192x4096 nvfp4 row+col", 104857604),
                         ("gradient 8192x5120 rht", 107479044),
                         ("weight 14336x4096 2d", 293830660),
                         ("if4 16384x8192", 343932932)):
        n = nbytes // 4                    # BF16 elements: n * 2 read + n * 2 written
        src = torch.empty(n, dtype=torch.bfloat16, device=dev).normal_()
        dst = torch.empty_like(src)
        us = run(lambda: dst.copy_(src))
        print(json.dumps({"copy_like": name, "bytes": 4 * n, "us": round(us, 2),
                          "GB/s": round(4 * n / us / 1e3, 1)}), flush=True)
        del src, dst
        torch.cuda.empty_cache()
    for op in a.ops.split(","):
        rows, cols, bpe = SWEEP[op]
        pts = []
        for r in rows:
            call = pc.make(op, r, cols, dev)
            us = run(call)
            nbytes = r * cols * bpe
            pts.append((nbytes, us))
            print(json.dumps({"op": op, "rows": r, "cols": cols, "bytes": int(nbytes),
                              "us": round(us, 2), "GB/s": round(nbytes / us / 1e3, 1)}), flush=True)
            del call
            torch.cuda.empty_cache()
        t0, rate = fit([p for p in pts if p[0] >= rows[1] * cols * bpe / 2])
        print(json.dumps({"op": op, "fit_t0_us": round(t0, 2), "fit_rate_GB/s": round(rate, 1)}),
              flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
