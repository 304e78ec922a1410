"""Times one entry point of the library on its own, for profiling a single kernel.

    python -m sample_gradient_clipping_b200.kernel_bench --op noise --rows 8192 --cols 8192
    python -m sample_gradient_clipping_b200.kernel_bench --op norms --method explicit \\
        --B 8 --T 2048 --d-in 4096 --d-out 4096

Ops: ``noise`` (dp_add_noise on an fp32 [rows, cols] buffer), ``projection``
(dp_projection_matrix, bf16 [rows, cols]), ``philox`` (dp_philox_blocks, rows*cols/4 blocks),
``norms`` (dp_per_sample_norms) and ``clip_accumulate`` (dp_clip_accumulate) on seeded bf16
inputs [B, T, d].  Prints one JSON line: microseconds per call (CUDA events around ``--iters``
calls after ``--warmup`` calls) and the algorithmic bytes or flops per second.
"""
from __future__ import annotations

import argparse
import json


def main(argv=None):
    import torch

    from . import _lib, inputs

    ap = argparse.ArgumentParser()
    ap.add_argument("--op", required=True, choices=["noise", "projection", "philox", "norms", "clip_accumulate"])
    ap.add_argument("--rows", type=int, default=8192)
    ap.add_argument("--cols", type=int, default=8192)
    ap.add_argument("--B", type=int, default=8)
    ap.add_argument("--T", type=int, default=2048)
    ap.add_argument("--d-in", type=int, default=4096)
    ap.add_argument("--d-out", type=int, default=4096)
    ap.add_argument("--method", default="auto", choices=list(_lib.METHODS))
    ap.add_argument("--iters", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    a = ap.parse_args(argv)
    _lib.lib()
    dev = torch.device("cuda")
    rows, cols = a.rows, a.cols
    if a.op == "noise":
        G = torch.zeros(rows, cols, dtype=torch.float32, device=dev)
        call = lambda k: _lib.dp_add_noise(G, 0.5, 7, k, 3)
        work, unit = 8.0 * rows * cols, "GB/s"      # read and write fp32
    elif a.op == "projection":
        P = torch.empty(rows, cols, dtype=torch.bfloat16, device=dev)
        call = lambda k: _lib.dp_projection_matrix(P, 7 + k, 3)
        work, unit = 2.0 * rows * cols, "GB/s"
    elif a.op == "philox":
        nblk = rows * cols // 4
        out = torch.empty(nblk, 4, dtype=torch.int32, device=dev)
        call = lambda k: _lib.dp_philox_blocks(nblk, 7, k, 3, 0, out=out)
        work, unit = 16.0 * nblk, "GB/s"
    else:
        w = inputs.custom("kernel_bench", B=a.B, T=a.T, d_in=a.d_in, d_out=a.d_out, C=1.0, sigma=0.0, seed=1)
        d = inputs.generate(w)
        X, dY = d["X"]["in"].to(dev), d["dY"]["linear"].to(dev)
        ws = torch.empty(_lib.workspace_size(a.B, a.T, a.d_in, a.d_out, 0, _lib.DP_BF16, a.method),
                         dtype=torch.uint8, device=dev)
        n = torch.empty(a.B, dtype=torch.float32, device=dev)
        flops = 2.0 * a.B * a.T * a.d_in * a.d_out
        if a.op == "norms":
            call = lambda k: _lib.dp_per_sample_norms(X, dY, method=a.method, norms=n, workspace=ws)
        else:
            _lib.dp_per_sample_norms(X, dY, method=a.method, norms=n, workspace=ws)
            G = torch.zeros(a.d_in, a.d_out, dtype=torch.float32, device=dev)
            call = lambda k: _lib.dp_clip_accumulate(X, dY, n, 1.0, G, workspace=ws)
        work, unit = flops, "TFLOP/s"
    for k in range(a.warmup):
        call(k)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for k in range(a.iters):
        call(a.warmup + k)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / a.iters
    rate = work / (us * 1e-6) / (1e9 if unit == "GB/s" else 1e12)
    print(json.dumps({"op": a.op, "us_per_call": us, "rate": rate, "unit": unit,
                      "shape": {"rows": rows, "cols": cols} if a.op in ("noise", "projection", "philox")
                      else {"B": a.B, "T": a.T, "d_in": a.d_in, "d_out": a.d_out, "method": a.method}}))


if __name__ == "__main__":
    main()
