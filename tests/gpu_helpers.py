"""Shared helpers of the GPU parity tests (tolerances, error measures, oracle runs)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sample_gradient_clipping_b200 import inputs

# Parity bounds for the step: fp32 inputs, bf16 inputs with fp32 accumulation, and noise.
TOL = {
    "f32": {"sum": 1e-5, "norm": 1e-6},
    "bf16": {"sum": 5e-3, "norm": 1e-3},
}
NOISE_ABS = 1e-6
CLIP_BAND = 1e-3   # clip decisions may differ only when |n_i / C - 1| <= 1e-3


def rel_fro(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def rel_max(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.max(np.abs(got - want) / np.maximum(np.abs(want), 1e-300)))


def host(t):
    return t.detach().to("cpu", torch.float64).numpy()


def check_clip_decisions(norms_gpu, norms_oracle, C):
    for i, (ng, no) in enumerate(zip(norms_gpu, norms_oracle)):
        if abs(no / C - 1.0) <= CLIP_BAND:
            continue
        assert (ng > C) == (no > C), f"clip decision of sample {i}: gpu {ng} oracle {no} C {C}"


def rounding_allowance(out_a, out_b):
    """fp32 rounding of the two outputs whose difference is compared with the noise: at most
    half an ulp of each, written as two ulps of the larger magnitude."""
    mag = np.maximum(np.abs(out_a), np.abs(out_b))
    return 2.0 * np.spacing(mag.astype(np.float32)).astype(np.float64)


def noise_tolerance(out_a, out_b):
    """1e-6 plus the fp32 rounding of adding the noise to values of this magnitude."""
    return NOISE_ABS + rounding_allowance(out_a, out_b)


def noise_excess(out_a, out_b, want):
    """Largest error of (out_a - out_b) against the exact noise beyond the fp32 rounding
    allowance: the figure that the 1e-6 bound applies to."""
    err = np.abs((np.asarray(out_a, np.float64) - np.asarray(out_b, np.float64)) - want)
    return float(np.max(err - rounding_allowance(out_a, out_b))) if err.size else 0.0


# Measured parity errors of this session, (test, item, quantity, value, bound); the summary
# hook in conftest.py prints them so that each run records how close it came to each bound.
MARGINS = []


def record(test, item, quantity, value, bound):
    MARGINS.append((test, str(item), quantity, float(value), float(bound)))


def draw(w, linears=None, device="cuda"):
    """Workload tensors on the host (for the oracle) and on the device (for the library)."""
    data = inputs.generate(w, linears=linears)
    dev = {"X": {k: v.to(device) for k, v in data["X"].items()},
           "dY": {k: v.to(device) for k, v in data["dY"].items()}}
    return data, dev


def oracle_projection(w, lin):
    """The oracle's own P for a projected workload, rounded as the library rounds it."""
    P = oracle.projection(lin.d_out, w.r, w.seed, lin.layer_id)
    return oracle.round_to(w.dtype, P)
