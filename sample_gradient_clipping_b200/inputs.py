"""Seeded synthetic workloads for the per-sample clip + sum + noise step.

This module only draws input tensors and lists the workload parameters.  It holds none of the
method's arithmetic.  Both the CUDA path and the fp64 oracle read the tensors it returns, so
the two sides see identical bits.

The shapes stand in for the layers the pages train:

* Llama-13B pre-training (FlashDP page, Abstract);
* RoBERTa-Large fine-tuning on SST-2 (DP-GRAPE page, Experimental Results);
* a GPT-2-small MLP and a Llama-7B block as two more transformer linears.

No dataset or trained weight is involved: X and dY are Gaussian.

Draw order (``numpy.random.default_rng(seed)``, standard normals drawn as float32):

1. The 13B block first draws ``s = rng.lognormal(0, 1, B)``.
2. Then, per linear in layer order, X is drawn when its input is new, then dY.

Inside a block, q, k and v share one X, gate and up share one X, and o and down each have their
own X, as in a transformer block.  bf16 tensors are the fp32 draws rounded by
``torch.Tensor.to(torch.bfloat16)`` (round to nearest even).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Linear:
    name: str
    d_in: int
    d_out: int
    x_key: str            # linears with the same key read the same X
    layer_id: int


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    dtype: str                    # "f32" or "bf16"
    linears: tuple
    C: float                      # per-layer clip bound C_l
    sigma: float
    seed: int
    step: int = 0
    x_std: float = 1.0
    dy_var: object = None         # float, or "per_layer" (13B block: C_l^2 / (d_in d_out T))
    sample_scale: str = ""        # "lognormal" for the 13B block
    r: int = 0                    # projection rank, 0 = unprojected
    description: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def tokens(self):
        return self.B * self.T


def _block(prefix_ids, d, ffn, qkv_out=None):
    q = qkv_out or d
    return (
        Linear("q", d, q, "attn_in", prefix_ids + 0),
        Linear("k", d, q, "attn_in", prefix_ids + 1),
        Linear("v", d, q, "attn_in", prefix_ids + 2),
        Linear("o", q, d, "attn_out", prefix_ids + 3),
        Linear("gate", d, ffn, "mlp_in", prefix_ids + 4),
        Linear("up", d, ffn, "mlp_in", prefix_ids + 5),
        Linear("down", ffn, d, "mlp_mid", prefix_ids + 6),
    )


WORKLOADS = {
    "tiny_f32": Workload(
        "tiny_f32", B=4, T=16, dtype="f32",
        linears=(Linear("linear", 64, 32, "in", 0),),
        C=1.0, sigma=1.0, seed=0, dy_var=1.0 / 16,
        description="tiny single linear, fp32: B=4, T=16, 64->32"),
    "gpt2_mlp_up": Workload(
        "gpt2_mlp_up", B=32, T=512, dtype="bf16",
        linears=(Linear("mlp_up", 768, 3072, "in", 0),),
        C=1.0, sigma=0.8, seed=1, dy_var=1e-4,
        description="GPT-2-small MLP up-projection: B=32, T=512, 768->3072, bf16"),
    "llama7b_block": Workload(
        "llama7b_block", B=8, T=2048, dtype="bf16",
        linears=_block(0, 4096, 11008),
        C=1.0 / math.sqrt(7.0), sigma=1.0, seed=2, dy_var=1e-5,
        description="Llama-7B-shaped block, 7 linears, B=8, T=2048, bf16, per-layer C_l=1/sqrt(7)"),
    "llama13b_block": Workload(
        "llama13b_block", B=4, T=2048, dtype="bf16",
        linears=_block(0, 5120, 13824),
        C=1.0 / math.sqrt(7.0), sigma=0.6, seed=3, dy_var="per_layer",
        sample_scale="lognormal",
        description="Llama-13B-shaped block, 7 linears, B=4, T=2048, bf16, "
                    "dY rows of sample i scaled by s_i ~ LogNormal(0,1)"),
    "roberta_large_projected": Workload(
        "roberta_large_projected", B=64, T=128, dtype="bf16",
        linears=(
            Linear("q", 1024, 1024, "attn_in", 0),
            Linear("k", 1024, 1024, "attn_in", 1),
            Linear("v", 1024, 1024, "attn_in", 2),
            Linear("o", 1024, 1024, "attn_out", 3),
            Linear("fc1", 1024, 4096, "mlp_in", 4),
            Linear("fc2", 4096, 1024, "mlp_mid", 5),
        ),
        C=1.0, sigma=1.0, seed=4, dy_var=1.0 / 128, r=128,
        description="RoBERTa-large-shaped linears, projected to r=128, B=64, T=128, bf16"),
}


def custom(name, B, T, d_in, d_out, dtype="bf16", C=1.0, sigma=1.0, seed=11, step=0,
           dy_var=None, r=0, layer_id=0):
    """A one-linear workload of any shape (parity tests: ragged tails, edge cases)."""
    if dy_var is None:
        dy_var = 1.0 / T
    return Workload(name, B=B, T=T, dtype=dtype,
                    linears=(Linear("linear", d_in, d_out, "in", layer_id),),
                    C=C, sigma=sigma, seed=seed, step=step, dy_var=dy_var, r=r,
                    description=f"custom {B}x{T}, {d_in}->{d_out}, {dtype}")


def _normal(rng, shape, scale):
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        a *= np.float32(scale)
    return a


def _dy_std(w, lin):
    if w.dy_var == "per_layer":
        return math.sqrt(w.C ** 2 / (lin.d_in * lin.d_out * w.T))
    return math.sqrt(float(w.dy_var))


def generate(w, linears=None, as_torch=True):
    """Draw the workload's tensors.

    Returns ``{"X": {x_key: array}, "dY": {name: array}, "s": s or None}``.  The arrays are
    ``[B, T, d]``.  They are torch CPU tensors in the workload dtype when ``as_torch`` is
    true, else fp32 numpy arrays.  ``linears`` (names) restricts which dY are kept.  All
    draws still happen, so the bits do not depend on the selection.
    """
    import torch

    rng = np.random.default_rng(w.seed)
    s = None
    if w.sample_scale == "lognormal":
        s = rng.lognormal(0.0, 1.0, w.B)
    keep = set(linears) if linears is not None else None
    X, dY = {}, {}

    def cast(a):
        if not as_torch:
            return a
        t = torch.from_numpy(a)
        return t.to(torch.bfloat16) if w.dtype == "bf16" else t

    need_x = set()
    for lin in w.linears:
        if keep is None or lin.name in keep:
            need_x.add(lin.x_key)
    for lin in w.linears:
        if lin.x_key not in X and lin.x_key not in ("__drawn__",):
            a = _normal(rng, (w.B, w.T, lin.d_in), w.x_std)
            X[lin.x_key] = cast(a) if lin.x_key in need_x else None
        a = _normal(rng, (w.B, w.T, lin.d_out), _dy_std(w, lin))
        if s is not None:
            a *= s.astype(np.float32)[:, None, None]
        if keep is None or lin.name in keep:
            dY[lin.name] = cast(a)
        del a
    X = {k: v for k, v in X.items() if v is not None}
    return {"X": X, "dY": dY, "s": s}


def as_f64(t):
    """Exact fp64 copy of a torch or numpy tensor (bf16 and fp32 widen exactly)."""
    import torch

    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)
