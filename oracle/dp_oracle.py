"""fp64 CPU oracle for the per-sample clip + sum + noise step of DP-SGD on one linear layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module: only the tests,
``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline`` and ``--impl reference``
legs) may call it.  It shares no code with the CUDA library.  The one module both sides use is
``sample_gradient_clipping_b200.inputs``, which only draws seeded synthetic tensors.

What it computes, for a linear layer Y = X W with X[B,T,d_in] and dY[B,T,d_out]:

* ``G_i = X_i^T dY_i``, the weight gradient of sample i.  The need to clip it per sample is
  the problem both pages address.  Sources: "FlashDP: Private Training Large Language Models
  with Efficient DP-SGD", Abstract ("per-sample gradient clipping", "per-layer clipped
  DP-SGD"); "Memory-Efficient Differentially Private Training with Gradient Random
  Projection", Problem Statement (per-sample gradients are clipped before noise is added).
* ``n_i = ||G_i||_F`` and the clip factor ``c_i = min(1, C / n_i)``, with ``c_i = 1`` when
  ``n_i <= C`` (so ``n_i = 0`` needs no division).
* ``S = sum_i c_i G_i``, then ``S~ = S + sigma * C * z``, where z is the Gaussian noise
  defined below.  Noise follows clipping (DP-GRAPE page, Methodology, "Order of Operations").
* The projected variant.  ``P[d_out, r]`` has N(0, 1/r) entries regenerated from a seed.  The
  raw per-sample gradient is projected first, ``R_i = G_i P``, and only then clipped, summed
  and noised in r-space (DP-GRAPE page, Methodology: "Random Projection over SVD" and
  "Order of Operations").

Every floating-point step is fp64.  Inputs are the exact fp64 values of the bits the GPU
reads (fp32, or bf16 widened exactly).  A library matmul serves as the contraction step; no
step is blocked, fused or reordered beyond the definition above.

Random numbers
--------------
Philox4x32-10 follows Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as easy as 1,
2, 3" (SC'11).  It runs ten rounds on a 4x32-bit counter with a 2x32-bit key.  Each round
takes two 32x32->64-bit products.  The key is bumped by the two Weyl constants between rounds.

The pages fix no counter layout, so this module reads it as follows:

* key = (seed mod 2^32, seed >> 32);
* counter = (j, layer_id, step mod 2^32, stream);
* stream 0 is the gradient noise, stream 1 the projection matrix;
* block j yields the four words (x0, x1, x2, x3).

Box and Muller, "A note on the generation of random normal deviates" (Ann. Math. Stat.,
1958), maps each pair (x_even, x_odd) as follows:

* u1 = (x_even + 1) 2^-32, which lies in (0, 1];
* u2 = x_odd 2^-32, which lies in [0, 1);
* z_even = sqrt(-2 ln u1) cos(2 pi u2);
* z_odd = sqrt(-2 ln u1) sin(2 pi u2).

Flat element k of a buffer takes z_{k mod 4} of block j = k div 4.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "philox4x32_10", "box_muller", "normals", "normals_at", "noise", "projection",
    "round_to", "per_sample_gradient", "per_sample_norm", "per_sample_norms",
    "clip_factors", "clipped_sum", "clipped_sum_entries", "linear_step", "block_step",
    "projected_adam",
    "NOISE_STREAM", "PROJECTION_STREAM",
]

# Philox4x32 round multipliers and Weyl key increments, as given by Salmon et al. (SC'11).
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
PHILOX_ROUNDS = 10

NOISE_STREAM = 0
PROJECTION_STREAM = 1

_MASK32 = np.uint64(0xFFFFFFFF)
_TWO_M32 = 2.0 ** -32
_CHUNK_BLOCKS = 1 << 20


def philox4x32_10(counters, key):
    """Philox4x32-10 bijection on counters ``uint32[..., 4]`` under ``key = (k0, k1)``.

    Returns ``uint32[..., 4]``.  Round r maps (c0, c1, c2, c3) to
    ``(hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0))``; the key is bumped
    by (W0, W1) before every round but the first.
    """
    ctr = np.asarray(counters, dtype=np.uint64)
    c0, c1, c2, c3 = (ctr[..., i].copy() for i in range(4))
    k0 = np.uint64(int(key[0]) & 0xFFFFFFFF)
    k1 = np.uint64(int(key[1]) & 0xFFFFFFFF)
    m0, m1 = np.uint64(PHILOX_M0), np.uint64(PHILOX_M1)
    for rnd in range(PHILOX_ROUNDS):
        if rnd:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK32
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK32
        p0 = m0 * c0          # exact: both factors < 2^32
        p1 = m1 * c2
        c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ k0, p1 & _MASK32,
                          (p0 >> np.uint64(32)) ^ c3 ^ k1, p0 & _MASK32)
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def box_muller(x_even, x_odd):
    """Box-Muller (1958) on one pair of uint32 words; returns fp64 (z_even, z_odd)."""
    u1 = (np.asarray(x_even, dtype=np.float64) + 1.0) * _TWO_M32
    u2 = np.asarray(x_odd, dtype=np.float64) * _TWO_M32
    radius = np.sqrt(-2.0 * np.log(u1))
    angle = 2.0 * math.pi * u2
    return radius * np.cos(angle), radius * np.sin(angle)


def _seed_key(seed):
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return (seed & 0xFFFFFFFF, seed >> 32)


def _blocks(j, seed, step, layer_id, stream):
    """Normals of Philox blocks ``j`` (uint64 array): fp64 ``[len(j), 4]``."""
    ctr = np.empty(j.shape + (4,), dtype=np.uint64)
    ctr[..., 0] = j
    ctr[..., 1] = int(layer_id) & 0xFFFFFFFF
    ctr[..., 2] = int(step) & 0xFFFFFFFF
    ctr[..., 3] = int(stream) & 0xFFFFFFFF
    x = philox4x32_10(ctr, _seed_key(seed))
    z = np.empty(x.shape, dtype=np.float64)
    z[..., 0], z[..., 1] = box_muller(x[..., 0], x[..., 1])
    z[..., 2], z[..., 3] = box_muller(x[..., 2], x[..., 3])
    return z


def normals(count, seed, step, layer_id, stream):
    """The first ``count`` standard normals z_0 .. z_{count-1} of one (seed, step, layer, stream)."""
    count = int(count)
    if count > 4 * (1 << 32):
        raise ValueError("a counter word addresses at most 2^32 Philox blocks")
    nblk = (count + 3) // 4
    out = np.empty(nblk * 4, dtype=np.float64)
    for b0 in range(0, nblk, _CHUNK_BLOCKS):
        j = np.arange(b0, min(nblk, b0 + _CHUNK_BLOCKS), dtype=np.uint64)
        out[4 * b0: 4 * (b0 + len(j))] = _blocks(j, seed, step, layer_id, stream).reshape(-1)
    return out[:count]


def normals_at(k, seed, step, layer_id, stream):
    """z_k for the flat element indices ``k`` (any int array), computed block by block."""
    k = np.asarray(k, dtype=np.uint64)
    z = _blocks(k >> np.uint64(2), seed, step, layer_id, stream)
    return np.take_along_axis(z, (k & np.uint64(3)).astype(np.int64)[..., None], axis=-1)[..., 0]


def noise(rows, cols, std, seed, step, layer_id):
    """Gaussian noise ``std * z`` for a ``[rows, cols]`` buffer; element (a, b) has k = a*cols + b."""
    return float(std) * normals(rows * cols, seed, step, layer_id, NOISE_STREAM).reshape(rows, cols)


def projection(d_out, r, seed, layer_id):
    """P[d_out, r] with N(0, 1/r) entries: P[b, j] = z_{b*r + j} / sqrt(r), stream 1, step 0.

    Random Gaussian projection regenerated from a seed, one per layer (DP-GRAPE page,
    Methodology, "Random Projection over SVD").
    """
    z = normals(d_out * r, seed, 0, layer_id, PROJECTION_STREAM).reshape(d_out, r)
    return z / math.sqrt(r)


def round_to(dtype, x):
    """fp64 values after the storage rounding of ``dtype`` ('f64', 'f32' or 'bf16').

    'f32' is IEEE round-to-nearest-even.  'bf16' first rounds to fp32 and then rounds the fp32
    bits to their top 16 bits, to nearest, ties to even.  Both sides of the parity test use
    this same two-step rounding for P.
    """
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f64":
        return x.copy()
    f = x.astype(np.float32)
    if dtype == "f32":
        return f.astype(np.float64)
    if dtype != "bf16":
        raise ValueError(dtype)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def per_sample_gradient(X_i, dY_i):
    """G_i = X_i^T dY_i: the weight gradient of one sample, ``[d_in, d_out]`` fp64."""
    return np.asarray(X_i, dtype=np.float64).T @ np.asarray(dY_i, dtype=np.float64)


def _gradient_in_clip_space(X_i, dY_i, P):
    G = per_sample_gradient(X_i, dY_i)
    return G if P is None else G @ np.asarray(P, dtype=np.float64)


def per_sample_norm(X_i, dY_i, P=None):
    """||G_i||_F, or ||G_i P||_F in the projected variant."""
    G = _gradient_in_clip_space(X_i, dY_i, P)
    return math.sqrt(float(np.sum(G * G)))


def per_sample_norms(X, dY, P=None):
    """n_i for every sample of X[B,T,d_in], dY[B,T,d_out]; fp64 ``[B]``."""
    return np.array([per_sample_norm(X[i], dY[i], P) for i in range(X.shape[0])])


def clip_factors(norms, C):
    """c_i = 1 if n_i <= C else C / n_i (C = inf never clips)."""
    norms = np.asarray(norms, dtype=np.float64)
    c = np.ones_like(norms)
    clip = norms > C
    c[clip] = float(C) / norms[clip]
    return c


def clipped_sum(X, dY, c, P=None):
    """S = sum_i c_i G_i (or sum_i c_i G_i P), fp64."""
    S = None
    for i in range(X.shape[0]):
        term = float(c[i]) * _gradient_in_clip_space(X[i], dY[i], P)
        S = term if S is None else S + term
    return S


def clipped_sum_entries(X, dY, c, rows, cols, P=None):
    """Selected entries S[rows[q], cols[q]] of the clipped sum, each computed on its own."""
    rows = np.asarray(rows, dtype=np.int64)
    cols = np.asarray(cols, dtype=np.int64)
    out = np.zeros(rows.shape, dtype=np.float64)
    for q in range(rows.size):
        a, b = int(rows.flat[q]), int(cols.flat[q])
        total = 0.0
        for i in range(X.shape[0]):
            x_col = np.asarray(X[i][:, a], dtype=np.float64)          # x_{t,a}, t < T
            if P is None:
                dy_col = np.asarray(dY[i][:, b], dtype=np.float64)    # dy_{t,b}
            else:
                dy_col = np.asarray(dY[i], dtype=np.float64) @ np.asarray(P[:, b], dtype=np.float64)
            total += float(c[i]) * float(x_col @ dy_col)
        out.flat[q] = total
    return out


def linear_step(X, dY, C, sigma, seed, step, layer_id, P=None):
    """One privatised step for one linear layer.

    Returns a dict with the per-sample norms, the clip factors, the clipped sum S, the noise
    (std = sigma * C, added once to the sum) and ``out = S + noise``.
    """
    if sigma != 0 and not np.isfinite(C):
        raise ValueError("noise std sigma*C is infinite when C = inf; use sigma = 0")
    norms = per_sample_norms(X, dY, P)
    c = clip_factors(norms, C)
    S = clipped_sum(X, dY, c, P)
    std = float(sigma) * float(C)
    z = noise(S.shape[0], S.shape[1], std, seed, step, layer_id) if sigma != 0 else np.zeros_like(S)
    return {"norms": norms, "c": c, "S": S, "noise": z, "out": S + z}


def block_step(layers, C, sigma, seed, step, mode="per_layer"):
    """One privatised step for a block of linear layers that see the same samples.

    ``layers`` is a list of dicts with X [B,T,d_in], dY [B,T,d_out], layer_id, optionally P
    [d_out, r] (the layer is then clipped, summed and noised in the projected space, as in
    ``linear_step``), and, for per-layer clipping, C (the layer's bound; ``C`` is then ignored).
    * mode "per_layer": each layer is clipped with its own bound, as in ``linear_step``
      (FlashDP Abstract: per-layer clipped DP-SGD).
    * mode "flat": one clip factor per sample for the whole block,
      c_i = min(1, C / sqrt(sum_l n_{i,l}^2)), i.e. the sample's gradient over all the
      block's weights is clipped as one vector; every layer's noise has std sigma * C.
    Returns {"layers": [per-layer dicts like linear_step], "flat_norms": [B] or None}.
    """
    if mode == "per_layer":
        return {"layers": [linear_step(l["X"], l["dY"], l["C"], sigma, seed, step, l["layer_id"], l.get("P"))
                           for l in layers], "flat_norms": None}
    if mode != "flat":
        raise ValueError(mode)
    if sigma != 0 and not np.isfinite(C):
        raise ValueError("noise std sigma*C is infinite when C = inf; use sigma = 0")
    per_layer_norms = [per_sample_norms(l["X"], l["dY"], l.get("P")) for l in layers]
    flat = np.sqrt(np.sum(np.stack(per_layer_norms) ** 2, axis=0))
    c = clip_factors(flat, C)
    out = []
    for l, n_l in zip(layers, per_layer_norms):
        S = clipped_sum(l["X"], l["dY"], c, l.get("P"))
        z = (noise(S.shape[0], S.shape[1], float(sigma) * float(C), seed, step, l["layer_id"])
             if sigma != 0 else np.zeros_like(S))
        out.append({"norms": n_l, "c": c, "S": S, "noise": z, "out": S + z})
    return {"layers": out, "flat_norms": flat}


def projected_adam(W, R, m, v, P, lr, beta1, beta2, eps, grad_scale, t):
    """One projected Adam update (DP-GRAPE page, Methodology, "Projected Optimizer States").

    The optimizer state lives in the projected space: m and v are [d_in, r], like the
    privatised projected gradient R (the noisy clipped sum of R_i = G_i P).  The page gives
    neither the averaging nor the map back to the weights.  The plainest readings are taken:
    the gradient estimate is g = grad_scale * R (grad_scale = 1/B averages over the batch),
    Adam with bias correction at step t >= 1 acts on g, and the r-space update goes back to
    the weights through P^T:
        m <- beta1 m + (1 - beta1) g,    v <- beta2 v + (1 - beta2) g^2,
        U = (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps),
        W <- W - lr U P^T.
    Returns (W, m, v) as new fp64 arrays.
    """
    g = float(grad_scale) * np.asarray(R, dtype=np.float64)
    m = float(beta1) * np.asarray(m, dtype=np.float64) + (1.0 - float(beta1)) * g
    v = float(beta2) * np.asarray(v, dtype=np.float64) + (1.0 - float(beta2)) * g * g
    m_hat = m / (1.0 - float(beta1) ** t)
    v_hat = v / (1.0 - float(beta2) ** t)
    U = m_hat / (np.sqrt(v_hat) + float(eps))
    W = np.asarray(W, dtype=np.float64) - float(lr) * (U @ np.asarray(P, dtype=np.float64).T)
    return W, m, v
