"""Checks that pin the fp64 oracle to facts outside itself.

Each ``pin_*`` function takes an oracle module (the real one, or a copy with a planted mistake)
and raises AssertionError when the oracle disagrees with the fact the pin encodes.  The facts
come from the mathematics or from published definitions; none is a retyped oracle formula:

* the published Philox4x32-10 known answers (``tests/golden``);
* closed forms of Box-Muller;
* brute force on tiny inputs (an explicit sum of outer products);
* finite differences of a loss that is linear in W;
* the ghost-norm identity;
* library routines (numpy matmul, torch's bf16 rounding);
* invariants of clipping.
"""
from __future__ import annotations

import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_kat():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            w = [int(x, 16) for x in line.split()]
            rows.append((w[0:4], w[4:6], w[6:10]))
    return rows


def philox_scalar(ctr, key):
    """Scalar Philox4x32-10 on Python integers, written separately from the oracle's vector form.

    Salmon et al. (SC'11): S-box = two 32x32 multiplies, P-box = a fixed word permutation,
    key schedule = Weyl sequence.  Constants are repeated here on purpose so that a typo in
    either copy shows up as a disagreement.
    """
    mul = (0xD2511F53, 0xCD9E8D57)
    weyl = (0x9E3779B9, 0xBB67AE85)
    x = [int(v) & 0xFFFFFFFF for v in ctr]
    k = [int(v) & 0xFFFFFFFF for v in key]
    for r in range(10):
        prod_a = mul[0] * x[0]
        prod_b = mul[1] * x[2]
        x = [((prod_b >> 32) ^ x[1] ^ k[0]) & 0xFFFFFFFF,
             prod_b & 0xFFFFFFFF,
             ((prod_a >> 32) ^ x[3] ^ k[1]) & 0xFFFFFFFF,
             prod_a & 0xFFFFFFFF]
        k = [(k[0] + weyl[0]) & 0xFFFFFFFF, (k[1] + weyl[1]) & 0xFFFFFFFF]
    return x


def pin_philox_kat(o):
    for ctr, key, want in load_kat():
        got = o.philox4x32_10(np.array([ctr], dtype=np.uint32), key)[0]
        assert [int(v) for v in got] == want, (ctr, key, [hex(int(v)) for v in got])


def pin_box_muller_closed_forms(o):
    full = 0xFFFFFFFF
    R = math.sqrt(-2.0 * math.log(2.0 ** -32))           # u1 = 2^-32 at x_even = 0
    cases = [
        (full, 0, 0.0, 0.0),                           # u1 = 1: radius 0
        (0, 0, R, 0.0),                                 # angle 0
        (0, 1 << 30, 0.0, R),                           # angle pi/2
        (0, 1 << 31, -R, 0.0),                          # angle pi
        (0, 3 << 30, 0.0, -R),                          # angle 3 pi / 2
    ]
    for xe, xo, want_e, want_o in cases:
        ze, zo = o.box_muller(np.array([xe], np.uint32), np.array([xo], np.uint32))
        assert abs(float(ze[0]) - want_e) <= 1e-14 * max(1.0, R), (xe, xo, ze, want_e)
        assert abs(float(zo[0]) - want_o) <= 1e-14 * max(1.0, R), (xe, xo, zo, want_o)
    # u1 just below 1 must give the small radius sqrt(-2 ln(1 - 2^-32)) exactly enough.
    ze, _ = o.box_muller(np.array([full - 1], np.uint32), np.array([0], np.uint32))
    want = math.sqrt(-2.0 * math.log1p(-(2.0 ** -32)))
    assert abs(float(ze[0]) - want) <= 1e-9 * want, (ze, want)


def pin_box_muller_mpmath(o, n=64, seed=5):
    import mpmath

    mpmath.mp.dps = 40
    rng = np.random.default_rng(seed)
    xe = rng.integers(0, 1 << 32, size=n, dtype=np.uint64).astype(np.uint32)
    xo = rng.integers(0, 1 << 32, size=n, dtype=np.uint64).astype(np.uint32)
    ze, zo = o.box_muller(xe, xo)
    for q in range(n):
        u1 = (mpmath.mpf(int(xe[q])) + 1) / mpmath.mpf(2) ** 32
        u2 = mpmath.mpf(int(xo[q])) / mpmath.mpf(2) ** 32
        rad = mpmath.sqrt(-2 * mpmath.log(u1))
        assert abs(float(rad * mpmath.cos(2 * mpmath.pi * u2)) - ze[q]) < 1e-13
        assert abs(float(rad * mpmath.sin(2 * mpmath.pi * u2)) - zo[q]) < 1e-13


def pin_counter_layout(o):
    seed, step, layer, stream = 0x0123456789ABCDEF, 7, 3, 0
    z = o.normals(37, seed, step, layer, stream)
    key = (seed & 0xFFFFFFFF, seed >> 32)
    for j in range(10):
        x = philox_scalar([j, layer, step, stream], key)
        ze0, zo0 = o.box_muller(np.array([x[0]], np.uint32), np.array([x[1]], np.uint32))
        ze1, zo1 = o.box_muller(np.array([x[2]], np.uint32), np.array([x[3]], np.uint32))
        want = [ze0[0], zo0[0], ze1[0], zo1[0]]
        for q in range(4):
            k = 4 * j + q
            if k < 37:
                assert z[k] == want[q], (k, z[k], want[q])
    k = np.array([0, 5, 36, 17])
    assert np.array_equal(o.normals_at(k, seed, step, layer, stream), z[k])


def pin_gradient_brute_force(o, seed=0):
    rng = np.random.default_rng(seed)
    T, m, n = 5, 4, 3
    X_i = rng.standard_normal((T, m))
    dY_i = rng.standard_normal((T, n))
    G = o.per_sample_gradient(X_i, dY_i)
    want = np.zeros((m, n))
    for t in range(T):
        for a in range(m):
            for b in range(n):
                want[a, b] += X_i[t, a] * dY_i[t, b]
    assert G.shape == (m, n)
    assert np.allclose(G, want, rtol=1e-13, atol=1e-13)


def pin_gradient_finite_difference(o, seed=1):
    """dL/dW for L(W) = <X_i W, dY_i>_F, by central differences (exact: L is linear in W)."""
    rng = np.random.default_rng(seed)
    T, m, n = 6, 5, 4
    X_i = rng.standard_normal((T, m))
    dY_i = rng.standard_normal((T, n))
    W = rng.standard_normal((m, n))

    def loss(Wv):
        return float(np.sum((X_i @ Wv) * dY_i))

    G = o.per_sample_gradient(X_i, dY_i)
    assert G.shape == (m, n)
    for a in range(m):
        for b in range(n):
            E = np.zeros((m, n))
            E[a, b] = 1.0
            fd = (loss(W + E) - loss(W - E)) / 2.0
            assert abs(fd - G[a, b]) <= 1e-9 * max(1.0, abs(fd)), (a, b, fd, G[a, b])


def pin_ghost_identity(o, seed=2, projected=False):
    """n_i^2 = sum_{t,s} (x_t . x_s)(dy_t . dy_s), or with dy replaced by P^T dy."""
    rng = np.random.default_rng(seed)
    B, T, m, n, r = 3, 7, 6, 5, 4
    X = rng.standard_normal((B, T, m))
    dY = rng.standard_normal((B, T, n))
    P = rng.standard_normal((n, r)) if projected else None
    norms = o.per_sample_norms(X, dY, P)
    for i in range(B):
        Z = dY[i] if P is None else dY[i] @ P
        ghost = float(np.sum((X[i] @ X[i].T) * (Z @ Z.T)))
        assert abs(norms[i] ** 2 - ghost) <= 1e-12 * ghost, (i, norms[i] ** 2, ghost)


def pin_clip_invariants(o, seed=3):
    rng = np.random.default_rng(seed)
    B, T, m, n = 5, 4, 6, 3
    X = rng.standard_normal((B, T, m))
    dY = rng.standard_normal((B, T, n)) * np.array([3.0, 0.01, 1.0, 0.2, 5.0])[:, None, None]
    norms = o.per_sample_norms(X, dY)
    C = float(np.median(norms))
    c = o.clip_factors(norms, C)
    for i in range(B):
        G = o.per_sample_gradient(X[i], dY[i])
        assert np.linalg.norm(c[i] * G) <= C * (1 + 1e-12)
        if norms[i] <= C:
            assert c[i] == 1.0
        else:
            assert abs(c[i] * norms[i] - C) <= 1e-12 * C
    # C = inf: the clipped sum is the plain batch gradient X^T dY (library matmul).
    S_inf = o.clipped_sum(X, dY, o.clip_factors(norms, math.inf))
    plain = X.reshape(-1, m).T @ dY.reshape(-1, n)
    assert np.allclose(S_inf, plain, rtol=1e-12, atol=1e-12)
    # Sample order does not matter.
    S = o.clipped_sum(X, dY, c)
    perm = np.array([3, 0, 4, 1, 2])
    S_perm = o.clipped_sum(X[perm], dY[perm], o.clip_factors(o.per_sample_norms(X[perm], dY[perm]), C))
    assert np.allclose(S, S_perm, rtol=1e-12, atol=1e-13)
    # An all-zero sample has norm 0, factor 1 and leaves the sum unchanged.
    Xz = np.concatenate([X, np.zeros((1, T, m))])
    dYz = np.concatenate([dY, rng.standard_normal((1, T, n))])
    nz = o.per_sample_norms(Xz, dYz)
    assert nz[-1] == 0.0
    cz = o.clip_factors(nz, C)
    assert cz[-1] == 1.0
    assert np.allclose(o.clipped_sum(Xz, dYz, cz), S, rtol=1e-12, atol=1e-13)
    # When every sample clips, scaling dY by alpha > 0 leaves the sum unchanged.
    C_small = 0.1 * float(norms.min())
    S1 = o.clipped_sum(X, dY, o.clip_factors(norms, C_small))
    S2 = o.clipped_sum(X, 7.5 * dY, o.clip_factors(o.per_sample_norms(X, 7.5 * dY), C_small))
    assert np.allclose(S1, S2, rtol=1e-12, atol=1e-14)
    # A norm equal to C is not clipped.
    assert o.clip_factors(np.array([2.0, 0.0]), 2.0).tolist() == [1.0, 1.0]


def pin_sigma_zero_deterministic(o, seed=4):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((3, 4, 5))
    dY = rng.standard_normal((3, 4, 6))
    r1 = o.linear_step(X, dY, 0.5, 0.0, 9, 1, 2)
    r2 = o.linear_step(X, dY, 0.5, 0.0, 9, 1, 2)
    assert np.array_equal(r1["out"], r2["out"])
    assert np.array_equal(r1["out"], r1["S"])


def pin_noise_is_added_once(o, seed=6):
    """With sigma > 0 the output minus the clipped sum is sigma*C times stream-0 normals."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((2, 3, 4))
    dY = rng.standard_normal((2, 3, 5))
    C, sigma = 0.7, 1.3
    r = o.linear_step(X, dY, C, sigma, 123, 4, 5)
    z = o.normals(4 * 5, 123, 4, 5, 0).reshape(4, 5)
    assert np.allclose(r["out"] - r["S"], sigma * C * z, rtol=0, atol=1e-14)


def pin_projection(o):
    d_out, r = 24, 16
    P = o.projection(d_out, r, 4, 0)
    assert P.shape == (d_out, r)
    assert np.array_equal(P, o.projection(d_out, r, 4, 0))          # regenerated from the seed
    assert not np.array_equal(P, o.projection(d_out, r, 4, 1))      # one per layer
    assert not np.array_equal(P, o.projection(d_out, r, 5, 0))
    # P = I reduces the variant to the plain step.
    rng = np.random.default_rng(7)
    X = rng.standard_normal((3, 4, 5))
    dY = rng.standard_normal((3, 4, 6))
    c = np.array([0.5, 1.0, 0.25])
    assert np.allclose(o.clipped_sum(X, dY, c, np.eye(6)), o.clipped_sum(X, dY, c), rtol=1e-13, atol=1e-13)
    assert np.allclose(o.per_sample_norms(X, dY, np.eye(6)), o.per_sample_norms(X, dY), rtol=1e-13)
    # Johnson-Lindenstrauss: E ||G P||^2 / ||G||^2 = 1 when P has N(0, 1/r) entries.
    G = rng.standard_normal((8, d_out))
    ratios = [np.sum((G @ o.projection(d_out, r, s, 3)) ** 2) / np.sum(G * G) for s in range(1000)]
    assert abs(np.mean(ratios) - 1.0) <= 3.0 * math.sqrt(2.0 / r) / math.sqrt(1000.0), np.mean(ratios)
    # E[P P^T] = I_{d_out}.
    acc = np.zeros((d_out, d_out))
    for s in range(400):
        Ps = o.projection(d_out, r, s, 9)
        acc += Ps @ Ps.T
    acc /= 400
    assert np.max(np.abs(acc - np.eye(d_out))) < 0.12, np.max(np.abs(acc - np.eye(d_out)))


def pin_normal_statistics(o, n=1_000_000):
    from scipy import stats

    z = o.normals(n, 2024, 0, 0, 0)
    assert abs(z.mean()) < 5.0 / math.sqrt(n)
    assert abs(z.var() - 1.0) < 5.0 * math.sqrt(2.0 / n)
    assert stats.kstest(z, "norm").pvalue > 1e-4
    # Even and odd lanes are independent N(0,1) too.
    assert stats.kstest(z[1::2], "norm").pvalue > 1e-4
    assert abs(np.corrcoef(z[0::2], z[1::2])[0, 1]) < 5.0 / math.sqrt(n / 2)


def pin_bf16_rounding(o):
    import torch

    rng = np.random.default_rng(8)
    f = rng.standard_normal(20000).astype(np.float32)
    # Add exact ties: values whose low 16 bits are 0x8000.
    u = f.view(np.uint32)
    ties = ((u[:2000] & np.uint32(0xFFFF0000)) | np.uint32(0x8000)).view(np.float32)
    f = np.concatenate([f, ties])
    want = torch.from_numpy(f).to(torch.bfloat16).to(torch.float64).numpy()
    got = o.round_to("bf16", f.astype(np.float64))
    assert np.array_equal(got, want)
    assert np.array_equal(o.round_to("f32", f.astype(np.float64)), f.astype(np.float64))


def pin_flat_clipping(o, seed=9):
    """Flat clipping bounds each sample's whole-block gradient by C, and one layer is per-layer."""
    rng = np.random.default_rng(seed)
    B, T = 4, 5
    shapes = [(6, 3), (3, 7), (5, 5)]
    X = [rng.standard_normal((B, T, m)) for m, _ in shapes]
    dY = [rng.standard_normal((B, T, n)) * np.array([2.0, 0.05, 1.0, 0.3])[:, None, None]
          for _, n in shapes]
    layers = [{"X": x, "dY": d, "layer_id": k, "C": 1.0} for k, (x, d) in enumerate(zip(X, dY))]
    C = 1.5
    r = o.block_step(layers, C, 0.0, 1, 0, mode="flat")
    G = [[o.per_sample_gradient(X[k][i], dY[k][i]) for k in range(3)] for i in range(B)]
    for i in range(B):
        whole = np.sqrt(sum(np.sum(g * g) for g in G[i]))          # the sample's block gradient
        assert abs(r["flat_norms"][i] - whole) <= 1e-12 * whole
        c_i = r["layers"][0]["c"][i]
        assert np.sqrt(sum(np.sum((c_i * g) ** 2) for g in G[i])) <= C * (1 + 1e-12)
        assert (c_i == 1.0) == (whole <= C)
    # C = inf: every layer gets its plain batch gradient.
    r_inf = o.block_step(layers, np.inf, 0.0, 1, 0, mode="flat")
    for k in range(3):
        plain = X[k].reshape(-1, shapes[k][0]).T @ dY[k].reshape(-1, shapes[k][1])
        assert np.allclose(r_inf["layers"][k]["S"], plain, rtol=1e-12, atol=1e-12)
    # A block of one layer: flat clipping is per-layer clipping with the same bound.
    one = o.block_step([dict(layers[1], C=C)], C, 0.8, 2, 3, mode="flat")["layers"][0]
    ref = o.linear_step(X[1], dY[1], C, 0.8, 2, 3, 1)
    assert np.allclose(one["out"], ref["out"], rtol=1e-13, atol=1e-13)


def pin_projected_adam(o, seed=10):
    """With P = I the projected update is plain Adam: torch.optim.Adam in fp64 is the reference."""
    import torch

    rng = np.random.default_rng(seed)
    d_in, n = 5, 6
    W0 = rng.standard_normal((d_in, n))
    grads = [rng.standard_normal((d_in, n)) for _ in range(3)]
    lr, b1, b2, eps, scale = 0.01, 0.9, 0.99, 1e-8, 0.25
    p_t = torch.nn.Parameter(torch.tensor(W0))
    opt = torch.optim.Adam([p_t], lr=lr, betas=(b1, b2), eps=eps)
    W, m, v = W0, np.zeros((d_in, n)), np.zeros((d_in, n))
    for t, R in enumerate(grads, start=1):
        p_t.grad = torch.tensor(scale * R)
        opt.step()
        W, m, v = o.projected_adam(W, R, m, v, np.eye(n), lr, b1, b2, eps, scale, t)
        assert np.allclose(W, p_t.detach().numpy(), rtol=1e-12, atol=1e-14), t
    # First step from zero moments: U = g / (|g| + eps), i.e. each weight moves by about lr.
    R = rng.standard_normal((d_in, 3))
    P = rng.standard_normal((n, 3))
    W1, _, _ = o.projected_adam(W0, R, np.zeros_like(R), np.zeros_like(R), P, lr, b1, b2, 0.0, 1.0, 1)
    assert np.allclose(W1, W0 - lr * np.sign(R) @ P.T, rtol=1e-12, atol=1e-12)


def pin_block_projection(o, seed=21):
    """Projected layers in the block step.  With P = 2 Pi (Pi a permutation matrix), G P doubles
    every entry of G and permutes its columns, so each clip-space norm doubles, and with no
    clipping the sum is twice the plain batch gradient (einsum) with its columns permuted."""
    rng = np.random.default_rng(seed)
    B, T = 3, 5
    X = rng.standard_normal((B, T, 6))
    layers = [{"X": X, "dY": rng.standard_normal((B, T, 4)), "layer_id": 0, "C": np.inf},
              {"X": rng.standard_normal((B, T, 5)), "dY": rng.standard_normal((B, T, 7)), "layer_id": 1,
               "C": np.inf}]
    perms = [np.array([2, 0, 3, 1]), np.array([4, 6, 0, 2, 5, 1, 3])]   # not involutions
    for l, pm in zip(layers, perms):
        n = len(pm)
        P = np.zeros((n, n))
        P[pm, np.arange(n)] = 2.0            # column j of G P is 2 * column pm[j] of G
        l["P"] = P
    for mode in ("per_layer", "flat"):
        out = o.block_step(layers, np.inf, 0.0, 0, 0, mode=mode)
        for l, pm, r in zip(layers, perms, out["layers"]):
            G = np.einsum("bta,btc->bac", l["X"], l["dY"])
            assert np.allclose(r["S"], 2.0 * G.sum(axis=0)[:, pm], rtol=1e-12, atol=1e-12), mode
            assert np.allclose(r["norms"], 2.0 * np.sqrt(np.sum(G * G, axis=(1, 2))), rtol=1e-12), mode


ALL_PINS = [
    pin_philox_kat, pin_box_muller_closed_forms, pin_box_muller_mpmath, pin_counter_layout,
    pin_gradient_brute_force, pin_gradient_finite_difference, pin_ghost_identity,
    pin_clip_invariants, pin_sigma_zero_deterministic, pin_noise_is_added_once,
    pin_projection, pin_normal_statistics, pin_bf16_rounding, pin_flat_clipping,
    pin_projected_adam, pin_block_projection,
]
