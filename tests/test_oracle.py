"""The fp64 oracle against facts outside itself (CPU only)."""
from __future__ import annotations

import importlib.util
import os

import numpy as np
import pytest

import oracle
from oracle import dp_oracle
from tests import oracle_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(dp_oracle)


def test_ghost_identity_projected():
    pins.pin_ghost_identity(dp_oracle, seed=12, projected=True)


def test_philox_matches_scalar_reference():
    rng = np.random.default_rng(0)
    ctr = rng.integers(0, 1 << 32, size=(200, 4), dtype=np.uint64).astype(np.uint32)
    keys = rng.integers(0, 1 << 32, size=(200, 2), dtype=np.uint64)
    for q in range(200):
        got = oracle.philox4x32_10(ctr[q:q + 1], keys[q])[0]
        assert [int(v) for v in got] == pins.philox_scalar(ctr[q], keys[q])


def test_streams_layers_steps_differ():
    a = oracle.normals(64, 1, 0, 0, 0)
    for args in [(1, 1, 0, 0), (1, 0, 1, 0), (1, 0, 0, 1), (2, 0, 0, 0), (1 + (1 << 32), 0, 0, 0)]:
        assert not np.array_equal(a, oracle.normals(64, *args))


def test_clipped_sum_entries_match_full():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((3, 5, 7))
    dY = rng.standard_normal((3, 5, 6))
    P = rng.standard_normal((6, 4))
    c = np.array([0.3, 1.0, 0.7])
    for proj in (None, P):
        S = oracle.clipped_sum(X, dY, c, proj)
        rows = np.array([0, 6, 3, 2])
        cols = np.array([0, 3, 1, 2])
        assert np.allclose(oracle.clipped_sum_entries(X, dY, c, rows, cols, proj), S[rows, cols],
                           rtol=1e-13, atol=1e-13)


def test_linear_step_rejects_infinite_noise():
    X = np.ones((1, 2, 3))
    with pytest.raises(ValueError):
        oracle.linear_step(X, X, np.inf, 1.0, 0, 0, 0)


# ---- planted mistakes: every plausible slip in the oracle must trip at least one pin ----

def _fresh_copy():
    path = os.path.join(os.path.dirname(dp_oracle.__file__), "dp_oracle.py")
    spec = importlib.util.spec_from_file_location("dp_oracle_mutant", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mut_transposed_gradient(m):
    m.per_sample_gradient = lambda X_i, dY_i: np.asarray(dY_i, float).T @ np.asarray(X_i, float)


def _mut_shifted_token(m):
    m.per_sample_gradient = lambda X_i, dY_i: np.asarray(X_i, float)[:-1].T @ np.asarray(dY_i, float)[1:]


def _mut_no_clip(m):
    m.clip_factors = lambda norms, C: np.ones_like(np.asarray(norms, float))


def _mut_clip_by_squared_norm(m):
    orig = m.clip_factors
    m.clip_factors = lambda norms, C: orig(np.asarray(norms, float) ** 2, C)


def _mut_sin_cos_swap(m):
    orig = m.box_muller
    m.box_muller = lambda xe, xo: tuple(reversed(orig(xe, xo)))


def _mut_key_bump_first(m):
    orig_w0 = m.PHILOX_W0

    def bad(counters, key):
        return dp_oracle.philox4x32_10(counters, ((int(key[0]) + orig_w0) & 0xFFFFFFFF, key[1]))
    m.philox4x32_10 = bad


def _mut_u1_without_offset(m):
    def bad(xe, xo):
        u1 = np.maximum(np.asarray(xe, float), 0.5) * 2.0 ** -32
        u2 = np.asarray(xo, float) * 2.0 ** -32
        rad = np.sqrt(-2.0 * np.log(u1))
        return rad * np.cos(2 * np.pi * u2), rad * np.sin(2 * np.pi * u2)
    m.box_muller = bad


def _mut_projection_unscaled(m):
    m.projection = lambda d_out, r, seed, layer_id: m.normals(
        d_out * r, seed, 0, layer_id, m.PROJECTION_STREAM).reshape(d_out, r)


def _mut_project_after_clip(m):
    def bad(X_i, dY_i, P=None):
        return m.math.sqrt(float(np.sum(m.per_sample_gradient(X_i, dY_i) ** 2)))
    m.per_sample_norm = bad


def _mut_noise_scaled_by_sigma_only(m):
    orig = m.noise
    m.noise = lambda rows, cols, std, seed, step, layer_id: orig(rows, cols, 1.0, seed, step, layer_id)


def _mut_bf16_truncates(m):
    orig = m.round_to

    def bad(dtype, x):
        if dtype != "bf16":
            return orig(dtype, x)
        f = np.asarray(x, np.float64).astype(np.float32)
        return (f.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)
    m.round_to = bad


def _mut_flat_without_square(m):
    orig = m.block_step

    def bad(layers, C, sigma, seed, step, mode="per_layer"):
        if mode != "flat":
            return orig(layers, C, sigma, seed, step, mode)
        norms = [m.per_sample_norms(l["X"], l["dY"]) for l in layers]
        flat = np.sum(np.stack(norms), axis=0)            # sum of norms, not of squares
        c = m.clip_factors(flat, C)
        out = [{"norms": n, "c": c, "S": m.clipped_sum(l["X"], l["dY"], c)} for l, n in zip(layers, norms)]
        for o_ in out:
            o_["noise"] = np.zeros_like(o_["S"]); o_["out"] = o_["S"]
        return {"layers": out, "flat_norms": flat}
    m.block_step = bad


def _mut_adam_without_bias_correction(m):
    def bad(W, R, mm, vv, P, lr, beta1, beta2, eps, grad_scale, t):
        g = grad_scale * np.asarray(R, float)
        mm = beta1 * mm + (1 - beta1) * g
        vv = beta2 * vv + (1 - beta2) * g * g
        return np.asarray(W, float) - lr * (mm / (np.sqrt(vv) + eps)) @ np.asarray(P, float).T, mm, vv
    m.projected_adam = bad


def _mut_adam_back_projection_transposed(m):
    orig = m.projected_adam

    def bad(W, R, mm, vv, P, lr, beta1, beta2, eps, grad_scale, t):
        Wn, mm, vv = orig(np.zeros_like(np.asarray(W, float)), R, mm, vv, P, lr, beta1, beta2, eps, grad_scale, t)
        return np.asarray(W, float) + Wn[::-1], mm, vv    # a row-flipped update
    m.projected_adam = bad


def _mut_block_ignores_projection(m):
    orig = m.block_step

    def bad(layers, C, sigma, seed, step, mode="per_layer"):
        return orig([{k: v for k, v in l.items() if k != "P"} for l in layers], C, sigma, seed, step, mode)
    m.block_step = bad


def _mut_block_projection_transposed(m):
    orig = m.block_step

    def bad(layers, C, sigma, seed, step, mode="per_layer"):
        flipped = [dict(l, P=np.asarray(l["P"]).T) if "P" in l else l for l in layers]
        return orig(flipped, C, sigma, seed, step, mode)
    m.block_step = bad


MUTANTS = [
    _mut_transposed_gradient, _mut_shifted_token, _mut_no_clip, _mut_clip_by_squared_norm,
    _mut_sin_cos_swap, _mut_key_bump_first, _mut_u1_without_offset, _mut_projection_unscaled,
    _mut_project_after_clip, _mut_noise_scaled_by_sigma_only, _mut_bf16_truncates,
    _mut_flat_without_square, _mut_adam_without_bias_correction,
    _mut_adam_back_projection_transposed, _mut_block_ignores_projection, _mut_block_projection_transposed,
]

_FAST_PINS = [p for p in pins.ALL_PINS if p is not pins.pin_normal_statistics]


@pytest.mark.parametrize("mutate", MUTANTS, ids=lambda f: f.__name__)
def test_planted_mistake_is_caught(mutate):
    m = _fresh_copy()
    mutate(m)
    caught = []
    for pin in _FAST_PINS + [lambda mm: pins.pin_ghost_identity(mm, projected=True)]:
        try:
            pin(m)
        except (AssertionError, ValueError, IndexError):
            caught.append(getattr(pin, "__name__", "pin"))
    assert caught, f"no pin caught {mutate.__name__}"
