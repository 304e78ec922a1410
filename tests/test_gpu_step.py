"""The fused dp_linear_step against the fp64 oracle on every workload, through the C ABI.

The noise norm sigma*C*sqrt(d_in d_out) dwarfs ||S||, so the clipped sum and the noise are
compared separately:
  (1) the step at sigma = 0 against the oracle's S (and norms);
  (2) the step at sigma > 0 minus the step at sigma = 0 against the oracle's noise, per element.
The full-size Llama-shaped blocks are compared in full too: every norm, every entry of every
linear's clipped sum and every noise element (the oracle forms each G_i with a BLAS matmul,
a few minutes a block on the host cores).
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from sample_gradient_clipping_b200 import _lib, inputs
from tests.gpu_helpers import (NOISE_ABS, TOL, check_clip_decisions, draw, host, noise_excess, noise_tolerance,
                               oracle_projection, record, rel_fro, rel_max)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _lib.lib()


def _f32(x):
    return float(np.float32(x))


def _step(w, lin, X, dY, sigma, method="auto", ws=None):
    return _lib.dp_linear_step(X, dY, w.C, sigma, w.seed, w.step, lin.layer_id, r=w.r,
                               method=method, workspace=ws)


def check_linear(w, lin, data, dev, method="auto", sample_entries=None, check_noise=True, got=None, tag=None):
    """Checks one linear's step against the oracle; ``got`` = (G at sigma 0, norms, G at sigma)
    from a call made elsewhere (the block call), else the linear's own dp_linear_step.
    Every entry of the sum and of the noise is compared unless ``sample_entries`` asks for a
    sample of the sum."""
    tag = tag or f"{w.name}[{method}]"
    tol = TOL[w.dtype]
    Xh = inputs.as_f64(data["X"][lin.x_key])
    dYh = inputs.as_f64(data["dY"][lin.name])
    Xd, dYd = dev["X"][lin.x_key], dev["dY"][lin.name]
    P = oracle_projection(w, lin) if w.r else None
    C = _f32(w.C)

    if got is not None:
        G0, n0, G1 = got
    else:
        G0, n0 = _step(w, lin, Xd, dYd, 0.0, method)
    torch.cuda.synchronize()
    norms = oracle.per_sample_norms(Xh, dYh, P)
    n_err = rel_max(host(n0), norms)
    record(tag, lin.name, "norm", n_err, tol["norm"])
    assert n_err <= tol["norm"], (lin.name, host(n0), norms)
    check_clip_decisions(host(n0), norms, C)
    c = oracle.clip_factors(norms, C)
    if sample_entries is None:
        S = oracle.clipped_sum(Xh, dYh, c, P)
        s_err = rel_fro(host(G0), S)
        del S
    else:
        rng = np.random.default_rng(lin.layer_id)
        rows_n, cols_n = G0.shape
        rows = np.concatenate([[0, rows_n - 1, 0, rows_n - 1], rng.integers(0, rows_n, sample_entries)])
        cols = np.concatenate([[0, 0, cols_n - 1, cols_n - 1], rng.integers(0, cols_n, sample_entries)])
        want = oracle.clipped_sum_entries(Xh, dYh, c, rows, cols, P)
        s_err = rel_fro(host(G0)[rows, cols], want)
    record(tag, lin.name, "sum", s_err, tol["sum"])
    assert s_err <= tol["sum"], (lin.name, s_err)
    if check_noise and w.sigma > 0:
        if got is None:
            G1, n1 = _step(w, lin, Xd, dYd, w.sigma, method)
        torch.cuda.synchronize()
        a, b = host(G1), host(G0)
        std = _f32(w.sigma) * C
        want = oracle.noise(a.shape[0], a.shape[1], std, w.seed, w.step, lin.layer_id)
        fa, fb = a.reshape(-1), b.reshape(-1)
        want = want.reshape(-1)
        err = np.abs((fa - fb) - want)
        tol_n = noise_tolerance(fa, fb)
        record(tag, lin.name, "noise", noise_excess(fa, fb, want), NOISE_ABS)
        bad = np.flatnonzero(err > tol_n)
        assert bad.size == 0, (lin.name, bad.size, [(int(q), fa[q], fb[q], want[q], err[q], tol_n[q])
                                                    for q in bad[:5]])
    return host(n0)


def test_tiny_f32_workload():
    w = inputs.WORKLOADS["tiny_f32"]
    data, dev = draw(w)
    check_linear(w, w.linears[0], data, dev)


@pytest.mark.parametrize("method", ["auto", "explicit", "ghost", "once"])
def test_gpt2_mlp_up_workload(method):
    w = inputs.WORKLOADS["gpt2_mlp_up"]
    data, dev = draw(w)
    check_linear(w, w.linears[0], data, dev, method=method)


@pytest.mark.parametrize("method", ["auto", "ghost", "once"])
def test_roberta_projected_workload(method):
    w = inputs.WORKLOADS["roberta_large_projected"]
    data, dev = draw(w)
    for lin in w.linears:
        check_linear(w, lin, data, dev, method=method)


@pytest.mark.parametrize("method", ["auto", "ghost"])
def test_roberta_projected_block(method):
    """The RoBERTa block in the call the benchmark times: one per-layer dp_block_step over the six
    projected linears (their Z = dY P in one grouped launch, the grouped ghost norms and clipped
    sums split over the tokens), at sigma 0 and sigma; every linear's norms, clipped sum and noise
    are compared with the oracle."""
    w = inputs.WORKLOADS["roberta_large_projected"]
    data, dev = draw(w)
    P = {l.name: _lib.dp_projection_matrix(torch.empty(l.d_out, w.r, dtype=torch.bfloat16, device="cuda"),
                                           w.seed, l.layer_id) for l in w.linears}

    def block(sigma):
        layers = [{"X": dev["X"][l.x_key], "dY": dev["dY"][l.name], "P": P[l.name], "layer_id": l.layer_id,
                   "C": w.C, "norms_out": torch.empty(w.B, dtype=torch.float32, device="cuda")}
                  for l in w.linears]
        outs, norms, _ = _lib.dp_block_step(layers, mode="per_layer", sigma=sigma, seed=w.seed, step=w.step,
                                            method=method)
        return outs, norms

    outs0, norms0 = block(0.0)
    outs1, _ = block(w.sigma)
    for k, lin in enumerate(w.linears):
        check_linear(w, lin, data, dev, method=method, got=(outs0[k], norms0[k], outs1[k]),
                     tag=f"roberta_large_projected[{method}] block")


@pytest.mark.slow
@pytest.mark.parametrize("name,method", [("llama7b_block", "auto"), ("llama13b_block", "auto"),
                                         ("llama13b_block", "ghost")])
def test_llama_block_full_size(name, method):
    """Full-size blocks in the launch configuration the benchmark times: one per-layer
    dp_block_step over the block (auto method: gradients once), at sigma 0 and sigma.  Every
    norm, every entry of every linear's clipped sum and every noise element is compared with
    the oracle, so every output tile of the two-SM kernels at their production shapes is
    checked."""
    w = inputs.WORKLOADS[name]
    data, dev = draw(w)

    def block(sigma):
        layers = [{"X": dev["X"][l.x_key], "dY": dev["dY"][l.name], "layer_id": l.layer_id, "C": w.C,
                   "norms_out": torch.empty(w.B, dtype=torch.float32, device="cuda")} for l in w.linears]
        outs, norms, _ = _lib.dp_block_step(layers, mode="per_layer", sigma=sigma, seed=w.seed, step=w.step,
                                            method=method)
        return outs, norms

    outs0, norms0 = block(0.0)
    outs1, _ = block(w.sigma)
    for k, lin in enumerate(w.linears):
        norms = check_linear(w, lin, data, dev, method=method, got=(outs0[k], norms0[k], outs1[k]),
                             tag=f"{name}[{method}] block, full size")
        if name == "llama13b_block":
            # s_i ~ LogNormal(0,1) makes samples 0 and 2 clip and 1 and 3 pass unclipped.
            assert list(norms > w.C) == [True, False, True, False], norms


# ------------------------------------------------------------------------------ edge cases

def _custom(B, T, m, n, dtype="bf16", **kw):
    w = inputs.custom("edge", B=B, T=T, d_in=m, d_out=n, dtype=dtype, **kw)
    data, dev = draw(w)
    return w, w.linears[0], data, dev


# (3, 200, 128, 1000) and (3, 200, 1000, 128): 9 ghost units, fewer than the SMs, with one Gram
# eight times the other's depth, so every unit is cut in two over the deeper Gram's K (ragged
# last K block and ragged T included).
@pytest.mark.parametrize("B,T,m,n", [(1, 1, 8, 8), (3, 200, 320, 392), (2, 257, 264, 136),
                                     (7, 64, 1024, 128), (1, 4096, 128, 128),
                                     (3, 200, 128, 1000), (3, 200, 1000, 128)])
@pytest.mark.parametrize("method", ["ghost", "explicit", "once"])
def test_ragged_shapes(B, T, m, n, method):
    w, lin, data, dev = _custom(B, T, m, n, C=0.5, sigma=0.7, seed=31)
    check_linear(w, lin, data, dev, method=method)


def test_ragged_shapes_f32():
    w, lin, data, dev = _custom(3, 37, 20, 12, dtype="f32", C=0.5, sigma=0.7, seed=32)
    check_linear(w, lin, data, dev)


@pytest.mark.parametrize("method", ["ghost", "explicit", "once"])
def test_zero_sample_is_unclipped_and_adds_nothing(method):
    w, lin, data, dev = _custom(4, 96, 136, 200, C=0.05, sigma=0.0, seed=33)
    data["X"]["in"][2].zero_()
    dev["X"]["in"][2].zero_()
    norms = check_linear(w, lin, data, dev, method=method)
    assert norms[2] == 0.0


@pytest.mark.parametrize("method", ["ghost", "once"])
def test_no_clipping_gives_the_plain_batch_gradient(method):
    w, lin, data, dev = _custom(5, 120, 256, 392, C=math.inf, sigma=0.0, seed=34)
    G, _ = _step(w, lin, dev["X"]["in"], dev["dY"]["linear"], 0.0, method)
    Xh = inputs.as_f64(data["X"]["in"]).reshape(-1, 256)
    dYh = inputs.as_f64(data["dY"]["linear"]).reshape(-1, 392)
    assert rel_fro(host(G), Xh.T @ dYh) <= TOL["bf16"]["sum"]


@pytest.mark.parametrize("method", ["auto", "ghost"])
def test_mixed_clipping_lognormal_scales(method):
    base = inputs.WORKLOADS["llama13b_block"]
    w = inputs.Workload("mixed", B=4, T=256, dtype="bf16", linears=inputs._block(0, 256, 512),
                        C=base.C, sigma=0.6, seed=3, dy_var="per_layer", sample_scale="lognormal")
    data, dev = draw(w)
    for lin in w.linears:
        norms = check_linear(w, lin, data, dev, method=method)
        assert list(norms > w.C) == [True, False, True, False], (lin.name, norms)


def test_split_k_accumulation_path():
    # 1 x 1 output tile over 64 K-blocks: the clipped sum is split across many CTAs.
    w, lin, data, dev = _custom(8, 512, 128, 128, C=0.3, sigma=1.0, seed=35)
    check_linear(w, lin, data, dev)


def test_given_projection_equals_seeded_projection():
    w = inputs.custom("p", B=6, T=64, d_in=256, d_out=512, r=64, C=0.4, sigma=0.0, seed=36)
    data, dev = draw(w)
    lin = w.linears[0]
    X, dY = dev["X"]["in"], dev["dY"]["linear"]
    G_seed, n_seed = _step(w, lin, X, dY, 0.0)
    P = torch.empty(512, 64, dtype=torch.bfloat16, device="cuda")
    _lib.dp_projection_matrix(P, w.seed, lin.layer_id)
    G_given, n_given = _lib.dp_linear_step(X, dY, w.C, 0.0, w.seed, 0, lin.layer_id, P=P)
    assert rel_max(host(n_seed), host(n_given)) <= 1e-5
    assert rel_fro(host(G_seed), host(G_given)) <= 1e-5
    check_linear(w, lin, data, dev)


@pytest.mark.parametrize("B,T,r", [(64, 128, 128),    # 64 row tiles: 128 x 64 projection tiles
                                   (80, 128, 128),    # 80 row tiles: 128 x 128 tiles
                                   (3, 100, 256),     # r > 128: 128 x 256 tiles, ragged N
                                   (5, 72, 40)])      # r < 64: one 64-wide tile, ragged
def test_projection_tile_shapes(B, T, r):
    """Every tile shape of the projection GEMM Z = dY P, checked through the projected step."""
    w = inputs.custom("ptile", B=B, T=T, d_in=256, d_out=512, r=r, C=0.3, sigma=0.9, seed=41)
    data, dev = draw(w)
    check_linear(w, w.linears[0], data, dev, method="ghost")


def test_norms_entry_matches_step_norms():
    w, lin, data, dev = _custom(4, 160, 264, 520, C=0.5, sigma=0.0, seed=37)
    X, dY = dev["X"]["in"], dev["dY"]["linear"]
    _, n_step = _step(w, lin, X, dY, 0.0)
    n_call = _lib.dp_per_sample_norms(X, dY)
    assert rel_max(host(n_call), host(n_step)) <= 1e-5


def test_noise_of_step_k_is_reproducible_in_isolation():
    # The noise is a pure function of (seed, step, layer): a restarted job reproduces step k.
    w, lin, data, dev = _custom(2, 64, 128, 256, C=0.5, sigma=1.0, seed=38)
    X, dY = dev["X"]["in"], dev["dY"]["linear"]
    outs = {}
    for k in range(3):
        G, _ = _lib.dp_linear_step(X, dY, w.C, 1.0, w.seed, k, 0)
        Z, _ = _lib.dp_linear_step(X, dY, w.C, 0.0, w.seed, k, 0)
        outs[k] = host(G) - host(Z)
    G, _ = _lib.dp_linear_step(X, dY, w.C, 1.0, w.seed, 1, 0)
    Z, _ = _lib.dp_linear_step(X, dY, w.C, 0.0, w.seed, 1, 0)
    assert np.max(np.abs((host(G) - host(Z)) - outs[1])) <= 1e-6
    assert not np.allclose(outs[0], outs[1])


def test_workspace_status_is_clean_after_calls():
    w, lin, data, dev = _custom(2, 64, 128, 256, C=0.5, sigma=1.0, seed=39)
    X, dY = dev["X"]["in"], dev["dY"]["linear"]
    ws = torch.empty(_lib.workspace_size(2, 64, 128, 256), dtype=torch.uint8, device="cuda")
    _step(w, lin, X, dY, 1.0, ws=ws)
    assert _lib.dp_workspace_status(ws) == _lib.DP_OK


@pytest.mark.parametrize("method", ["ghost", "explicit", "once"])
def test_norms_and_sums_are_reproducible(method):
    # Norm partials are summed in a fixed order, so reruns give the same bits; without noise,
    # the step's output is reproducible too (no atomics in the unsplit clipped sum or reduce).
    # 16 x 10 output tiles >= the SM count: the clipped sum runs unsplit.
    w, lin, data, dev = _custom(2, 256, 2048, 2560, C=0.2, sigma=0.0, seed=40)
    X, dY = dev["X"]["in"], dev["dY"]["linear"]
    G1, n1 = _step(w, lin, X, dY, 0.0, method)
    G2, n2 = _step(w, lin, X, dY, 0.0, method)
    assert torch.equal(n1, n2)
    assert torch.equal(G1, G2)


@pytest.mark.parametrize("method", ["ghost", "explicit"])
def test_split_k_sums_are_reproducible_with_noise(method):
    # One 128 x 128 output tile over 4096 tokens: the clipped sum is split over K into many
    # parts.  Each part stores its partial sum and one combining launch adds them in split
    # order to the noise already in the output, so reruns give the same bits whatever order
    # the parts ran in, and the result matches the oracle's sum and noise.
    w, lin, data, dev = _custom(8, 512, 128, 128, C=0.3, sigma=1.0, seed=36)
    X, dY = dev["X"]["in"], dev["dY"]["linear"]
    G1, n1 = _step(w, lin, X, dY, w.sigma, method)
    G2, n2 = _step(w, lin, X, dY, w.sigma, method)
    torch.cuda.synchronize()
    assert torch.equal(n1, n2)
    assert torch.equal(G1, G2)
    check_linear(w, lin, data, dev, method=method, tag=f"split-K reproducible[{method}]")
