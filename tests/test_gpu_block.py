"""dp_block_step against the fp64 oracle: per-layer and flat clipping over a block of linears."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from sample_gradient_clipping_b200 import _lib, inputs
from tests.gpu_helpers import (NOISE_ABS, TOL, check_clip_decisions, host, noise_excess, noise_tolerance, record,
                               rel_fro, rel_max)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _lib.lib()


def _block(dtype="bf16", d=256, ffn=512, B=4, T=256, seed=3, lognormal=True):
    w = inputs.Workload("blk", B=B, T=T, dtype=dtype, linears=inputs._block(0, d, ffn),
                        C=1.0 / math.sqrt(7.0), sigma=0.6, seed=seed, dy_var="per_layer",
                        sample_scale="lognormal" if lognormal else "")
    data = inputs.generate(w)
    dev = {"X": {k: v.cuda() for k, v in data["X"].items()},
           "dY": {k: v.cuda() for k, v in data["dY"].items()}}
    return w, data, dev


def _layers(w, dev, C):
    return [{"X": dev["X"][l.x_key], "dY": dev["dY"][l.name], "layer_id": l.layer_id, "C": C,
             "norms_out": torch.empty(w.B, dtype=torch.float32, device="cuda")} for l in w.linears]


def _oracle_layers(w, data, C):
    return [{"X": inputs.as_f64(data["X"][l.x_key]), "dY": inputs.as_f64(data["dY"][l.name]),
             "layer_id": l.layer_id, "C": C} for l in w.linears]


@pytest.mark.parametrize("method", ["auto", "ghost", "explicit", "once"])
def test_flat_clipping_block(method):
    w, data, dev = _block()
    C = float(np.float32(1.0))           # the block's bound: sqrt(7) per-layer bounds of 1/sqrt(7)
    sigma = float(np.float32(w.sigma))
    tol = TOL["bf16"]
    outs0, norms0, flat0 = _lib.dp_block_step(_layers(w, dev, C), mode="flat", C=C, sigma=0.0,
                                              seed=w.seed, step=5, method=method)
    outs1, _, _ = _lib.dp_block_step(_layers(w, dev, C), mode="flat", C=C, sigma=sigma, seed=w.seed,
                                     step=5, method=method)
    torch.cuda.synchronize()
    ref = oracle.block_step(_oracle_layers(w, data, C), C, 0.0, w.seed, 5, mode="flat")
    assert rel_max(host(flat0), ref["flat_norms"]) <= tol["norm"]
    check_clip_decisions(host(flat0), ref["flat_norms"], C)
    # Samples 0 and 2 exceed the block bound, 1 and 3 do not (lognormal scales 7.7, 0.08, 1.5, 0.57).
    assert list(host(flat0) > C) == [True, False, True, False]
    tag = f"block flat [{method}]"
    for k, lin in enumerate(w.linears):
        r = ref["layers"][k]
        n_err, s_err = rel_max(host(norms0[k]), r["norms"]), rel_fro(host(outs0[k]), r["S"])
        record(tag, lin.name, "norm", n_err, tol["norm"])
        record(tag, lin.name, "sum", s_err, tol["sum"])
        assert n_err <= tol["norm"], lin.name
        assert s_err <= tol["sum"], (lin.name, s_err)
        a, b = host(outs1[k]), host(outs0[k])
        want = oracle.noise(a.shape[0], a.shape[1], sigma * C, w.seed, 5, lin.layer_id)
        record(tag, lin.name, "noise", noise_excess(a, b, want), NOISE_ABS)
        assert np.all(np.abs((a - b) - want) <= noise_tolerance(a, b)), lin.name


def test_flat_clipping_block_f32():
    w, data, dev = _block(dtype="f32", d=64, ffn=96, B=3, T=24, seed=8, lognormal=False)
    C = 0.9
    outs, norms, flat = _lib.dp_block_step(_layers(w, dev, C), mode="flat", C=C, sigma=0.0, seed=1)
    ref = oracle.block_step(_oracle_layers(w, data, C), np.float32(C), 0.0, 1, 0, mode="flat")
    assert rel_max(host(flat), ref["flat_norms"]) <= TOL["f32"]["norm"]
    for k in range(len(w.linears)):
        assert rel_fro(host(outs[k]), ref["layers"][k]["S"]) <= TOL["f32"]["sum"]


def test_per_layer_block_equals_linear_steps():
    w, data, dev = _block(seed=4)
    C = 1.0 / math.sqrt(7.0)
    outs, norms, _ = _lib.dp_block_step(_layers(w, dev, C), mode="per_layer", sigma=w.sigma, seed=w.seed,
                                        step=2)
    for k, lin in enumerate(w.linears):
        G, n = _lib.dp_linear_step(dev["X"][lin.x_key], dev["dY"][lin.name], C, w.sigma, w.seed, 2,
                                   lin.layer_id)
        assert torch.equal(n, norms[k]), lin.name
        assert rel_fro(host(outs[k]), host(G)) <= 1e-6, lin.name


@pytest.mark.parametrize("sigma", [0.0, 0.6])
def test_overlapped_reduces_equal_serial_order(sigma, monkeypatch):
    """Per-layer gradients-once block: each reduce runs on a second stream beside the next
    layer's tensor-core pass, in a different layer order, with alternating tile regions.  The
    results must be bitwise those of the serial schedule (DPCLIP_OVERLAP_REDUCE=0)."""
    w, data, dev = _block(seed=6)
    C = 1.0 / math.sqrt(7.0)
    monkeypatch.setenv("DPCLIP_OVERLAP_REDUCE", "1")
    outs_o, norms_o, _ = _lib.dp_block_step(_layers(w, dev, C), mode="per_layer", sigma=sigma, seed=w.seed,
                                            step=3, method="once")
    monkeypatch.setenv("DPCLIP_OVERLAP_REDUCE", "0")
    outs_s, norms_s, _ = _lib.dp_block_step(_layers(w, dev, C), mode="per_layer", sigma=sigma, seed=w.seed,
                                            step=3, method="once")
    torch.cuda.synchronize()
    for k, lin in enumerate(w.linears):
        assert torch.equal(norms_o[k], norms_s[k]), lin.name
        assert torch.equal(outs_o[k], outs_s[k]), lin.name
    ref = oracle.block_step(_oracle_layers(w, data, C), C, 0.0, w.seed, 3, mode="per_layer")
    if sigma == 0:
        for k, lin in enumerate(w.linears):
            assert rel_fro(host(outs_o[k]), ref["layers"][k]["S"]) <= TOL["bf16"]["sum"], lin.name


@pytest.mark.slow
def test_flat_clipping_llama7b_block_full():
    """Flat clipping over the full 7B block, every entry of every linear's sum compared."""
    w = inputs.WORKLOADS["llama7b_block"]
    data = inputs.generate(w)
    dev = {"X": {k: v.cuda() for k, v in data["X"].items()},
           "dY": {k: v.cuda() for k, v in data["dY"].items()}}
    C = 1.0
    outs, norms, flat = _lib.dp_block_step(_layers(w, dev, C), mode="flat", C=C, sigma=0.0, seed=w.seed)
    torch.cuda.synchronize()
    olayers = _oracle_layers(w, data, C)
    n_layers = [oracle.per_sample_norms(l["X"], l["dY"]) for l in olayers]
    flat_ref = np.sqrt(np.sum(np.stack(n_layers) ** 2, axis=0))
    assert rel_max(host(flat), flat_ref) <= TOL["bf16"]["norm"]
    record("llama7b_block flat, full size", "flat", "norm", rel_max(host(flat), flat_ref), TOL["bf16"]["norm"])
    c = oracle.clip_factors(flat_ref, C)
    for k, l in enumerate(olayers):
        n_err = rel_max(host(norms[k]), n_layers[k])
        s_err = rel_fro(host(outs[k]), oracle.clipped_sum(l["X"], l["dY"], c))
        record("llama7b_block flat, full size", w.linears[k].name, "norm", n_err, TOL["bf16"]["norm"])
        record("llama7b_block flat, full size", w.linears[k].name, "sum", s_err, TOL["bf16"]["sum"])
        assert n_err <= TOL["bf16"]["norm"], w.linears[k].name
        assert s_err <= TOL["bf16"]["sum"], (w.linears[k].name, s_err)


@pytest.mark.parametrize("mode", ["per_layer", "flat"])
@pytest.mark.parametrize("shape", ["plain", "tail_split"])
def test_shared_x_gram_ghost_block(mode, shape):
    """q/k/v and gate/up read the same X: one X Gram per group, same norms as one linear at a time.

    tail_split: gate/up (256 -> 1024, B = 5, T = 256) have 15 ghost units, fewer than the SMs, and
    a dY Gram four times the X Gram's depth, so each unit is split in 4 parts over the dY Grams'
    K, in the shared launch and in the one-linear launch alike: the norms stay bitwise equal."""
    if shape == "plain":
        w, data, dev = _block(d=256, ffn=384, B=3, T=384, seed=11)
    else:
        w, data, dev = _block(d=256, ffn=1024, B=5, T=256, seed=13)
    C = 1.0 if mode == "flat" else 1.0 / math.sqrt(7.0)
    _lib.profiling_enable(True)
    _lib.profiling_collect()
    outs, norms, flat = _lib.dp_block_step(_layers(w, dev, C), mode=mode, C=C, sigma=0.0, seed=w.seed, step=1,
                                           method="ghost")
    torch.cuda.synchronize()
    kinds = _lib.profiling_collect()
    _lib.profiling_enable(False)
    # q/k/v share one launch, gate/up another; o and down run the plain ghost kernel: one grouped
    # launch for both in per-layer mode (its batched schedule), one launch each in flat mode.
    assert kinds["umma_ghost_shared"][1] == 2, kinds
    assert kinds["umma_ghost_norm"][1] == (1 if mode == "per_layer" else 2), kinds
    for k, lin in enumerate(w.linears):
        n1 = _lib.dp_per_sample_norms(dev["X"][lin.x_key], dev["dY"][lin.name], method="ghost")
        assert torch.equal(norms[k], n1), lin.name      # same Gram tiles, same partial slots
    ref = oracle.block_step(_oracle_layers(w, data, C), C, 0.0, w.seed, 1, mode=mode)
    tol = TOL["bf16"]
    if mode == "flat":
        assert rel_max(host(flat), ref["flat_norms"]) <= tol["norm"]
    for k, lin in enumerate(w.linears):
        r = ref["layers"][k]
        assert rel_max(host(norms[k]), r["norms"]) <= tol["norm"], lin.name
        assert rel_fro(host(outs[k]), r["S"]) <= tol["sum"], lin.name


def _projected_block(r=64, B=4, T=128, seed=17):
    w = inputs.Workload("pblk", B=B, T=T, dtype="bf16", linears=inputs._block(0, 256, 512),
                        C=1.0, sigma=0.7, seed=seed, dy_var="per_layer")
    data = inputs.generate(w)
    X = {k: v.cuda() for k, v in data["X"].items()}
    dY = {k: v.cuda() for k, v in data["dY"].items()}
    P = {l.name: _lib.dp_projection_matrix(torch.empty(l.d_out, r, dtype=torch.bfloat16, device="cuda"),
                                           w.seed, l.layer_id) for l in w.linears}
    return w, data, X, dY, P


# (r, B, T): the small block forms Z = dY P in 128 x 64 tiles (4 row tiles a linear); the larger ones have
# 24 row tiles per linear, a ragged last one (N = 3000), and 128 x 128 tiles whose columns r = 96
# only partly fill.
@pytest.mark.parametrize("shape", [(64, 4, 128), (128, 6, 500), (96, 6, 500)], ids=["r64", "r128_ragged", "r96_ragged"])
@pytest.mark.parametrize("mode", ["per_layer", "flat"])
def test_projected_block_against_oracle(mode, shape):
    """DP-GRAPE layers in one block call: each clips, sums and noises G_i P; q/k/v and gate/up
    share their X Grams (equal widths r)."""
    r_width, B, T = shape
    w, data, X, dY, P = _projected_block(r=r_width, B=B, T=T)
    C = 0.8
    layers = [{"X": X[l.x_key], "dY": dY[l.name], "P": P[l.name], "layer_id": l.layer_id, "C": C,
               "norms_out": torch.empty(w.B, dtype=torch.float32, device="cuda")} for l in w.linears]
    _lib.profiling_enable(True)
    _lib.profiling_collect()
    outs, norms, flat = _lib.dp_block_step(layers, mode=mode, C=C, sigma=0.0, seed=w.seed, step=2, method="ghost")
    torch.cuda.synchronize()
    kinds = _lib.profiling_collect()
    _lib.profiling_enable(False)
    assert kinds["umma_ghost_shared"][1] == 2, kinds
    olayers = [{"X": inputs.as_f64(data["X"][l.x_key]), "dY": inputs.as_f64(data["dY"][l.name]),
                "P": host(P[l.name]), "layer_id": l.layer_id, "C": C} for l in w.linears]
    ref = oracle.block_step(olayers, C, 0.0, w.seed, 2, mode=mode)
    tol = TOL["bf16"]
    if mode == "flat":
        assert rel_max(host(flat), ref["flat_norms"]) <= tol["norm"]
    for k, lin in enumerate(w.linears):
        r = ref["layers"][k]
        assert outs[k].shape == (lin.d_in, r_width)
        assert rel_max(host(norms[k]), r["norms"]) <= tol["norm"], lin.name
        assert rel_fro(host(outs[k]), r["S"]) <= tol["sum"], lin.name
    # The noise of a projected layer has the [d_in, r] shape and is added once.
    outs1, _, _ = _lib.dp_block_step(layers, mode=mode, C=C, sigma=w.sigma, seed=w.seed, step=2, method="ghost")
    torch.cuda.synchronize()
    for k, lin in enumerate(w.linears):
        a, b = host(outs1[k]), host(outs[k])
        want = oracle.noise(a.shape[0], a.shape[1], float(np.float32(w.sigma)) * float(np.float32(C)), w.seed, 2,
                            lin.layer_id)
        record(f"projected block [{mode}]", lin.name, "noise", noise_excess(a, b, want), NOISE_ABS)
        assert np.all(np.abs((a - b) - want) <= noise_tolerance(a, b)), lin.name


def test_projected_block_with_split_x_grams_against_oracle():
    """Few ghost units (B = 4, one 128-token block) over wide inputs (d = 1024, ffn = 2048): the
    per-layer block step splits each X Gram over K (the shared q/k/v Gram in 2, o in 2, down in 4),
    the single ghost layers run in one grouped launch, and the split partial sums must add up to
    the oracle's norms; the clipped sums and the noise follow them."""
    w = inputs.Workload("psplit", B=4, T=128, dtype="bf16", linears=inputs._block(0, 1024, 2048),
                        C=0.9, sigma=0.8, seed=23, dy_var="per_layer")
    data = inputs.generate(w)
    X = {k: v.cuda() for k, v in data["X"].items()}
    dY = {k: v.cuda() for k, v in data["dY"].items()}
    r = 64
    P = {l.name: _lib.dp_projection_matrix(torch.empty(l.d_out, r, dtype=torch.bfloat16, device="cuda"),
                                           w.seed, l.layer_id) for l in w.linears}
    layers = [{"X": X[l.x_key], "dY": dY[l.name], "P": P[l.name], "layer_id": l.layer_id, "C": w.C,
               "norms_out": torch.empty(w.B, dtype=torch.float32, device="cuda")} for l in w.linears]
    _lib.profiling_enable(True)
    _lib.profiling_collect()
    outs0, norms, _ = _lib.dp_block_step(layers, mode="per_layer", sigma=0.0, seed=w.seed, step=6, method="ghost")
    torch.cuda.synchronize()
    kinds = _lib.profiling_collect()
    _lib.profiling_enable(False)
    assert kinds["umma_ghost_shared"][1] == 2 and kinds["umma_ghost_norm"][1] == 1, kinds
    outs1, _, _ = _lib.dp_block_step(layers, mode="per_layer", sigma=w.sigma, seed=w.seed, step=6, method="ghost")
    torch.cuda.synchronize()
    olayers = [{"X": inputs.as_f64(data["X"][l.x_key]), "dY": inputs.as_f64(data["dY"][l.name]),
                "P": host(P[l.name]), "layer_id": l.layer_id, "C": float(np.float32(w.C))} for l in w.linears]
    ref = oracle.block_step(olayers, None, 0.0, w.seed, 6, mode="per_layer")
    tol = TOL["bf16"]
    for k, lin in enumerate(w.linears):
        rr = ref["layers"][k]
        n_err, s_err = rel_max(host(norms[k]), rr["norms"]), rel_fro(host(outs0[k]), rr["S"])
        record("projected block, split X Grams", lin.name, "norm", n_err, tol["norm"])
        record("projected block, split X Grams", lin.name, "sum", s_err, tol["sum"])
        assert n_err <= tol["norm"], (lin.name, n_err)
        check_clip_decisions(host(norms[k]), rr["norms"], float(np.float32(w.C)))
        assert s_err <= tol["sum"], (lin.name, s_err)
        a, b = host(outs1[k]), host(outs0[k])
        want = oracle.noise(a.shape[0], a.shape[1], float(np.float32(w.sigma)) * float(np.float32(w.C)), w.seed, 6,
                            lin.layer_id)
        record("projected block, split X Grams", lin.name, "noise", noise_excess(a, b, want), NOISE_ABS)
        assert np.all(np.abs((a - b) - want) <= noise_tolerance(a, b)), lin.name


@pytest.mark.parametrize("method", ["ghost", "once", "explicit"])
def test_projected_block_equals_projected_linear_steps(method):
    w, data, X, dY, P = _projected_block(seed=19)
    layers = [{"X": X[l.x_key], "dY": dY[l.name], "P": P[l.name], "layer_id": l.layer_id, "C": 0.5,
               "norms_out": torch.empty(w.B, dtype=torch.float32, device="cuda")} for l in w.linears]
    outs, norms, _ = _lib.dp_block_step(layers, mode="per_layer", sigma=w.sigma, seed=w.seed, step=4,
                                        method=method)
    for k, lin in enumerate(w.linears):
        G, n = _lib.dp_linear_step(X[lin.x_key], dY[lin.name], 0.5, w.sigma, w.seed, 4, lin.layer_id,
                                   P=P[lin.name], method=method)
        assert torch.equal(n, norms[k]), lin.name
        assert rel_fro(host(outs[k]), host(G)) <= 1e-6, lin.name
