"""Seeded synthetic workloads: shapes, sharing of X, and reproducibility."""
import math

import numpy as np
import torch

from sample_gradient_clipping_b200 import inputs


def test_workload_table():
    w = inputs.WORKLOADS
    assert [l.name for l in w["llama7b_block"].linears] == ["q", "k", "v", "o", "gate", "up", "down"]
    assert w["llama7b_block"].tokens == 16384 and w["llama13b_block"].tokens == 8192
    assert abs(w["llama13b_block"].C - 1 / math.sqrt(7)) < 1e-15
    assert w["roberta_large_projected"].r == 128
    assert [l.layer_id for l in w["llama7b_block"].linears] == list(range(7))


def test_generate_is_reproducible_and_shared():
    w = inputs.custom("t", B=2, T=3, d_in=8, d_out=16, dtype="bf16")
    a = inputs.generate(w)
    b = inputs.generate(w)
    assert a["X"]["in"].dtype == torch.bfloat16 and a["X"]["in"].shape == (2, 3, 8)
    assert torch.equal(a["X"]["in"], b["X"]["in"]) and torch.equal(a["dY"]["linear"], b["dY"]["linear"])


def test_block_draw_order_and_selection():
    # A small stand-in with the 13B block's structure: selection must not change the bits.
    w = inputs.WORKLOADS["llama13b_block"]
    small = inputs.Workload("s", B=4, T=2, dtype="f32", linears=inputs._block(0, 8, 16), C=w.C,
                            sigma=w.sigma, seed=3, dy_var="per_layer", sample_scale="lognormal")
    full = inputs.generate(small)
    part = inputs.generate(small, linears=["up"])
    assert set(part["dY"]) == {"up"} and set(part["X"]) == {"mlp_in"}
    assert torch.equal(full["dY"]["up"], part["dY"]["up"])
    assert torch.equal(full["X"]["mlp_in"], part["X"]["mlp_in"])
    assert np.allclose(full["s"], [7.69768105, 0.07764058, 1.51907082, 0.56678819], atol=1e-7)
    assert full["X"]["mlp_mid"].shape == (4, 2, 16)


def test_as_f64_is_exact():
    t = torch.randn(100).to(torch.bfloat16)
    assert np.array_equal(inputs.as_f64(t), t.float().double().numpy())
