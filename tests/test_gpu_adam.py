"""dp_projected_adam_step against the fp64 oracle (DP-GRAPE projected optimizer states)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from sample_gradient_clipping_b200 import _lib
from tests.gpu_helpers import TOL, host, rel_fro, rel_max

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _lib.lib()


@pytest.mark.parametrize("d_in,d_out,r", [(1024, 4096, 128), (264, 392, 64), (4096, 1024, 128)])
def test_projected_adam_three_steps(d_in, d_out, r):
    rng = np.random.default_rng(d_in + r)
    W0 = rng.standard_normal((d_in, d_out)).astype(np.float32)
    P = oracle.round_to("bf16", oracle.projection(d_out, r, 4, 2))
    Pd = torch.from_numpy(P).to(torch.bfloat16).cuda()
    W = torch.from_numpy(W0).cuda()
    m = torch.zeros(d_in, r, device="cuda")
    v = torch.zeros(d_in, r, device="cuda")
    Wo, mo, vo = W0.astype(np.float64), np.zeros((d_in, r)), np.zeros((d_in, r))
    # The C ABI takes fp32 hyperparameters; the oracle gets the same (fp32-rounded) values.
    lr, b1, b2, eps, scale = (float(np.float32(x)) for x in (1e-3, 0.9, 0.999, 1e-8, 1.0 / 64))
    for t in range(1, 4):
        R = (rng.standard_normal((d_in, r)) * 3.0).astype(np.float32)
        W_before = host(W)
        _lib.dp_projected_adam_step(W, torch.from_numpy(R).cuda(), m, v, Pd, lr, t, b1, b2, eps, scale)
        W_before_o = Wo
        Wo, mo, vo = oracle.projected_adam(Wo, R, mo, vo, P, lr, b1, b2, eps, scale, t)
        torch.cuda.synchronize()
        # Normwise: after the first step m mixes signs and some entries cancel towards 0.
        assert rel_fro(host(m), mo) <= 1e-6 and rel_fro(host(v), vo) <= 1e-6, t
        # The weight update lr U P^T goes through bf16 U on the tensor cores.
        assert rel_fro(host(W) - W_before, Wo - W_before_o) <= TOL["bf16"]["sum"], t
        Wo = host(W)          # continue from the device weights (their fp32 rounding is data)


def test_zero_learning_rate_updates_moments_only():
    d_in, d_out, r = 128, 256, 64
    W = torch.randn(d_in, d_out, device="cuda")
    W0 = W.clone()
    R = torch.randn(d_in, r, device="cuda")
    m = torch.zeros(d_in, r, device="cuda")
    v = torch.zeros(d_in, r, device="cuda")
    P = torch.randn(d_out, r, device="cuda").to(torch.bfloat16)
    _lib.dp_projected_adam_step(W, R, m, v, P, 0.0, 1)
    assert torch.equal(W, W0)
    one_minus_b1 = 1.0 - float(np.float32(0.9))      # the defaults, as fp32 reaches them
    one_minus_b2 = 1.0 - float(np.float32(0.999))
    assert torch.allclose(m, one_minus_b1 * R, rtol=1e-6) and torch.allclose(v, one_minus_b2 * R * R, rtol=1e-6)
