"""The allocation-free norm entry point against the workspace one (needs a B200).

dp_per_sample_norms_static serves callers that cannot allocate device memory: code inside
another framework's allocator hook, or a real-time loop that forbids allocations after
start-up.  Its scratch is a fixed device array inside the library instead of a caller
workspace.  These tests call it through the C ABI and check its norms, on consecutive calls, against
those of dp_per_sample_norms and against the fp64 oracle, within the parity tolerance.  The
calls use different shapes and methods, so stale contents of the shared array would show up.

This file is collected last on purpose: a run that stops at the first failure has then
already run every other test.
"""
from __future__ import annotations

import pytest
import torch

import oracle
from sample_gradient_clipping_b200 import _lib, inputs
from tests.gpu_helpers import TOL, host, record, rel_max

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _lib.lib()


def _draw(B, T, m, n, dtype, seed, with_host=False):
    w = inputs.custom("static", B=B, T=T, d_in=m, d_out=n, dtype=dtype, seed=seed)
    d = inputs.generate(w)
    dev = d["X"]["in"].cuda(), d["dY"]["linear"].cuda()
    return (dev, (d["X"]["in"], d["dY"]["linear"])) if with_host else dev


def _static_norms(X, dY, method):
    B, T, m = X.shape
    n = dY.shape[2]
    out = torch.full((B,), -1.0, dtype=torch.float32, device=X.device)
    code = _lib.DP_BF16 if X.dtype == torch.bfloat16 else _lib.DP_F32
    status = _lib.lib().dp_per_sample_norms_static(
        X.data_ptr(), dY.data_ptr(), code, B, T, m, n, _lib.METHODS[method], out.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert status == _lib.DP_OK, _lib.lib().dp_last_cuda_error()
    return out


CALLS = [  # consecutive calls: shapes and methods change between them
    ((3, 200, 320, 392), "bf16", "explicit"),
    ((5, 64, 512, 256), "bf16", "ghost"),
    ((3, 200, 320, 392), "bf16", "explicit"),
    ((8, 2048, 1024, 512), "bf16", "auto"),
    ((4, 16, 64, 32), "f32", "explicit"),
    ((4, 16, 64, 32), "f32", "explicit"),
]


def test_static_scratch_norms_match_workspace_norms_on_consecutive_calls():
    for k, (shape, dtype, method) in enumerate(CALLS):
        (X, dY), (Xh, dYh) = _draw(*shape, dtype, seed=50 + k, with_host=True)
        want = host(_lib.dp_per_sample_norms(X, dY, method=method))
        got = host(_static_norms(X, dY, method))
        assert rel_max(got, want) <= TOL[dtype]["norm"], (k, shape, method, got, want)
        exact = oracle.per_sample_norms(inputs.as_f64(Xh), inputs.as_f64(dYh))
        err = rel_max(got, exact)
        record("static-scratch norms", f"call {k} {shape} {method}", "norm", err, TOL[dtype]["norm"])
        assert err <= TOL[dtype]["norm"], (k, shape, method, got, exact)


def test_static_scratch_refuses_shapes_beyond_its_size():
    X, dY = _draw(64, 8, 4096, 4096, "bf16", seed=60)   # 64 samples x 16 KB of slots > 1 MiB
    out = torch.empty(64, dtype=torch.float32, device="cuda")
    status = _lib.lib().dp_per_sample_norms_static(
        X.data_ptr(), dY.data_ptr(), _lib.DP_BF16, 64, 8, 4096, 4096, _lib.DP_NORM_EXPLICIT,
        out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert status == _lib.DP_ERR_WORKSPACE
    assert b"fixed array" in _lib.lib().dp_last_cuda_error()
