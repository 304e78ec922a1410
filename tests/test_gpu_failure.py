"""Failure detection on the GPU without a fault: a bounded wait that runs out is reported.

Every in-kernel wait of the library gives up after a limit, records where it gave up in the
workspace's status word and returns.  This test makes such a wait run out on purpose: it
waits on a barrier that nothing arrives at, with a 20 ms limit.  It then checks that the host
reads DP_ERR_TIMEOUT and that the device still runs a normal step correctly afterwards.
"""
import numpy as np
import pytest
import torch

from sample_gradient_clipping_b200 import _lib, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _lib.lib()


def test_bounded_wait_timeout_is_reported_and_device_stays_usable():
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert _lib.lib().dp_selftest_wait_timeout(ws.data_ptr(), 20_000_000, stream) == _lib.DP_OK
    assert _lib.dp_workspace_status(ws) == _lib.DP_ERR_TIMEOUT
    assert int(ws[:4].view(torch.int32).item()) == 99          # the site the wait recorded
    # The context is intact: a normal step runs and its own status is clean.
    w = inputs.custom("after", B=2, T=64, d_in=128, d_out=256, C=0.5, sigma=0.0, seed=3)
    d = inputs.generate(w)
    X, dY = d["X"]["in"].cuda(), d["dY"]["linear"].cuda()
    wsp = torch.empty(_lib.workspace_size(2, 64, 128, 256), dtype=torch.uint8, device="cuda")
    G, n = _lib.dp_linear_step(X, dY, 0.5, 0.0, 3, 0, 0, workspace=wsp)
    assert _lib.dp_workspace_status(wsp) == _lib.DP_OK
    assert torch.isfinite(G).all() and bool((n > 0).all())


def test_refused_launch_is_reported_and_the_next_call_is_whole():
    """Host-side fault injection: a launch the runtime refuses (here as out of memory, through
    the library's fake of the launch call) makes the call return DP_ERR_CUDA with the launch
    named; nothing was enqueued for it, and the next call gives the same bits as a clean run."""
    L = _lib.lib()
    w = inputs.custom("inject", B=2, T=256, d_in=256, d_out=512, C=0.5, sigma=0.7, seed=5)
    d = inputs.generate(w)
    X, dY = d["X"]["in"].cuda(), d["dY"]["linear"].cuda()
    G_ref, n_ref = _lib.dp_linear_step(X, dY, 0.5, 0.7, 5, 1, 0, method="ghost")
    torch.cuda.synchronize()
    for skip in (0, 1, 2):  # the first, second or third kernel launch of the call is refused
        assert L.dp_selftest_fail_launches(skip, 1, 2) == _lib.DP_OK  # 2: cudaErrorMemoryAllocation
        with pytest.raises(_lib.DPError) as err:
            _lib.dp_linear_step(X, dY, 0.5, 0.7, 5, 1, 0, method="ghost")
        assert err.value.status == _lib.DP_ERR_CUDA
        assert b"out of memory" in L.dp_last_cuda_error()
        G, n = _lib.dp_linear_step(X, dY, 0.5, 0.7, 5, 1, 0, method="ghost")
        torch.cuda.synchronize()
        assert torch.equal(n, n_ref) and torch.equal(G, G_ref), skip
    assert L.dp_selftest_fail_launches(0, 0, 0) == _lib.DP_OK
