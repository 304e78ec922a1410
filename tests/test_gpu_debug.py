"""The checked build (libdpclip_debug.so, -DDPCLIP_DEBUG) on small, well-formed calls.

Its device-side index checks must stay silent on valid input: every call below leaves the
status DP_OK, and the results equal those of the normal build (the checks only guard
accesses; the arithmetic is the same) and match the oracle.  No test feeds the checks an
out-of-range index on purpose.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from sample_gradient_clipping_b200 import _lib, build, inputs
from tests.gpu_helpers import TOL, host, rel_fro, rel_max

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def D():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _lib.lib()
    build.build(debug=True)
    return _lib.debug_lib()


def _status(D, ws):
    with _lib.using(D):
        return _lib.dp_workspace_status(ws)


@pytest.mark.parametrize("method", ["ghost", "explicit", "once"])
def test_debug_build_linear_step(D, method):
    w = inputs.custom("dbg", B=3, T=200, d_in=320, d_out=392, C=0.5, sigma=0.7, seed=61)
    d = inputs.generate(w)
    X, dY = d["X"]["in"].cuda(), d["dY"]["linear"].cuda()
    ws = torch.empty(_lib.workspace_size(3, 200, 320, 392, 0, _lib.DP_BF16, method), dtype=torch.uint8,
                     device="cuda")
    with _lib.using(D):
        G_dbg, n_dbg = _lib.dp_linear_step(X, dY, w.C, w.sigma, w.seed, 2, 0, method=method, workspace=ws)
    assert _status(D, ws) == _lib.DP_OK, D.dp_last_cuda_error()
    G, n = _lib.dp_linear_step(X, dY, w.C, w.sigma, w.seed, 2, 0, method=method)
    torch.cuda.synchronize()
    assert torch.equal(n_dbg, n)
    assert rel_fro(host(G_dbg), host(G)) <= 1e-6
    ref = oracle.linear_step(inputs.as_f64(d["X"]["in"]), inputs.as_f64(d["dY"]["linear"]), np.float32(w.C), 0.0,
                             w.seed, 2, 0)
    assert rel_max(host(n_dbg), ref["norms"]) <= TOL["bf16"]["norm"]


def test_debug_build_block_and_projection(D):
    w = inputs.Workload("dbgblk", B=3, T=256, dtype="bf16", linears=inputs._block(0, 256, 384),
                        C=1.0 / math.sqrt(7.0), sigma=0.6, seed=62, dy_var="per_layer")
    d = inputs.generate(w)
    X = {k: v.cuda() for k, v in d["X"].items()}
    dY = {k: v.cuda() for k, v in d["dY"].items()}

    def layers(P=None):
        return [{"X": X[l.x_key], "dY": dY[l.name], "layer_id": l.layer_id, "C": w.C,
                 "norms_out": torch.empty(w.B, dtype=torch.float32, device="cuda"),
                 **({"P": P[l.name]} if P else {})} for l in w.linears]

    with _lib.using(D):
        P = {l.name: _lib.dp_projection_matrix(torch.empty(l.d_out, 64, dtype=torch.bfloat16, device="cuda"),
                                               w.seed, l.layer_id) for l in w.linears}
    for method in ("ghost", "once"):
        for P_ in (None, P):
            with _lib.using(D):
                outs, norms, _ = _lib.dp_block_step(layers(P_), mode="per_layer", sigma=w.sigma, seed=w.seed,
                                                    step=1, method=method)
            want, want_n, _ = _lib.dp_block_step(layers(P_), mode="per_layer", sigma=w.sigma, seed=w.seed,
                                                 step=1, method=method)
            torch.cuda.synchronize()
            for k in range(len(w.linears)):
                assert torch.equal(norms[k], want_n[k]), (method, k)
                assert rel_fro(host(outs[k]), host(want[k])) <= 1e-6, (method, k)
    # One status read covers every kernel above through the module's debug word.
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    assert _status(D, ws) == _lib.DP_OK, D.dp_last_cuda_error()
