"""A CUDA graph captured once around the fused step serves every training step.

The step number comes from device memory (dp_linear_step_dev_step, dp_block_step_dev_step):
the graph is captured with a device counter, the counter is advanced between replays, and
each replay must give what an ordinary call with that step gives.
"""
import math

import pytest
import torch

from sample_gradient_clipping_b200 import _lib, inputs
from tests.gpu_helpers import rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _lib.lib()


def _same(a, b, exact):
    if exact:
        return torch.equal(a, b)
    return rel_fro(a.cpu().double().numpy(), b.cpu().double().numpy()) <= 1e-6


@pytest.mark.parametrize("method,r", [("once", 0), ("ghost", 0), ("explicit", 64), ("ghost", 64)])
def test_linear_step_graph_replays_each_step(method, r):
    w = inputs.custom("graph", B=4, T=256, d_in=512, d_out=384, C=0.5, sigma=0.7, seed=21)
    d = inputs.generate(w)
    X, dY = d["X"]["in"].cuda(), d["dY"]["linear"].cuda()
    ws = torch.empty(_lib.workspace_size(4, 256, 512, 384, r, _lib.DP_BF16, method), dtype=torch.uint8,
                     device="cuda")
    G = torch.empty(512, r or 384, dtype=torch.float32, device="cuda")
    n = torch.empty(4, dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    eager = {}
    with torch.cuda.stream(s):
        for k in (3, 4):
            _lib.dp_linear_step(X, dY, w.C, w.sigma, w.seed, k, 5, r=r, method=method, norms_out=n, G_out=G,
                                workspace=ws, stream=s)
            s.synchronize()
            eager[k] = (G.clone(), n.clone())
    step = torch.zeros(1, dtype=torch.int64, device="cuda")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        _lib.dp_linear_step(X, dY, w.C, w.sigma, w.seed, step, 5, r=r, method=method, norms_out=n, G_out=G,
                            workspace=ws, stream=s)
    assert not torch.equal(eager[3][0], eager[4][0])     # the noise moves with the step
    # The clipped sums with split-K accumulate in an unordered way; everything else is exact.
    exact = method == "once"
    for k in (3, 4, 3):
        with torch.cuda.stream(s):
            step.fill_(k)
            g.replay()
        s.synchronize()
        assert torch.equal(n, eager[k][1]), k
        assert _same(G, eager[k][0], exact), k
    assert _lib.dp_workspace_status(ws) == _lib.DP_OK


@pytest.mark.parametrize("method,overlap", [("ghost", "0"), ("once", "0"), ("once", "1")])
def test_block_step_graph_replays_each_step(method, overlap, monkeypatch):
    # overlap "1": the gradients-once reduces run on a second stream, forked and joined in the graph
    monkeypatch.setenv("DPCLIP_OVERLAP_REDUCE", overlap)
    w = inputs.Workload("gblk", B=3, T=256, dtype="bf16", linears=inputs._block(0, 256, 384),
                        C=1.0 / math.sqrt(7.0), sigma=0.6, seed=5, dy_var="per_layer")
    d = inputs.generate(w)
    X = {k: v.cuda() for k, v in d["X"].items()}
    dY = {k: v.cuda() for k, v in d["dY"].items()}
    layers = [{"X": X[l.x_key], "dY": dY[l.name], "layer_id": l.layer_id, "C": w.C,
               "G_out": torch.empty(l.d_in, l.d_out, dtype=torch.float32, device="cuda"),
               "norms_out": torch.empty(w.B, dtype=torch.float32, device="cuda")} for l in w.linears]
    arr = (_lib.DpLayer * len(layers))(*[
        _lib.DpLayer(l["X"].data_ptr(), l["dY"].data_ptr(), l["X"].shape[2], l["dY"].shape[2], l["layer_id"],
                     l["C"], l["G_out"].data_ptr(), l["norms_out"].data_ptr()) for l in layers])
    ws = torch.empty(_lib.lib().dp_block_workspace_size(arr, len(layers), w.B, w.T, _lib.DP_BF16,
                                                         _lib.DP_CLIP_PER_LAYER, _lib.METHODS[method]),
                     dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    eager = {}
    with torch.cuda.stream(s):
        for k in (7, 8):
            _lib.dp_block_step(layers, mode="per_layer", sigma=w.sigma, seed=w.seed, step=k, method=method,
                               workspace=ws, stream=s)
            s.synchronize()
            eager[k] = [l["G_out"].clone() for l in layers]
    step = torch.zeros(1, dtype=torch.int64, device="cuda")
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        _lib.dp_block_step(layers, mode="per_layer", sigma=w.sigma, seed=w.seed, step=step, method=method,
                           workspace=ws, stream=s)
    for k in (8, 7):
        with torch.cuda.stream(s):
            step.fill_(k)
            g.replay()
        s.synchronize()
        for j, l in enumerate(layers):
            assert _same(l["G_out"], eager[k][j], False), (k, j)
