"""The sample-sharded step on one GPU through NCCL (a one-rank process group).

With one rank the all-reduce leaves each sum as it is, so the sharded step must give what the
block step gives on the same samples: the same norms, and the same noisy sums up to where the
noise is rounded (the sharded step adds it in a separate pass).  This runs the GPU side of the
orchestration (library calls on the current stream, NCCL ordered after them, the noise after
the all-reduce); the two-rank logic is covered on CPU ranks.
"""
import datetime
import math
import socket

import pytest
import torch
import torch.distributed as dist

from sample_gradient_clipping_b200 import _lib, inputs, sharded
from tests.gpu_helpers import rel_fro

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _nccl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _lib.lib()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("mode", ["per_layer", "flat"])
def test_one_rank_sharded_step_matches_block_step(mode):
    w = inputs.Workload("shard", B=4, T=256, dtype="bf16", linears=inputs._block(0, 256, 384),
                        C=1.0 / math.sqrt(7.0), sigma=0.6, seed=9, dy_var="per_layer")
    d = inputs.generate(w)
    X = {k: v.cuda() for k, v in d["X"].items()}
    dY = {k: v.cuda() for k, v in d["dY"].items()}
    C = 1.0

    def layers():
        return [{"X": X[l.x_key], "dY": dY[l.name], "layer_id": l.layer_id, "C": w.C,
                 "G_out": torch.empty(l.d_in, l.d_out, dtype=torch.float32, device="cuda"),
                 "norms_out": torch.empty(w.B, dtype=torch.float32, device="cuda")} for l in w.linears]

    got, got_n = sharded.sharded_step(layers(), w.sigma, w.seed, 3, mode=mode, C=C)
    want, want_n, _ = _lib.dp_block_step(layers(), mode=mode, C=C, sigma=w.sigma, seed=w.seed, step=3)
    torch.cuda.synchronize()
    for k in range(len(w.linears)):
        assert torch.equal(got_n[k], want_n[k]), k
        assert rel_fro(got[k].cpu().double().numpy(), want[k].cpu().double().numpy()) <= 1e-6, k
