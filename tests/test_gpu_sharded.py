"""The sample-sharded step on one GPU through NCCL (a one-rank process group).

With one rank the all-reduce leaves each sum as it is, so the sharded step must reproduce the
oracle's one-device block step on the same samples: the same norms (1e-3), the same clipped
sums (5e-3 relative Frobenius) and, per element, the same noise.  It must also give what the
block step gives, up to where the noise is rounded (the sharded step adds it in a separate
pass).  This runs the GPU side of the orchestration (library calls on the current stream, NCCL
ordered after them, the noise after the all-reduce); the two-rank logic is covered on CPU
ranks.
"""
import datetime
import math
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from sample_gradient_clipping_b200 import _lib, inputs, sharded
from tests.gpu_helpers import (TOL, check_clip_decisions, host, noise_excess, noise_tolerance, record, rel_fro,
                               rel_max)

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
def test_one_rank_sharded_step_against_oracle(mode):
    w = inputs.Workload("shard", B=4, T=256, dtype="bf16", linears=inputs._block(0, 256, 384),
                        C=1.0 / math.sqrt(7.0), sigma=0.6, seed=9, dy_var="per_layer")
    d = inputs.generate(w)
    X = {k: v.cuda() for k, v in d["X"].items()}
    dY = {k: v.cuda() for k, v in d["dY"].items()}
    C = 1.0
    Cl = float(np.float32(w.C))
    sigma = float(np.float32(w.sigma))

    def layers():
        return [{"X": X[l.x_key], "dY": dY[l.name], "layer_id": l.layer_id, "C": w.C,
                 "G_out": torch.empty(l.d_in, l.d_out, dtype=torch.float32, device="cuda"),
                 "norms_out": torch.empty(w.B, dtype=torch.float32, device="cuda")} for l in w.linears]

    got0, got_n = sharded.sharded_step(layers(), 0.0, w.seed, 3, mode=mode, C=C)
    got1, _ = sharded.sharded_step(layers(), w.sigma, w.seed, 3, mode=mode, C=C)
    want1, want_n, _ = _lib.dp_block_step(layers(), mode=mode, C=C, sigma=w.sigma, seed=w.seed, step=3)
    torch.cuda.synchronize()

    olayers = [{"X": inputs.as_f64(d["X"][l.x_key]), "dY": inputs.as_f64(d["dY"][l.name]),
                "layer_id": l.layer_id, "C": Cl} for l in w.linears]
    ref = oracle.block_step(olayers, C, 0.0, w.seed, 3, mode=mode)
    tol = TOL["bf16"]
    for k, lin in enumerate(w.linears):
        r = ref["layers"][k]
        bound = Cl if mode == "per_layer" else C
        n_err = rel_max(host(got_n[k]), r["norms"])
        s_err = rel_fro(host(got0[k]), r["S"])
        record(f"sharded[{mode}]", lin.name, "norm", n_err, tol["norm"])
        record(f"sharded[{mode}]", lin.name, "sum", s_err, tol["sum"])
        assert n_err <= tol["norm"], (lin.name, n_err)
        if mode == "per_layer":
            check_clip_decisions(host(got_n[k]), r["norms"], bound)
        assert s_err <= tol["sum"], (lin.name, s_err)
        a, b = host(got1[k]), host(got0[k])
        std = sigma * (Cl if mode == "per_layer" else C)
        want = oracle.noise(a.shape[0], a.shape[1], std, w.seed, 3, lin.layer_id)
        err = np.abs((a - b) - want)
        record(f"sharded[{mode}]", lin.name, "noise", noise_excess(a, b, want), 1e-6)
        assert np.all(err <= noise_tolerance(a, b)), (lin.name, float(err.max()))
        # and the one-device block step on the same samples
        assert torch.equal(got_n[k], want_n[k]), k
        assert rel_fro(host(got1[k]), host(want1[k])) <= 1e-6, k
