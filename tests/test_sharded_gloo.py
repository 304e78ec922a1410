"""The sample-sharded step's orchestration on two and three CPU ranks (gloo), with the fp64
oracle as each rank's local compute.

The ranks each hold a contiguous share of the batch, clip and sum their own samples,
all-reduce the sums and add the noise once on every rank.  Every rank must end with the one-device result on the
whole batch: the oracle's step, noise included.  This checks the sharding logic (which
samples, which bound, noise added once, flat norms local to a sample); the GPU path plugs the
CUDA library into the same function.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sample_gradient_clipping_b200 import sharded


class OracleOps:
    """Per-rank compute for the test: the oracle on this rank's samples, torch fp64 out."""

    def local_sum(self, layer, C, seed, step, stream=None):
        X, dY = layer["X"].numpy(), layer["dY"].numpy()
        norms = oracle.per_sample_norms(X, dY)
        G = torch.from_numpy(oracle.clipped_sum(X, dY, oracle.clip_factors(norms, C)))
        layer["G_out"], layer["norms_out"] = G, torch.from_numpy(norms)
        return G

    def local_block_sums(self, layers, C, seed, step, stream=None):
        per = [oracle.per_sample_norms(l["X"].numpy(), l["dY"].numpy()) for l in layers]
        flat = np.sqrt(np.sum(np.stack(per) ** 2, axis=0))
        c = oracle.clip_factors(flat, C)
        outs = []
        for l, n in zip(layers, per):
            l["G_out"] = torch.from_numpy(oracle.clipped_sum(l["X"].numpy(), l["dY"].numpy(), c))
            l["norms_out"] = torch.from_numpy(n)
            outs.append(l["G_out"])
        return outs, torch.from_numpy(flat)

    def add_noise(self, G, std, seed, step, layer_id, stream=None):
        G += torch.from_numpy(oracle.noise(G.shape[0], G.shape[1], std, seed, step, layer_id))


def _batch(B=5, T=6, seed=0):
    rng = np.random.default_rng(seed)
    scale = np.exp(rng.normal(0.0, 1.0, size=(B, 1, 1)))      # some samples clip, some do not
    X = rng.standard_normal((B, T, 8)) * scale
    layers = [{"X": X, "dY": rng.standard_normal((B, T, 6)), "layer_id": 0, "C": 2.0},
              {"X": X, "dY": rng.standard_normal((B, T, 6)), "layer_id": 1, "C": 3.0},
              {"X": rng.standard_normal((B, T, 6)), "dY": rng.standard_normal((B, T, 8)), "layer_id": 2,
               "C": 1.5}]
    return layers


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, mode, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        full = _batch()
        lo, hi = sharded.shard_rows(full[0]["X"].shape[0], rank, world)
        mine = [{"X": torch.from_numpy(l["X"][lo:hi].copy()), "dY": torch.from_numpy(l["dY"][lo:hi].copy()),
                 "layer_id": l["layer_id"], "C": l["C"]} for l in full]
        sums, norms = sharded.sharded_step(mine, sigma=0.8, seed=11, step=4, mode=mode, C=2.5, ops=OracleOps())
        out[rank] = ([s.numpy() for s in sums], [n.numpy() for n in norms], (lo, hi))
        dist.barrier()
    finally:
        dist.destroy_process_group()


# Two ranks split the 5 samples 3 / 2; three ranks 2 / 2 / 1.
@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("mode", ["per_layer", "flat"])
def test_ranks_match_one_device_step(mode, world):
    port = _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank, args=(world, port, mode, out), nprocs=world, join=True, start_method="spawn")
    full = _batch()
    want = oracle.block_step([dict(l) for l in full], 2.5, 0.8, 11, 4, mode=mode)
    covered = []
    for rank in range(world):
        sums, norms, (lo, hi) = out[rank]
        covered.append((lo, hi))
        for k, layer in enumerate(want["layers"]):
            np.testing.assert_allclose(sums[k], layer["out"], rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(norms[k], layer["norms"][lo:hi], rtol=1e-13)
    assert sorted(covered) == sharded_spans(full[0]["X"].shape[0], world)
    # Every rank holds identical noisy sums: the noise was drawn once from the shared counter.
    for rank in range(1, world):
        for a, b in zip(out[0][0], out[rank][0]):
            assert np.array_equal(a, b)


def sharded_spans(B, world):
    return [sharded.shard_rows(B, r, world) for r in range(world)]


def test_shard_rows_cover_the_batch():
    for B in (1, 4, 5, 7):
        for world in (1, 2, 3, 4):
            spans = [sharded.shard_rows(B, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == B
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert max(h - l for l, h in spans) - min(h - l for l, h in spans) <= 1


def test_flat_mode_needs_a_bound():
    with pytest.raises(ValueError):
        sharded.sharded_step([], 1.0, 0, 0, mode="flat", C=None, ops=OracleOps())
    with pytest.raises(ValueError):
        sharded.sharded_step([], 1.0, 0, 0, mode="flat", C=math.inf, ops=OracleOps())
