"""Sample-sharded DP-SGD step over several GPUs, one process per GPU.

Each sample's gradient, norm and clip factor depend on that sample alone, so the batch splits
across ranks with no exchange for the norms.  A step is then:

1. every rank forms the clipped sum of its own samples for every linear, without noise;
2. one fp32 all-reduce (sum) per linear;
3. every rank adds the same Gaussian noise, drawn from the (seed, step, layer) Philox counter,
   to the reduced sum.  The counter is deterministic, so no message carries the noise, and it
   is added exactly once to the global sum, as in the one-GPU step.

The all-reduce of linear l is issued as soon as its sum is enqueued, so it overlaps the next
linear's kernels.  With flat (whole-block) clipping the clip factor of a sample needs only
that sample's norms over the block's linears, which live on the same rank.

``ops`` supplies the per-rank compute.  The default is the CUDA library; there is no CPU
path in the product.  Tests substitute their own ops to check this orchestration on CPU
ranks with the gloo backend.
"""
from __future__ import annotations

import math


class LibraryOps:
    """The per-rank compute of a sharded step: the CUDA library through its C ABI."""

    def __init__(self, method="auto"):
        from . import _lib

        self._lib = _lib
        self.method = method
        self._ws = None   # one workspace, grown to the largest linear seen

    def _workspace(self, X, dY):
        import torch

        B, T, d_in, d_out = (int(v) for v in (X.shape[0], X.shape[1], X.shape[2], dY.shape[2]))
        need = self._lib.workspace_size(B, T, d_in, d_out, 0, self._lib._dtype_code(X), self.method)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=X.device)
        return self._ws

    def local_sum(self, layer, C, seed, step, stream=None):
        """Clipped sum of this rank's samples for one linear (sigma = 0, so no noise)."""
        G, n = self._lib.dp_linear_step(layer["X"], layer["dY"], C, 0.0, seed, step, layer["layer_id"],
                                        method=self.method, norms_out=layer.get("norms_out"),
                                        G_out=layer.get("G_out"), workspace=self._workspace(layer["X"], layer["dY"]),
                                        stream=stream)
        layer["G_out"], layer["norms_out"] = G, n
        return G

    def local_block_sums(self, layers, C, seed, step, stream=None):
        """Flat clipping over the block on this rank's samples, without noise."""
        outs, norms, flat = self._lib.dp_block_step(layers, mode="flat", C=C, sigma=0.0, seed=seed, step=step,
                                                    method=self.method, stream=stream)
        for layer, G, n in zip(layers, outs, norms):
            layer["G_out"], layer["norms_out"] = G, n
        return outs, flat

    def add_noise(self, G, std, seed, step, layer_id, stream=None):
        self._lib.dp_add_noise(G, std, seed, step, layer_id, stream=stream)


def sharded_step(layers, sigma, seed, step, mode="per_layer", C=None, group=None, ops=None, stream=None):
    """One privatised step of a block whose batch is split across the ranks of ``group``.

    ``layers``: this rank's shard, dicts with X [B_r, T, d_in], dY [B_r, T, d_out], layer_id, C
    (per-layer bound) and optional G_out / norms_out.  ``mode``: "per_layer" (each linear its
    own C_l, noise sigma * C_l) or "flat" (bound ``C`` for the whole block, noise sigma * C).
    Every rank returns the same noisy global sums, one per linear, and its own samples' norms.
    """
    import contextlib

    import torch
    import torch.distributed as dist

    if ops is None:
        ops = LibraryOps()
    if mode not in ("per_layer", "flat"):
        raise ValueError(f"unknown clipping mode {mode!r}")
    if mode == "flat" and not (C is not None and C > 0 and math.isfinite(C)):
        raise ValueError("flat clipping needs a finite bound C > 0")
    # NCCL orders a collective after the work already on the *current* stream, so the
    # library calls run on the current stream (``stream``, when given, becomes it).
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        pending = []
        if mode == "per_layer":
            for layer in layers:
                G = ops.local_sum(layer, layer["C"], seed, step)
                pending.append((layer, G, dist.all_reduce(G, group=group, async_op=True), sigma * layer["C"]))
        else:
            outs, _ = ops.local_block_sums(layers, C, seed, step)
            for layer, G in zip(layers, outs):
                pending.append((layer, G, dist.all_reduce(G, group=group, async_op=True), sigma * C))
        results = []
        for layer, G, work, std in pending:
            work.wait()          # NCCL: the current stream waits; gloo: the host waits
            if std != 0.0:
                ops.add_noise(G, std, seed, step, layer["layer_id"])
            results.append(G)
    return results, [layer.get("norms_out") for layer in layers]


def shard_rows(batch, rank, world):
    """The contiguous slice of a batch dimension of size ``batch`` that ``rank`` owns."""
    per, extra = divmod(batch, world)
    start = rank * per + min(rank, extra)
    return start, start + per + (1 if rank < extra else 0)
