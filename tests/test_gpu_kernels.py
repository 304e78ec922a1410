"""Per-entry-point parity against the fp64 oracle, through the C ABI (needs a B200)."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from sample_gradient_clipping_b200 import _lib, inputs
from tests.gpu_helpers import (NOISE_ABS, TOL, check_clip_decisions, host, rel_fro, rel_max)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    _lib.lib()


@pytest.mark.parametrize("seed,step,layer,stream", [
    (0, 0, 0, 0), (0xFFFFFFFFFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF, 1), (2, 5, 3, 0),
    (0x0123456789ABCDEF, (1 << 32) + 7, 6, 1),
])
def test_philox_words_bit_exact(seed, step, layer, stream):
    nblk = 4099
    got = _lib.dp_philox_blocks(nblk, seed, step, layer, stream).cpu().numpy().view(np.uint32)
    ctr = np.zeros((nblk, 4), dtype=np.uint64)
    ctr[:, 0] = np.arange(nblk)
    ctr[:, 1] = layer & 0xFFFFFFFF
    ctr[:, 2] = step & 0xFFFFFFFF
    ctr[:, 3] = stream
    want = oracle.philox4x32_10(ctr, (seed & 0xFFFFFFFF, seed >> 32))
    assert np.array_equal(got, want)


def _edge_words():
    """Words at every breakpoint of the transform's tables, their neighbours and the extremes:
    x_even where x + 1 = 2^k (1 + j/128) starts a ln-table interval (and its centre), x_odd at
    the start, centre and end of every 1/128-turn sector."""
    xe = {0, 1, 2, 3, 0x7FFFFFFF, 0x80000000, 0xFFFFFFFD, 0xFFFFFFFE, 0xFFFFFFFF}
    for k in (0, 1, 2, 5, 12, 20, 26, 30, 31):
        for j in range(128):
            for num in (2 * j, 2 * j + 1):           # interval start and centre, in 1/256 steps
                v = ((256 + num) << k) // 256 - 1
                for d in (-1, 0, 1):
                    if 0 <= v + d < 1 << 32:
                        xe.add(v + d)
    xo = set()
    for j in range(128):
        for off in (0, 1, (1 << 24) - 1, 1 << 24, (1 << 24) + 1, (1 << 25) - 1):
            xo.add((j << 25) + off)
    return np.array(sorted(xe), np.uint32), np.array(sorted(xo), np.uint32)


def test_box_muller_transform_on_edge_words():
    # The transform alone, on chosen words, against the oracle's fp64 Box-Muller (itself within
    # 1e-13 of 40-digit arithmetic): far tighter than the 1e-6 noise tolerance.
    xe, xo = _edge_words()
    pe, po = np.repeat(xe, xo.size), np.tile(xo, xe.size)
    rng = np.random.default_rng(11)
    pe = np.concatenate([pe, rng.integers(0, 1 << 32, 1 << 20, dtype=np.uint64).astype(np.uint32)])
    po = np.concatenate([po, rng.integers(0, 1 << 32, 1 << 20, dtype=np.uint64).astype(np.uint32)])
    words = torch.from_numpy(np.stack([pe, po], axis=1).view(np.int32)).cuda()
    got = _lib.dp_box_muller(words).cpu().numpy()
    ze, zo = oracle.box_muller(pe, po)
    err = max(np.max(np.abs(got[:, 0] - ze)), np.max(np.abs(got[:, 1] - zo)))
    assert err <= 1e-11, err
    # u1 = 1: radius 0 (the transform returns a radius of 2^-50 there)
    last = np.flatnonzero(pe == 0xFFFFFFFF)
    assert np.all(np.abs(got[last]) <= 1e-14)


@pytest.mark.parametrize("rows,cols", [(1, 1), (3, 5), (64, 32), (257, 520), (1000, 1003), (768, 3072),
                                       (2048, 2052)])   # the last stages the tables in shared memory
@pytest.mark.parametrize("std", [1.0, 0.6 / math.sqrt(7.0)])
def test_noise_on_zero_buffer(rows, cols, std):
    G = torch.zeros(rows, cols, dtype=torch.float32, device="cuda")
    _lib.dp_add_noise(G, std, 77, 3, 5)
    want = oracle.noise(rows, cols, np.float32(std), 77, 3, 5)
    err = np.max(np.abs(host(G) - want))
    assert err <= NOISE_ABS, err


def test_noise_adds_to_existing_values():
    rng = np.random.default_rng(1)
    base = rng.standard_normal((129, 72)).astype(np.float32)
    G = torch.from_numpy(base).cuda()
    _lib.dp_add_noise(G, 0.5, 9, 1, 2)
    want = base.astype(np.float64) + oracle.noise(129, 72, 0.5, 9, 1, 2)
    assert np.max(np.abs(host(G) - want)) <= NOISE_ABS + 2 * np.spacing(np.float32(8.0))


def test_noise_steps_and_layers_are_independent_streams():
    a = torch.zeros(64, 64, device="cuda")
    b = torch.zeros(64, 64, device="cuda")
    _lib.dp_add_noise(a, 1.0, 5, 0, 0)
    _lib.dp_add_noise(b, 1.0, 5, 1, 0)
    assert not torch.equal(a, b)
    c = torch.zeros(64, 64, device="cuda")
    _lib.dp_add_noise(c, 1.0, 5, 0, 0)
    assert torch.equal(a, c)                # the same counters reproduce the same noise


@pytest.mark.parametrize("d_out,r", [(1024, 128), (4096, 128), (24, 16), (40, 8), (3072, 256)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_projection_bit_exact(d_out, r, dtype):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    P = torch.empty(d_out, r, dtype=tdt, device="cuda")
    _lib.dp_projection_matrix(P, 4, 3)
    want = oracle.round_to(dtype, oracle.projection(d_out, r, 4, 3))
    assert np.array_equal(host(P), want)


NORM_SHAPES = [
    # B, T, d_in, d_out: several tiles with ragged tails in every dimension
    (3, 200, 320, 392),
    (2, 64, 128, 256),
    (1, 1, 8, 8),
    (4, 130, 136, 520),
    (2, 257, 264, 136),
    (5, 48, 1024, 64),
]


def _draw(B, T, m, n, dtype="bf16", seed=21, dy_var=None):
    w = inputs.custom("t", B=B, T=T, d_in=m, d_out=n, dtype=dtype, seed=seed, dy_var=dy_var)
    d = inputs.generate(w)
    return d["X"]["in"], d["dY"]["linear"]


@pytest.mark.parametrize("shape", NORM_SHAPES, ids=lambda s: "x".join(map(str, s)))
@pytest.mark.parametrize("method", ["ghost", "explicit", "once"])
def test_norms_bf16(shape, method):
    X, dY = _draw(*shape)
    got = host(_lib.dp_per_sample_norms(X.cuda(), dY.cuda(), method=method))
    want = oracle.per_sample_norms(host(X), host(dY))
    assert rel_max(got, want) <= TOL["bf16"]["norm"], (got, want)


@pytest.mark.parametrize("shape", [(4, 16, 64, 32), (3, 37, 20, 12), (2, 5, 4, 4)])
def test_norms_f32(shape):
    X, dY = _draw(*shape, dtype="f32")
    got = host(_lib.dp_per_sample_norms(X.cuda(), dY.cuda()))
    want = oracle.per_sample_norms(host(X), host(dY))
    assert rel_max(got, want) <= TOL["f32"]["norm"], (got, want)


def test_norms_projected_bf16():
    X, dY = _draw(3, 130, 264, 200)
    P = torch.from_numpy(oracle.round_to("bf16", oracle.projection(200, 64, 8, 2))).to(torch.bfloat16)
    for method in ("ghost", "explicit"):
        got = host(_lib.dp_per_sample_norms(X.cuda(), dY.cuda(), P=P.cuda(), method=method))
        want = oracle.per_sample_norms(host(X), host(dY), host(P))
        assert rel_max(got, want) <= TOL["bf16"]["norm"], (method, got, want)


@pytest.mark.parametrize("shape", [(3, 200, 320, 392), (4, 64, 136, 64), (2, 128, 512, 1024)],
                         ids=lambda s: "x".join(map(str, s)))
def test_clip_accumulate_bf16_two_microbatches(shape):
    X, dY = _draw(*shape)
    X2, dY2 = _draw(*shape, seed=99)
    Xh, dYh, X2h, dY2h = host(X), host(dY), host(X2), host(dY2)
    n1 = oracle.per_sample_norms(Xh, dYh)
    n2 = oracle.per_sample_norms(X2h, dY2h)
    C = float(np.median(np.concatenate([n1, n2])))
    n1f, n2f = n1.astype(np.float32), n2.astype(np.float32)
    G = torch.zeros(shape[2], shape[3], dtype=torch.float32, device="cuda")
    _lib.dp_clip_accumulate(X.cuda(), dY.cuda(), torch.from_numpy(n1f).cuda(), C, G)
    _lib.dp_clip_accumulate(X2.cuda(), dY2.cuda(), torch.from_numpy(n2f).cuda(), C, G)
    want = (oracle.clipped_sum(Xh, dYh, oracle.clip_factors(n1f.astype(np.float64), np.float32(C)))
            + oracle.clipped_sum(X2h, dY2h, oracle.clip_factors(n2f.astype(np.float64), np.float32(C))))
    assert rel_fro(host(G), want) <= TOL["bf16"]["sum"]


def test_clip_accumulate_f32():
    X, dY = _draw(4, 16, 64, 32, dtype="f32")
    Xh, dYh = host(X), host(dY)
    n = oracle.per_sample_norms(Xh, dYh).astype(np.float32)
    C = float(n[1])  # one sample exactly at C (not clipped), the others either side
    G = torch.full((64, 32), 0.25, dtype=torch.float32, device="cuda")
    _lib.dp_clip_accumulate(X.cuda(), dY.cuda(), torch.from_numpy(n).cuda(), C, G)
    want = 0.25 + oracle.clipped_sum(Xh, dYh, oracle.clip_factors(n.astype(np.float64), np.float32(C)))
    assert rel_fro(host(G), want) <= TOL["f32"]["sum"]


def test_norms_zero_sample_and_ghost_equals_explicit():
    X, dY = _draw(3, 100, 136, 264)
    X[1].zero_()
    Xd, dYd = X.cuda(), dY.cuda()
    g = host(_lib.dp_per_sample_norms(Xd, dYd, method="ghost"))
    e = host(_lib.dp_per_sample_norms(Xd, dYd, method="explicit"))
    assert g[1] == 0.0 and e[1] == 0.0
    assert rel_max(np.delete(g, 1), np.delete(e, 1)) <= 1e-4
