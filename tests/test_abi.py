"""The C ABI without a GPU: the library loads, exports every declared entry point, sizes its
workspace, and rejects bad arguments on the host before touching the device."""
import math
import os
import re

import pytest

from sample_gradient_clipping_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dpclip.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dp_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert len(names) >= 10
    for name in names:
        assert hasattr(L, name), name
    assert set(names) == set(_lib.SIGNATURES), "binding and header disagree"


def test_status_strings(L):
    for code in range(7):
        assert L.dp_status_string(code) and L.dp_status_string(code) != b"unknown status"
    assert L.dp_status_string(0) == b"ok"


def test_debug_build_compiles_and_exports_every_symbol():
    """The checked variant (-DDPCLIP_DEBUG) builds from the same sources and exports the same
    entry points; its device-side checks are exercised by the GPU tests."""
    path = build.build(debug=True)
    D = _lib.load(path)
    for name in declared_functions():
        assert hasattr(D, name), name
    assert D.dp_status_string(_lib.DP_ERR_DEVICE_CHECK) == b"device-side check failed (debug build)"


def test_workspace_size(L):
    # AUTO picks "once" here: status + norm2 + c + the per-warp norm partials (4 per 128x128
    # tile) + the scaled narrower operand (4096 wide) + the bf16 per-sample tiles.
    ws = L.dp_workspace_size(8, 2048, 4096, 11008, 0, _lib.DP_BF16)
    scaled, tiles = 8 * 2048 * 4096 * 2, 8 * 4096 * 11008 * 2
    partials = 8 * 4 * 32 * 86 * 4
    assert scaled + tiles + partials <= ws < scaled + tiles + partials + 4096
    ghost = L.dp_workspace_size_for(8, 2048, 4096, 11008, 0, _lib.DP_BF16, _lib.DP_NORM_GHOST)
    assert scaled + partials <= ghost < scaled + partials + 4096
    assert L.dp_workspace_size_for(8, 2048, 4096, 11008, 0, _lib.DP_BF16, 9) == 0
    assert L.dp_workspace_size(64, 128, 1024, 1024, 128, _lib.DP_BF16) >= 64 * 128 * 128 * 2 * 2
    assert L.dp_workspace_size(0, 1, 8, 8, 0, _lib.DP_BF16) == 0
    assert L.dp_workspace_size(1, 1, 12, 8, 0, _lib.DP_BF16) == 0     # d_in not a multiple of 8
    assert L.dp_workspace_size(1, 1, 12, 8, 0, _lib.DP_F32) > 0        # fp32 needs multiples of 4


def test_norm_method_environment_override(L):
    try:
        for name in ("ghost", "explicit", "once"):
            os.environ["DPCLIP_NORM"] = name
            assert _lib.auto_norm_method(8, 2048, 4096, 4096) == name
            assert _lib.auto_norm_method(4, 16, 64, 32, dtype_code=_lib.DP_F32) == "explicit"
        os.environ["DPCLIP_NORM"] = "once"      # the workspace query sees the same choice
        assert L.dp_workspace_size(32, 512, 768, 3072, 0, _lib.DP_BF16) == \
            L.dp_workspace_size_for(32, 512, 768, 3072, 0, _lib.DP_BF16, _lib.DP_NORM_ONCE)
        os.environ["DPCLIP_NORM"] = "fastest"   # not a method: the cost model decides
        assert _lib.auto_norm_method(32, 512, 768, 3072) == "ghost"
    finally:
        os.environ.pop("DPCLIP_NORM", None)
    assert _lib.auto_norm_method(8, 2048, 4096, 4096) == "once"


def test_workspace_holds_split_partials(L):
    # GPT-2's 768 x 3072 output fills 36 of 74 SM pairs with 256 x 256 tiles, so its clipped
    # sum is split in two over the tokens and each split's fp32 partial sum gets a slot.
    ghost = L.dp_workspace_size_for(32, 512, 768, 3072, 0, _lib.DP_BF16, _lib.DP_NORM_GHOST)
    scaled = 32 * 512 * 768 * 2                      # the narrower operand, X, scaled in bf16
    partials = 2 * 768 * 3072 * 4
    assert scaled + partials <= ghost < scaled + partials + (1 << 20)
    # The gradients-once layout holds them too, so that it stays the largest.
    once = L.dp_workspace_size_for(32, 512, 768, 3072, 0, _lib.DP_BF16, _lib.DP_NORM_ONCE)
    assert once - ghost == 32 * 768 * 3072 * 2       # plus the bf16 per-sample tiles


def test_auto_method_cost_model(L):
    # Long sequences over wide layers: forming each G_i once beats a second contraction.
    assert _lib.auto_norm_method(8, 2048, 4096, 4096) == "once"
    assert _lib.auto_norm_method(4, 2048, 5120, 13824) == "once"
    # Short sequences: the ghost Grams are nearly free.
    assert _lib.auto_norm_method(64, 16, 4096, 4096) == "ghost"
    # GPT-2 MLP up at T = 512: per-sample tiles over 512 tokens run at half rate, and the ghost
    # step measured 0.138 ms against 0.177 ms for gradients once (CUDA-graph replay).
    assert _lib.auto_norm_method(32, 512, 768, 3072) == "ghost"
    # Very long sequences over narrow layers: the explicit tiles are cheapest.
    assert _lib.auto_norm_method(2, 8192, 64, 64) in ("explicit", "once")
    assert _lib.auto_norm_method(4, 16, 64, 32, 0, _lib.DP_F32) == "explicit"


FAKE = 0x10000          # 16-byte aligned, never dereferenced: every case fails on the host
ODD = FAKE + 4


def _step(L, **kw):
    a = dict(X=FAKE, dY=FAKE, P=None, r=0, dt=_lib.DP_BF16, B=2, T=4, d_in=16, d_out=16, C=1.0,
             sigma=1.0, seed=0, step=0, layer=0, method=0, norms=None, G=FAKE, ws=FAKE,
             ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return L.dp_linear_step(a["X"], a["dY"], a["P"], a["r"], a["dt"], a["B"], a["T"], a["d_in"],
                            a["d_out"], a["C"], a["sigma"], a["seed"], a["step"], a["layer"],
                            a["method"], a["norms"], a["G"], a["ws"], a["ws_bytes"], a["stream"])


@pytest.mark.parametrize("kw,want", [
    (dict(X=None), _lib.DP_ERR_INVALID_ARG),
    (dict(dY=None), _lib.DP_ERR_INVALID_ARG),
    (dict(G=None), _lib.DP_ERR_INVALID_ARG),
    (dict(ws=None), _lib.DP_ERR_INVALID_ARG),
    (dict(X=ODD), _lib.DP_ERR_INVALID_ARG),
    (dict(G=ODD), _lib.DP_ERR_INVALID_ARG),
    (dict(ws=FAKE + 16), _lib.DP_ERR_INVALID_ARG),         # workspace must be 256-byte aligned
    (dict(B=0), _lib.DP_ERR_INVALID_ARG),
    (dict(T=0), _lib.DP_ERR_INVALID_ARG),
    (dict(d_in=12), _lib.DP_ERR_INVALID_ARG),
    (dict(d_out=20), _lib.DP_ERR_INVALID_ARG),
    (dict(dt=7), _lib.DP_ERR_INVALID_ARG),
    (dict(C=0.0), _lib.DP_ERR_INVALID_ARG),
    (dict(C=-1.0), _lib.DP_ERR_INVALID_ARG),
    (dict(C=float("nan")), _lib.DP_ERR_INVALID_ARG),
    (dict(sigma=-0.5), _lib.DP_ERR_INVALID_ARG),
    (dict(sigma=float("inf")), _lib.DP_ERR_INVALID_ARG),
    (dict(C=math.inf, sigma=1.0), _lib.DP_ERR_INVALID_ARG),  # noise std would be infinite
    (dict(P=FAKE, r=0), _lib.DP_ERR_INVALID_ARG),
    (dict(r=12), _lib.DP_ERR_INVALID_ARG),
    (dict(method=9), _lib.DP_ERR_INVALID_ARG),
    (dict(dt=_lib.DP_F32, method=_lib.DP_NORM_GHOST), _lib.DP_ERR_UNSUPPORTED),
    (dict(dt=_lib.DP_F32, method=_lib.DP_NORM_ONCE), _lib.DP_ERR_UNSUPPORTED),
    (dict(ws_bytes=512), _lib.DP_ERR_WORKSPACE),
    (dict(method=_lib.DP_NORM_ONCE, ws_bytes=1024), _lib.DP_ERR_WORKSPACE),   # needs the tiles
    (dict(B=1 << 16, T=1 << 15), _lib.DP_ERR_INVALID_ARG),   # B*T >= 2^31
])
def test_linear_step_rejects_on_host(L, kw, want):
    assert _step(L, **kw) == want


def test_launch_fault_injection_arguments(L):
    E = _lib.DP_ERR_INVALID_ARG
    assert L.dp_selftest_fail_launches(-1, 1, 2) == E
    assert L.dp_selftest_fail_launches(0, -1, 2) == E
    assert L.dp_selftest_fail_launches(0, 1, 0) == E      # an error code is needed
    assert L.dp_selftest_fail_launches(0, 0, 0) == _lib.DP_OK  # clears (nothing pending)


def test_other_entry_points_reject_on_host(L):
    E = _lib.DP_ERR_INVALID_ARG
    assert L.dp_add_noise(None, 4, 4, 1.0, 0, 0, 0, None) == E
    assert L.dp_add_noise(ODD, 4, 4, 1.0, 0, 0, 0, None) == E
    assert L.dp_add_noise(FAKE, 0, 4, 1.0, 0, 0, 0, None) == E
    assert L.dp_add_noise(FAKE, 4, 4, -1.0, 0, 0, 0, None) == E
    assert L.dp_add_noise(FAKE, 4, 4, float("nan"), 0, 0, 0, None) == E
    assert L.dp_add_noise(FAKE, 1 << 20, 1 << 20, 1.0, 0, 0, 0, None) == E   # > 2^34 elements
    assert L.dp_add_noise(FAKE, 4, 4, 0.0, 0, 0, 0, None) == _lib.DP_OK      # std 0: nothing to do
    assert L.dp_projection_matrix(None, _lib.DP_BF16, 16, 8, 0, 0, None) == E
    assert L.dp_projection_matrix(FAKE, _lib.DP_BF16, 16, 12, 0, 0, None) == E
    assert L.dp_projection_matrix(FAKE, 5, 16, 8, 0, 0, None) == E
    assert L.dp_per_sample_norms(FAKE, FAKE, None, 0, _lib.DP_BF16, 2, 4, 16, 16, 0, None, FAKE,
                                 1 << 30, None) == E                          # norms is null
    assert L.dp_per_sample_norms(FAKE, FAKE, None, 8, _lib.DP_BF16, 2, 4, 16, 16, 0, FAKE, FAKE,
                                 1 << 30, None) == E                          # r without P
    assert L.dp_clip_accumulate(FAKE, FAKE, None, 0, _lib.DP_BF16, 2, 4, 16, 16, FAKE, 0.0, FAKE,
                                FAKE, 1 << 30, None) == E                     # C = 0
    assert L.dp_clip_accumulate(FAKE, FAKE, None, 0, _lib.DP_BF16, 2, 4, 16, 16, None, 1.0, FAKE,
                                FAKE, 1 << 30, None) == E                     # norms null
    assert L.dp_workspace_status(None, None) == E


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _lib.lib()


def test_philox_blocks_rejects_on_host(L):
    E = _lib.DP_ERR_INVALID_ARG
    assert L.dp_philox_blocks(None, 4, 0, 0, 0, 0, None) == E
    assert L.dp_philox_blocks(ODD, 4, 0, 0, 0, 0, None) == E
    assert L.dp_philox_blocks(FAKE, 0, 0, 0, 0, 0, None) == E
    assert L.dp_philox_blocks(FAKE, (1 << 32) + 1, 0, 0, 0, 0, None) == E


def test_box_muller_rejects_on_host(L):
    E = _lib.DP_ERR_INVALID_ARG
    assert L.dp_box_muller(None, 4, FAKE, None) == E
    assert L.dp_box_muller(FAKE, 4, None, None) == E
    assert L.dp_box_muller(ODD, 4, FAKE, None) == E
    assert L.dp_box_muller(FAKE, 4, ODD, None) == E
    assert L.dp_box_muller(FAKE, 0, FAKE, None) == E
    assert L.dp_box_muller(FAKE, (1 << 40) + 1, FAKE, None) == E


def test_block_workspace_size_and_host_rejections(L):
    from sample_gradient_clipping_b200._lib import DpLayer
    lay = (DpLayer * 2)(DpLayer(FAKE, FAKE, 4096, 4096, 0, 0.3, FAKE, None),
                        DpLayer(FAKE, FAKE, 4096, 11008, 1, 0.3, FAKE, None))
    per = L.dp_block_workspace_size(lay, 2, 8, 2048, _lib.DP_BF16, 0, _lib.DP_NORM_ONCE)
    flat = L.dp_block_workspace_size(lay, 2, 8, 2048, _lib.DP_BF16, 1, _lib.DP_NORM_ONCE)
    # per-layer mode alternates two tile regions sized for the largest layer (each reduce runs
    # beside the next layer's tensor-core pass); flat once keeps every layer's tiles
    tiles = 8 * 2 * 4096 * 11008
    one = L.dp_workspace_size_for(8, 2048, 4096, 11008, 0, _lib.DP_BF16, _lib.DP_NORM_ONCE)
    assert tiles <= per <= one                       # serial schedule (the default): one region
    os.environ["DPCLIP_OVERLAP_REDUCE"] = "1"        # overlapped reduces: two regions
    try:
        assert 2 * tiles <= L.dp_block_workspace_size(lay, 2, 8, 2048, _lib.DP_BF16, 0, _lib.DP_NORM_ONCE) <= one + tiles
    finally:
        del os.environ["DPCLIP_OVERLAP_REDUCE"]
    assert flat >= 8 * 2 * (4096 * 4096 + 4096 * 11008)
    assert L.dp_block_workspace_size(lay, 2, 8, 2048, _lib.DP_BF16, 7, 0) == 0
    assert L.dp_block_workspace_size(lay, 0, 8, 2048, _lib.DP_BF16, 0, 0) == 0
    E = _lib.DP_ERR_INVALID_ARG
    args = lambda **k: dict(dict(mode=1, C=1.0, sigma=1.0, ws=FAKE, ws_bytes=1 << 40), **k)
    def call(**k):
        a = args(**k)
        return L.dp_block_step(lay, 2, _lib.DP_BF16, 8, 2048, a["mode"], a["C"], a["sigma"], 0, 0, 0,
                               None, a["ws"], a["ws_bytes"], None)
    assert call(mode=5) == E
    assert call(C=0.0) == E
    assert call(C=float("inf")) == E                    # flat noise std would be infinite
    assert call(sigma=-1.0) == E
    assert call(ws=None) == E
    assert call(ws_bytes=4096) == _lib.DP_ERR_WORKSPACE
    bad = (DpLayer * 1)(DpLayer(ODD, FAKE, 64, 64, 0, 1.0, FAKE, None))
    assert L.dp_block_step(bad, 1, _lib.DP_BF16, 2, 4, 1, 1.0, 0.0, 0, 0, 0, None, FAKE, 1 << 30, None) == E
    # A projection width without P, a misaligned P, or a width not a multiple of 8 is refused.
    for P, r in ((None, 64), (ODD, 64), (FAKE, 12)):
        proj = (DpLayer * 1)(DpLayer(FAKE, FAKE, 64, 64, 0, 1.0, FAKE, None, P, r))
        assert L.dp_block_step(proj, 1, _lib.DP_BF16, 2, 4, 0, 1.0, 0.0, 0, 0, 0, None, FAKE, 1 << 30, None) == E
    # With P the workspace also holds Z = dY P (2 x 64 tokens x r bf16), and the scaled copy
    # of the narrower operand is r wide instead of d_out.
    sizes = {}
    for r in (16, 32):
        proj = (DpLayer * 1)(DpLayer(FAKE, FAKE, 64, 64, 0, 1.0, FAKE, None, FAKE, r))
        sizes[r] = L.dp_block_workspace_size(proj, 1, 2, 64, _lib.DP_BF16, 0, _lib.DP_NORM_GHOST)
    assert sizes[32] - sizes[16] == 2 * 128 * 16 * 2


def test_projected_adam_rejects_on_host(L):
    E = _lib.DP_ERR_INVALID_ARG
    assert L.dp_adam_workspace_size(128, 64) == 256 + 128 * 64 * 2
    assert L.dp_adam_workspace_size(128, 12) == 0

    def call(**k):
        a = dict(W=FAKE, dt=_lib.DP_BF16, d_in=128, d_out=256, r=64, lr=1e-3, b1=0.9, b2=0.999,
                 eps=1e-8, t=1, ws=FAKE, ws_bytes=1 << 20)
        a.update(k)
        return L.dp_projected_adam_step(a["W"], FAKE, FAKE, FAKE, FAKE, a["dt"], a["d_in"], a["d_out"],
                                        a["r"], a["lr"], a["b1"], a["b2"], a["eps"], 1.0, a["t"], a["ws"],
                                        a["ws_bytes"], None)
    assert call(W=None) == E
    assert call(W=ODD) == E
    assert call(t=0) == E
    assert call(b1=1.0) == E
    assert call(b2=-0.1) == E
    assert call(lr=-1.0) == E
    assert call(r=12) == E
    assert call(dt=_lib.DP_F32) == _lib.DP_ERR_UNSUPPORTED
    assert call(ws_bytes=100) == _lib.DP_ERR_WORKSPACE


def test_selftest_rejects_on_host(L):
    E = _lib.DP_ERR_INVALID_ARG
    assert L.dp_selftest_wait_timeout(None, 10**6, None) == E
    assert L.dp_selftest_wait_timeout(FAKE + 16, 10**6, None) == E
    assert L.dp_selftest_wait_timeout(FAKE, 10, None) == E              # below 1 us
    assert L.dp_selftest_wait_timeout(FAKE, 10**10, None) == E          # above the 2 s limit


def test_device_step_entry_points_reject_on_host(L):
    E = _lib.DP_ERR_INVALID_ARG
    ws = 1 << 30
    # null and misaligned step addresses are refused before any launch
    for step_ptr in (None, FAKE + 4):
        assert L.dp_linear_step_dev_step(FAKE, FAKE, None, 0, _lib.DP_BF16, 2, 64, 128, 128, 1.0, 0.0, 0,
                                         step_ptr, 0, 0, None, FAKE, FAKE, ws, None) == E
    from sample_gradient_clipping_b200._lib import DpLayer
    lay = (DpLayer * 1)(DpLayer(FAKE, FAKE, 128, 128, 0, 1.0, FAKE, None))
    assert L.dp_block_step_dev_step(lay, 1, _lib.DP_BF16, 2, 64, 0, 1.0, 0.0, 0, None, 0, None, FAKE, ws,
                                    None) == E

