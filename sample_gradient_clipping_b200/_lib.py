"""ctypes binding of libdpclip.so: the C ABI of include/dpclip.h, one Python function per entry.

This module only marshals arguments.  It turns torch tensors into device pointers and shapes,
and the current torch stream into a ``cudaStream_t``.  Every step of the computation runs in
the CUDA library.  When the library is missing this module raises; it never falls back to
other code.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libdpclip.so")
# The same library built with -DDPCLIP_DEBUG: device-side index checks (see dp_workspace_status).
DEBUG_LIB_PATH = os.path.join(PKG, "libdpclip_debug.so")

(DP_OK, DP_ERR_INVALID_ARG, DP_ERR_UNSUPPORTED, DP_ERR_WORKSPACE, DP_ERR_CUDA, DP_ERR_TIMEOUT,
 DP_ERR_DEVICE_CHECK) = range(7)
DP_F32, DP_BF16 = 0, 1
DP_NORM_AUTO, DP_NORM_GHOST, DP_NORM_EXPLICIT, DP_NORM_ONCE = 0, 1, 2, 3
METHODS = {"auto": DP_NORM_AUTO, "ghost": DP_NORM_GHOST, "explicit": DP_NORM_EXPLICIT,
           "once": DP_NORM_ONCE}
METHOD_NAMES = {v: k for k, v in METHODS.items()}

_c_void_p, _c_int, _c_float = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_c_size_t, _c_ll, _c_ull, _c_uint = ctypes.c_size_t, ctypes.c_longlong, ctypes.c_ulonglong, ctypes.c_uint

class DpLayer(ctypes.Structure):
    """Mirror of the C struct dp_layer (include/dpclip.h)."""
    _fields_ = [("X", ctypes.c_void_p), ("dY", ctypes.c_void_p), ("d_in", ctypes.c_int),
                ("d_out", ctypes.c_int), ("layer_id", ctypes.c_uint), ("C", ctypes.c_float),
                ("G_out", ctypes.c_void_p), ("norms_out", ctypes.c_void_p), ("P", ctypes.c_void_p),
                ("r", ctypes.c_int)]


DP_CLIP_PER_LAYER, DP_CLIP_FLAT = 0, 1
CLIP_MODES = {"per_layer": DP_CLIP_PER_LAYER, "flat": DP_CLIP_FLAT}

SIGNATURES = {
    "dp_workspace_size": (_c_size_t, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "dp_workspace_size_for": (_c_size_t, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "dp_per_sample_norms": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int,
                                     _c_int, _c_int, _c_int, _c_void_p, _c_void_p, _c_size_t, _c_void_p]),
    "dp_clip_accumulate": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int,
                                    _c_int, _c_int, _c_void_p, _c_float, _c_void_p, _c_void_p,
                                    _c_size_t, _c_void_p]),
    "dp_add_noise": (_c_int, [_c_void_p, _c_ll, _c_ll, _c_float, _c_ull, _c_ull, _c_uint, _c_void_p]),
    "dp_projection_matrix": (_c_int, [_c_void_p, _c_int, _c_int, _c_int, _c_ull, _c_uint, _c_void_p]),
    "dp_linear_step": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int,
                                _c_int, _c_int, _c_float, _c_float, _c_ull, _c_ull, _c_uint, _c_int,
                                _c_void_p, _c_void_p, _c_void_p, _c_size_t, _c_void_p]),
    "dp_linear_step_dev_step": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int,
                                         _c_int, _c_int, _c_float, _c_float, _c_ull, _c_void_p, _c_uint,
                                         _c_int, _c_void_p, _c_void_p, _c_void_p, _c_size_t, _c_void_p]),
    "dp_workspace_status": (_c_int, [_c_void_p, _c_void_p]),
    "dp_selftest_wait_timeout": (_c_int, [_c_void_p, _c_ull, _c_void_p]),
    "dp_selftest_fail_launches": (_c_int, [_c_ll, _c_ll, _c_int]),
    "dp_per_sample_norms_static": (_c_int, [_c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_int,
                                            _c_int, _c_void_p, _c_void_p]),
    "dp_philox_blocks": (_c_int, [_c_void_p, _c_ull, _c_ull, _c_ull, _c_uint, _c_uint, _c_void_p]),
    "dp_box_muller": (_c_int, [_c_void_p, _c_ll, _c_void_p, _c_void_p]),
    "dp_auto_norm_method": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "dp_status_string": (ctypes.c_char_p, [_c_int]),
    "dp_last_cuda_error": (ctypes.c_char_p, []),
    "dp_block_workspace_size": (_c_size_t, [ctypes.POINTER(DpLayer), _c_int, _c_int, _c_int, _c_int,
                                            _c_int, _c_int]),
    "dp_block_step": (_c_int, [ctypes.POINTER(DpLayer), _c_int, _c_int, _c_int, _c_int, _c_int, _c_float,
                               _c_float, _c_ull, _c_ull, _c_int, _c_void_p, _c_void_p, _c_size_t,
                               _c_void_p]),
    "dp_block_step_dev_step": (_c_int, [ctypes.POINTER(DpLayer), _c_int, _c_int, _c_int, _c_int, _c_int,
                                        _c_float, _c_float, _c_ull, _c_void_p, _c_int, _c_void_p, _c_void_p,
                                        _c_size_t, _c_void_p]),
    "dp_adam_workspace_size": (_c_size_t, [_c_int, _c_int]),
    "dp_projected_adam_step": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_int, _c_int,
                                        _c_int, _c_int, _c_float, _c_float, _c_float, _c_float, _c_float,
                                        _c_int, _c_void_p, _c_size_t, _c_void_p]),
    "dp_profiling_enable": (_c_int, [_c_int]),
    "dp_profiling_kinds": (_c_int, []),
    "dp_profiling_kind_name": (ctypes.c_char_p, [_c_int]),
    "dp_profiling_collect": (_c_int, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_c_ll)]),
    "dp_kernel_launches": (_c_ll, []),
}

_lib = None
_debug_lib = None


def load(path):
    """A ctypes handle of the library at ``path`` with every entry point's signature set."""
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with "
            "`python -m sample_gradient_clipping_b200.build` (nvcc, sm_100a)")
    handle = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(handle, name)
        fn.restype = res
        fn.argtypes = args
    return handle


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        _lib = load(LIB_PATH)
    return _lib


def debug_lib():
    """The checked build of the library (libdpclip_debug.so), loaded beside the normal one."""
    global _debug_lib
    if _debug_lib is None:
        _debug_lib = load(DEBUG_LIB_PATH)
    return _debug_lib


class using:
    """Context manager: the functions of this module call ``handle`` (e.g. debug_lib())
    instead of the normal library while it is active."""

    def __init__(self, handle):
        self.handle = handle

    def __enter__(self):
        global _lib
        lib()
        self.saved, _lib = _lib, self.handle
        return self.handle

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


class DPError(RuntimeError):
    def __init__(self, status, what):
        detail = lib().dp_last_cuda_error().decode() if status == DP_ERR_CUDA else ""
        msg = f"{what}: {lib().dp_status_string(status).decode()}"
        super().__init__(msg + (f" ({detail})" if detail else ""))
        self.status = status


def check(status, what):
    if status != DP_OK:
        raise DPError(status, what)


def _dtype_code(t):
    import torch

    if t.dtype == torch.bfloat16:
        return DP_BF16
    if t.dtype == torch.float32:
        return DP_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream):
    import torch

    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _bt_dims(X, dY):
    if X.dim() != 3 or dY.dim() != 3 or X.shape[:2] != dY.shape[:2]:
        raise ValueError("X must be [B, T, d_in] and dY [B, T, d_out]")
    if not (X.is_contiguous() and dY.is_contiguous()):
        raise ValueError("X and dY must be contiguous")
    if X.dtype != dY.dtype:
        raise ValueError("X and dY must share a dtype")
    return int(X.shape[0]), int(X.shape[1]), int(X.shape[2]), int(dY.shape[2])


def workspace_size(B, T, d_in, d_out, r=0, dtype_code=DP_BF16, method="auto"):
    return int(lib().dp_workspace_size_for(B, T, d_in, d_out, r, dtype_code, METHODS[method]))


def _workspace(X, dY, r, workspace, method="auto"):
    import torch

    B, T, d_in, d_out = _bt_dims(X, dY)
    need = workspace_size(B, T, d_in, d_out, r, _dtype_code(X), method)
    if need == 0:
        raise DPError(DP_ERR_INVALID_ARG, "workspace size")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    return workspace


def dp_per_sample_norms(X, dY, P=None, method="auto", norms=None, workspace=None, stream=None):
    """Per-sample norms n_i (fp32 [B]) of X_i^T dY_i [P]."""
    import torch

    B, T, d_in, d_out = _bt_dims(X, dY)
    r = int(P.shape[1]) if P is not None else 0
    ws = _workspace(X, dY, r, workspace)
    if norms is None:
        norms = torch.empty(B, dtype=torch.float32, device=X.device)
    check(lib().dp_per_sample_norms(_ptr(X), _ptr(dY), _ptr(P), r, _dtype_code(X), B, T, d_in, d_out,
                                    METHODS[method], _ptr(norms), _ptr(ws), ws.numel(), _stream(stream)),
          "dp_per_sample_norms")
    return norms


def dp_clip_accumulate(X, dY, norms, C, G_sum, P=None, workspace=None, stream=None):
    """G_sum += sum_i c_i X_i^T dY_i [P] with c_i = min(1, C / norms[i])."""
    B, T, d_in, d_out = _bt_dims(X, dY)
    r = int(P.shape[1]) if P is not None else 0
    ws = _workspace(X, dY, r, workspace)
    check(lib().dp_clip_accumulate(_ptr(X), _ptr(dY), _ptr(P), r, _dtype_code(X), B, T, d_in, d_out,
                                   _ptr(norms), float(C), _ptr(G_sum), _ptr(ws), ws.numel(),
                                   _stream(stream)),
          "dp_clip_accumulate")
    return G_sum


def dp_add_noise(G, std, seed, step, layer_id, stream=None):
    """G += std * z (Philox stream 0 at (seed, step, layer_id)), in place."""
    rows = int(G.shape[0])
    cols = int(G.numel() // max(rows, 1))
    check(lib().dp_add_noise(_ptr(G), rows, cols, float(std), int(seed), int(step), int(layer_id),
                             _stream(stream)),
          "dp_add_noise")
    return G


def dp_projection_matrix(P, seed, layer_id, stream=None):
    """Fills P[d_out, r] with z / sqrt(r) from Philox stream 1 at (seed, layer_id)."""
    check(lib().dp_projection_matrix(_ptr(P), _dtype_code(P), int(P.shape[0]), int(P.shape[1]),
                                     int(seed), int(layer_id), _stream(stream)),
          "dp_projection_matrix")
    return P


def _device_step(step):
    """A device tensor holding the step (int64/uint64, one element), or None for a number."""
    import torch

    if not isinstance(step, torch.Tensor):
        return None
    if step.numel() != 1 or step.dtype not in (torch.int64, torch.uint64) or not step.is_cuda:
        raise ValueError("a device step must be a one-element int64 CUDA tensor")
    return step


def dp_linear_step(X, dY, C, sigma, seed, step, layer_id, P=None, r=0, method="auto",
                   norms_out=None, G_out=None, workspace=None, stream=None):
    """One privatised step; returns (G_out, norms_out).

    ``step`` is a number, or a one-element int64 CUDA tensor read when the kernels run
    (dp_linear_step_dev_step), so that a CUDA graph of this call serves every step.
    """
    import torch

    B, T, d_in, d_out = _bt_dims(X, dY)
    if P is not None:
        r = int(P.shape[1])
    ws = _workspace(X, dY, r, workspace, method)
    width = r if r else d_out
    if G_out is None:
        G_out = torch.empty(d_in, width, dtype=torch.float32, device=X.device)
    if norms_out is None:
        norms_out = torch.empty(B, dtype=torch.float32, device=X.device)
    dstep = _device_step(step)
    if dstep is not None:
        check(lib().dp_linear_step_dev_step(_ptr(X), _ptr(dY), _ptr(P), r, _dtype_code(X), B, T, d_in, d_out,
                                            float(C), float(sigma), int(seed), _ptr(dstep), int(layer_id),
                                            METHODS[method], _ptr(norms_out), _ptr(G_out), _ptr(ws),
                                            ws.numel(), _stream(stream)),
              "dp_linear_step_dev_step")
    else:
        check(lib().dp_linear_step(_ptr(X), _ptr(dY), _ptr(P), r, _dtype_code(X), B, T, d_in, d_out,
                                   float(C), float(sigma), int(seed), int(step), int(layer_id),
                                   METHODS[method], _ptr(norms_out), _ptr(G_out), _ptr(ws), ws.numel(),
                                   _stream(stream)),
              "dp_linear_step")
    return G_out, norms_out


def dp_philox_blocks(nblocks, seed, step, layer_id, stream_id, out=None, device="cuda", stream=None):
    """Raw Philox4x32-10 words [nblocks, 4] (int32 tensor holding the uint32 bits)."""
    import torch

    if out is None:
        out = torch.empty(int(nblocks), 4, dtype=torch.int32, device=device)
    check(lib().dp_philox_blocks(_ptr(out), int(nblocks), int(seed), int(step), int(layer_id),
                                 int(stream_id), _stream(stream)),
          "dp_philox_blocks")
    return out


def dp_box_muller(words, out=None, stream=None):
    """The noise's Box-Muller transform of word pairs: words int32/uint32 [n, 2] on the device
    (the uint32 bits) -> fp64 [n, 2] (z_even, z_odd) before the sigma*C scaling."""
    import torch

    n = int(words.shape[0])
    if out is None:
        out = torch.empty(n, 2, dtype=torch.float64, device=words.device)
    check(lib().dp_box_muller(_ptr(words), n, _ptr(out), _stream(stream)), "dp_box_muller")
    return out


def dp_workspace_status(workspace, stream=None):
    return lib().dp_workspace_status(_ptr(workspace), _stream(stream))


def auto_norm_method(B, T, d_in, d_out, r=0, dtype_code=DP_BF16):
    return METHOD_NAMES[lib().dp_auto_norm_method(B, T, d_in, d_out, r, dtype_code)]


def kernel_launches():
    """Kernels launched by the library so far in this process."""
    return int(lib().dp_kernel_launches())


def profiling_enable(on=True):
    check(lib().dp_profiling_enable(1 if on else 0), "dp_profiling_enable")


def profiling_collect():
    """{kernel kind: (device ms, launches)} for the launches recorded since the last collect."""
    n = int(lib().dp_profiling_kinds())
    ms = (ctypes.c_double * n)()
    cnt = (_c_ll * n)()
    check(lib().dp_profiling_collect(ms, cnt), "dp_profiling_collect")
    return {lib().dp_profiling_kind_name(k).decode(): (ms[k], cnt[k]) for k in range(n) if cnt[k]}


def dp_block_step(layers, mode="per_layer", C=1.0, sigma=0.0, seed=0, step=0, method="auto",
                  flat_norms_out=None, workspace=None, stream=None):
    """One step for a block of linears sharing the batch.

    ``layers``: dicts with X, dY, layer_id, C (per-layer bound), and optional G_out, norms_out and
    P (a [d_out, r] projection: the layer then clips and noises G_i P).
    ``step``: a number, or a one-element int64 CUDA tensor read when the kernels run.
    Returns (list of G_out, list of norms_out or None, flat_norms_out or None).
    """
    import torch

    first = layers[0]
    B, T = int(first["X"].shape[0]), int(first["X"].shape[1])
    dt = _dtype_code(first["X"])
    arr = (DpLayer * len(layers))()
    outs, norms = [], []
    for k, l in enumerate(layers):
        _, _, d_in, d_out = _bt_dims(l["X"], l["dY"])
        P = l.get("P")
        r = int(P.shape[1]) if P is not None else 0
        G = l.get("G_out")
        if G is None:
            G = torch.empty(d_in, r or d_out, dtype=torch.float32, device=l["X"].device)
        n = l.get("norms_out")
        arr[k] = DpLayer(_ptr(l["X"]), _ptr(l["dY"]), d_in, d_out, int(l["layer_id"]), float(l.get("C", C)),
                         _ptr(G), _ptr(n), _ptr(P), r)
        outs.append(G)
        norms.append(n)
    need = int(lib().dp_block_workspace_size(arr, len(layers), B, T, dt, CLIP_MODES[mode], METHODS[method]))
    if need == 0:
        raise DPError(DP_ERR_INVALID_ARG, "dp_block_workspace_size")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=first["X"].device)
    if mode == "flat" and flat_norms_out is None:
        flat_norms_out = torch.empty(B, dtype=torch.float32, device=first["X"].device)
    dstep = _device_step(step)
    if dstep is not None:
        check(lib().dp_block_step_dev_step(arr, len(layers), dt, B, T, CLIP_MODES[mode], float(C), float(sigma),
                                           int(seed), _ptr(dstep), METHODS[method], _ptr(flat_norms_out),
                                           _ptr(workspace), workspace.numel(), _stream(stream)),
              "dp_block_step_dev_step")
    else:
        check(lib().dp_block_step(arr, len(layers), dt, B, T, CLIP_MODES[mode], float(C), float(sigma),
                                  int(seed), int(step), METHODS[method], _ptr(flat_norms_out),
                                  _ptr(workspace), workspace.numel(), _stream(stream)),
              "dp_block_step")
    return outs, norms, flat_norms_out


def dp_projected_adam_step(W, R, m, v, P, lr, t, beta1=0.9, beta2=0.999, eps=1e-8, grad_scale=1.0,
                           workspace=None, stream=None):
    """One projected Adam update: W -= lr * U P^T with Adam moments m, v kept in r-space."""
    import torch

    d_in, d_out = int(W.shape[0]), int(W.shape[1])
    r = int(R.shape[1])
    if workspace is None:
        workspace = torch.empty(int(lib().dp_adam_workspace_size(d_in, r)), dtype=torch.uint8, device=W.device)
    check(lib().dp_projected_adam_step(_ptr(W), _ptr(R), _ptr(m), _ptr(v), _ptr(P), _dtype_code(P), d_in, d_out,
                                       r, float(lr), float(beta1), float(beta2), float(eps), float(grad_scale),
                                       int(t), _ptr(workspace), workspace.numel(), _stream(stream)),
          "dp_projected_adam_step")
    return W, m, v
