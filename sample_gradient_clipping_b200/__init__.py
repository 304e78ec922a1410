"""B200-native (sm_100a) per-sample gradient clipping for DP-SGD on linear layers.

The computation lives in ``libdpclip.so`` (CUDA, C ABI in ``include/dpclip.h``).  This package
holds the ctypes binding (``_lib``), the in-tree build script (``build``) and the seeded
synthetic workloads (``inputs``).
"""
from ._lib import (  # noqa: F401
    DPError, auto_norm_method, dp_add_noise, dp_block_step, dp_clip_accumulate, dp_linear_step, dp_philox_blocks,
    dp_projected_adam_step,
    dp_per_sample_norms, dp_projection_matrix, dp_workspace_status, lib, workspace_size,
)
