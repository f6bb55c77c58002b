"""B200-native (sm_100a) library for the ESA gated linear recurrence scan.

The hot path -- forward scan with fused gate sigmoid and per-head RMS
readout, its backward scan, and the one-token decode update -- is
hand-written CUDA behind a C ABI (``include/esa.h``); this package is the thin
ctypes binding over it, a torch autograd function and ``ESA`` layer on top of
the binding (``layer.py``), the build script and seeded input generators.
"""
from .esa import (  # noqa: F401
    CONTROLLED,
    DIRECT,
    EsaError,
    LIB_PATH,
    PreparedStep,
    esa_check,
    esa_compose,
    esa_fused_fwd,
    esa_fused_layer_fwd,
    esa_scan_bwd,
    esa_scan_bwd_map,
    esa_scan_fwd,
    esa_scan_map,
    esa_step,
    esa_strerror,
    esa_version,
    esa_workspace_init,
    esa_workspace_size,
    load_library,
    new_workspace,
)
from .layer import ESA, esa_scan  # noqa: F401

__all__ = [
    "CONTROLLED", "DIRECT", "EsaError", "LIB_PATH", "PreparedStep", "esa_check", "esa_compose", "esa_fused_fwd", "esa_fused_layer_fwd", "esa_scan_bwd",
    "esa_scan_bwd_map", "esa_scan_fwd", "esa_scan_map", "esa_step", "esa_strerror", "esa_version",
    "esa_workspace_init", "esa_workspace_size", "load_library", "new_workspace", "ESA", "esa_scan",
]
