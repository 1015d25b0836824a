"""Exact IO-aware attention (FlashAttention-2 style) for B200 / sm_100a.

``forward`` / ``backward`` call the C-ABI library ``libfa_sm100.so`` (built
from ``csrc/`` by ``build.py``); there is no CPU fallback.  Importing this
package loads nothing: the library is opened on first use.
"""
from __future__ import annotations

__all__ = ["forward", "backward", "forward_fp8", "attention", "backward_workspace_bytes",
           "check_device_error", "FaError", "load_library", "workloads"]


def __getattr__(name):
    # importlib, not "from . import x": that form looks the name up on this
    # package first, which would re-enter __getattr__.
    import importlib
    if name in ("forward", "backward", "forward_fp8", "backward_workspace_bytes", "FaError",
                "load_library", "forward_raw", "attention", "check_device_error"):
        return getattr(importlib.import_module(__name__ + ".binding"), name)
    if name == "workloads":
        return importlib.import_module(__name__ + ".workloads")
    raise AttributeError(name)
