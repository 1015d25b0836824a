"""Exact IO-aware attention (FlashAttention-2 style) for B200 / sm_100a.

``forward`` / ``backward`` call the C-ABI library ``libfa_sm100.so`` (built
from ``csrc/`` by ``build.py``); there is no CPU fallback.  Importing this
package loads nothing: the library is opened on first use.
"""
from __future__ import annotations

__all__ = ["forward", "backward", "backward_workspace_bytes", "FaError", "load_library",
           "workloads"]


def __getattr__(name):
    if name in ("forward", "backward", "backward_workspace_bytes", "FaError", "load_library",
                "forward_raw", "backward_raw", "attention"):
        from . import binding
        return getattr(binding, name)
    if name == "workloads":
        from . import workloads
        return workloads
    raise AttributeError(name)
