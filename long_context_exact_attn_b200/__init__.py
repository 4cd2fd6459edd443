"""Exact blockwise (Ring / Striped) causal attention on B200 (sm_100a).

The compute path is the C-ABI library ``libringattn.so`` built from
``csrc/``; ``ops`` is a thin ctypes binding over it (argument marshalling
only).  ``workloads`` holds the seeded synthetic inputs.
"""

import importlib

__all__ = ["ops", "workloads"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
