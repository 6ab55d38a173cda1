"""B200-native Mamba-2 SSD layer: ``forward`` (chunked prefill) and ``step`` (decode).

The compute lives in the C-ABI library ``libssd_b200.so`` (hand-written
sm_100a CUDA, declared in ``include/ssd.h``); ``ssd.py`` is a thin ctypes
binding that only marshals arguments. Importing this package does not load the
library; the first use of ``forward``/``step``/``lib`` does, and fails loudly
if it is missing. ``inputs`` (seeded synthetic data) needs no GPU.
"""
from __future__ import annotations

import importlib

__all__ = ["forward", "step", "workspace_size", "lib", "SSDError", "inputs", "ssd"]


def __getattr__(name):
    if name in ("inputs", "ssd"):
        return importlib.import_module(f".{name}", __name__)
    if name in ("forward", "step", "workspace_size", "lib", "SSDError", "poll_status",
                "forward_host", "library_path"):
        mod = importlib.import_module(".ssd", __name__)
        return getattr(mod, name)
    raise AttributeError(name)
