"""B200-native (sm_100a) Gated Delta Rule-2 sequence mixer.

The kernels live in ``libgdr2.so`` (sources in ``csrc/``, C ABI in ``include/gdr2.h``); ``gdr2`` is
the ctypes binding and ``workloads`` draws seeded synthetic inputs.
"""
from .gdr2 import (GDR2Error, alloc_workspace, chunk_bwd, chunk_fwd, decode_step, lib,  # noqa: F401
                   status_string, workspace_bytes)

__all__ = ["GDR2Error", "alloc_workspace", "chunk_bwd", "chunk_fwd", "decode_step", "lib", "status_string",
           "workspace_bytes"]
