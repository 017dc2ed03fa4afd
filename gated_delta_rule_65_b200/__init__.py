"""B200-native (sm_100a) Gated Delta Rule-2 sequence mixer.

The kernels live in ``libgdr2.so`` (sources in ``csrc/``, C ABI in ``include/gdr2.h``); ``gdr2`` is
the ctypes binding and ``workloads`` draws seeded synthetic inputs.
"""
from .gdr2 import (GDR2Error, alloc_workspace, alloc_workspace_gva, alloc_workspace_varlen,  # noqa: F401
                   check, chunk_bwd, chunk_bwd_gva, chunk_bwd_varlen, chunk_fwd, chunk_fwd_gva, chunk_fwd_varlen,
                   decode_step, gate_prologue_bwd, gate_prologue_fwd, lib, status_string, workspace_bytes,
                   workspace_bytes_gva, workspace_bytes_varlen)

__all__ = ["GDR2Error", "alloc_workspace", "alloc_workspace_gva", "alloc_workspace_varlen", "check", "chunk_bwd",
           "chunk_bwd_gva", "chunk_bwd_varlen", "chunk_fwd", "chunk_fwd_gva", "chunk_fwd_varlen", "decode_step",
           "gate_prologue_bwd", "gate_prologue_fwd", "lib", "status_string", "workspace_bytes", "workspace_bytes_gva",
           "workspace_bytes_varlen"]
