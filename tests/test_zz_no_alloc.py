"""The no-allocation forward entry point, gdr2_chunk_fwd_noalloc.

It serves callers that cannot allocate device memory (plugins handed only input and output
buffers by a framework that owns all device memory, latency-critical loops that may not call
cudaMalloc). It must give the same results as gdr2_chunk_fwd, call after call, while using the
library's fixed scratch array instead of a caller workspace. This file is collected last so that a
run stopping at the first failure has already run every other test.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from gated_delta_rule_65_b200 import gdr2, workloads
from tests.parity import assert_close, cuda


def _noalloc_via_c_abi(g, B, T, H, dk, dv):
    """Call the entry point through the C ABI directly (ctypes, no binding helper)."""
    L = gdr2.lib()
    o = torch.empty((B, T, H, dv), dtype=g["q"].dtype, device="cuda")
    ST = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda")
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = L.gdr2_chunk_fwd_noalloc(p(g["q"]), p(g["k"]), p(g["v"]), p(g["log_alpha"]), p(g["b"]), p(g["w"]),
                                  p(g["initial_state"]), p(o), p(ST), B, T, H, dk, dv,
                                  gdr2.GDR2_BF16 if g["q"].dtype == torch.bfloat16 else gdr2.GDR2_F32,
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == gdr2.OK, gdr2.status_string(st)
    return o, ST


@pytest.mark.gpu
def test_noalloc_matches_chunk_fwd_on_two_calls_in_a_row():
    cases = [
        workloads.ChunkWorkload("na1", B=1, T=300, H=4, dk=128, dv=128, dtype="bf16", s0_std=0.1, seed=71),
        workloads.ChunkWorkload("na2", B=2, T=200, H=3, dk=64, dv=128, dtype="f32", seed=72),
    ]
    for wl in cases:
        g = cuda(workloads.chunk_inputs(wl))
        o_ref, ST_ref = gdr2.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["b"], g["w"], g["initial_state"])
        o, ST = _noalloc_via_c_abi(g, wl.B, wl.T, wl.H, wl.dk, wl.dv)
        torch.cuda.synchronize()
        assert_close("o", o, o_ref.double(), wl.dtype)
        assert_close("final_state", ST, ST_ref.double(), wl.dtype)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    """Sizes beyond the fixed scratch are refused before any CUDA call (runs without a GPU)."""
    L = gdr2.lib()
    fake = ctypes.c_void_p(0x10000)
    args = [fake] * 6 + [None, fake, None]
    # dk = dv = 128 allows B*H*ceil(T/64) <= 113 chunks: 114 chunks must be refused
    assert L.gdr2_chunk_fwd_noalloc(*args, 1, 114 * 64, 1, 128, 128, 1, None) == gdr2.ERR_WORKSPACE
    assert L.gdr2_chunk_fwd_noalloc(*args, 2, 4096, 16, 128, 128, 1, None) == gdr2.ERR_WORKSPACE
    assert L.gdr2_chunk_fwd_noalloc(*args, 1, 64, 1, 96, 128, 1, None) == gdr2.ERR_UNSUPPORTED
    assert L.gdr2_chunk_fwd_noalloc(*([None] + args[1:]), 1, 64, 1, 128, 128, 1, None) == gdr2.ERR_INVALID_ARG
