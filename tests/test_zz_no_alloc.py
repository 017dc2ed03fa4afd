"""The no-allocation forward entry point, gdr2_chunk_fwd_noalloc.

It serves callers that cannot allocate device memory (plugins handed only input and output buffers by a
framework that owns all device memory, latency-critical loops that may not call cudaMalloc). Its results are
compared with the fp64 oracle on the same inputs and, as a second check, with gdr2_chunk_fwd, call after
call, while it uses the library's fixed scratch array instead of a caller workspace. The cases include a
problem that fills the array to its documented limit, absent initial and final states, and a call through the
Python binding. This file is collected last so that a run stopping at the first failure has already run every
other test.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from gated_delta_rule_65_b200 import gdr2, workloads
from tests.parity import assert_close, cuda, oracle_fwd


def _noalloc_via_c_abi(g, B, T, H, dk, dv, want_final=True):
    """Call the entry point through the C ABI directly (ctypes, no binding helper)."""
    L = gdr2.lib()
    o = torch.empty((B, T, H, dv), dtype=g["q"].dtype, device="cuda")
    ST = torch.empty((B, H, dk, dv), dtype=torch.float32, device="cuda") if want_final else None
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = L.gdr2_chunk_fwd_noalloc(p(g["q"]), p(g["k"]), p(g["v"]), p(g["log_alpha"]), p(g["b"]), p(g["w"]),
                                  p(g["initial_state"]), p(o), p(ST), B, T, H, dk, dv,
                                  gdr2.GDR2_BF16 if g["q"].dtype == torch.bfloat16 else gdr2.GDR2_F32,
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == gdr2.OK, gdr2.status_string(st)
    return o, ST


CASES = [
    # (B, T, H, dk, dv, dtype, s0_std, want_final): 113 chunks fill the 32 MiB array for dk = dv = 128,
    # 204 chunks for dk = dv = 64
    (1, 113 * 64, 1, 128, 128, "bf16", 0.1, True),
    (2, 102 * 64 - 5, 1, 64, 64, "f32", None, True),
    (1, 300, 4, 128, 128, "bf16", 0.1, True),
    (2, 200, 3, 64, 128, "f32", None, False),
]


@pytest.mark.gpu
@pytest.mark.parametrize("B,T,H,dk,dv,dtype,s0_std,want_final", CASES)
def test_noalloc_matches_oracle_on_two_calls_in_a_row(B, T, H, dk, dv, dtype, s0_std, want_final):
    wl = workloads.ChunkWorkload("na", B=B, T=T, H=H, dk=dk, dv=dv, dtype=dtype, s0_std=s0_std, seed=70 + T)
    inp = workloads.chunk_inputs(wl)
    g = cuda(inp)
    ro, rST = oracle_fwd(inp)
    o_ref, ST_ref = gdr2.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["b"], g["w"], g["initial_state"])
    for _ in range(2):
        o, ST = _noalloc_via_c_abi(g, B, T, H, dk, dv, want_final)
        torch.cuda.synchronize()
        assert_close("o", o, ro, dtype)
        assert_close("o vs gdr2_chunk_fwd", o, o_ref.double(), dtype)
        if want_final:
            assert_close("final_state", ST, rST, dtype)
            assert_close("final_state vs gdr2_chunk_fwd", ST, ST_ref.double(), dtype)


@pytest.mark.gpu
def test_noalloc_through_the_binding():
    wl = workloads.ChunkWorkload("na_py", B=1, T=256, H=2, dk=64, dv=64, dtype="f32", seed=79)
    inp = workloads.chunk_inputs(wl)
    g = cuda(inp)
    o, ST = gdr2.chunk_fwd_noalloc(g["q"], g["k"], g["v"], g["log_alpha"], g["b"], g["w"], g["initial_state"])
    torch.cuda.synchronize()
    ro, rST = oracle_fwd(inp)
    assert_close("o", o, ro, "f32")
    assert_close("final_state", ST, rST, "f32")


def test_noalloc_rejects_problems_larger_than_its_scratch():
    """Sizes beyond the fixed scratch are refused before any CUDA call (runs without a GPU)."""
    L = gdr2.lib()
    fake = ctypes.c_void_p(0x10000)
    args = [fake] * 6 + [None, fake, None]
    # dk = dv = 128 allows B*H*ceil(T/64) <= 113 chunks: 114 chunks must be refused
    assert L.gdr2_chunk_fwd_noalloc(*args, 1, 114 * 64, 1, 128, 128, 1, None) == gdr2.ERR_WORKSPACE
    assert L.gdr2_chunk_fwd_noalloc(*args, 1, 205 * 64, 1, 64, 64, 0, None) == gdr2.ERR_WORKSPACE
    assert L.gdr2_chunk_fwd_noalloc(*args, 1, 171 * 64, 1, 64, 128, 0, None) == gdr2.ERR_WORKSPACE
    assert L.gdr2_chunk_fwd_noalloc(*args, 1, 129 * 64, 1, 128, 64, 0, None) == gdr2.ERR_WORKSPACE
    assert L.gdr2_chunk_fwd_noalloc(*args, 2, 4096, 16, 128, 128, 1, None) == gdr2.ERR_WORKSPACE
    # a chunk count of exactly 2^32 (64 * 1024 * 2^16 chunks) must not wrap to a small size
    assert L.gdr2_chunk_fwd_noalloc(*args, 64, 1 << 22, 1024, 128, 128, 1, None) == gdr2.ERR_WORKSPACE
    assert L.gdr2_chunk_fwd_noalloc(*args, 65535, 1 << 30, 65535, 64, 64, 0, None) == gdr2.ERR_WORKSPACE
    assert L.gdr2_chunk_fwd_noalloc(*args, 1, 64, 1, 96, 128, 1, None) == gdr2.ERR_UNSUPPORTED
    assert L.gdr2_chunk_fwd_noalloc(*([None] + args[1:]), 1, 64, 1, 128, 128, 1, None) == gdr2.ERR_INVALID_ARG
