"""GPU checks of the device status path (gdr2_check): kernels never trap; what they cannot do is reported.

* Ordinary calls leave the status clean.
* A chunk whose cumulative log-decay leaves the path's range in some channel ([-160, 160] on the
  tensor-core path, whose factors are relative to the mid-chunk value; [-80, 80] on the fp32 path), where
  the chunk form's exponential factors leave fp32's normal range, is reported as GDR2_ERR_RANGE, and the
  report clears once read; a decode step (no chunk form) has no such limit.
* A bounded mbarrier wait on which nothing ever arrives gives up after its poll limit and sets the
  timeout bit instead of spinning on (self-test library, a short limit); with an arrival it succeeds.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from gated_delta_rule_65_b200 import build, gdr2, workloads
from tests.parity import cuda

pytestmark = pytest.mark.gpu

TOKENS = ("q", "k", "v", "log_alpha", "b", "w")


def _chunk_inputs(dtype: str, dk: int, la_value: float | None, T: int = 128):
    wl = workloads.ChunkWorkload("status", B=1, T=T, H=2, dk=dk, dv=dk, dtype=dtype, backward=True, seed=77)
    g = cuda(workloads.chunk_inputs(wl))
    if la_value is not None:
        g["log_alpha"] = torch.full_like(g["log_alpha"], la_value)
    return g


def test_clean_calls_report_ok():
    assert gdr2.check() in (gdr2.OK, gdr2.ERR_RANGE)  # whatever earlier tests left, read and cleared
    g = _chunk_inputs("bf16", 128, None)
    gdr2.chunk_fwd(*(g[n] for n in TOKENS), g["initial_state"])
    gdr2.chunk_bwd(*(g[n] for n in TOKENS), g["initial_state"], g["d_o"], g["d_final_state"])
    assert gdr2.check() == gdr2.OK


@pytest.mark.parametrize("dtype,dk,outside,inside", [("bf16", 128, -3.0, -2.4), ("f32", 64, -2.0, -1.2)])
def test_strong_decay_is_reported_then_cleared(dtype, dk, outside, inside):
    gdr2.check()
    g = _chunk_inputs(dtype, dk, outside)  # 64 rows: -192 (tensor-core path) or -128 (fp32 path) per chunk
    o, _ = gdr2.chunk_fwd(*(g[n] for n in TOKENS), g["initial_state"])
    assert gdr2.check() == gdr2.ERR_RANGE
    assert gdr2.check() == gdr2.OK  # cleared on read
    g = _chunk_inputs(dtype, dk, inside)  # -153.6 or -76.8 per chunk: inside the path's bound
    o, _ = gdr2.chunk_fwd(*(g[n] for n in TOKENS), g["initial_state"])
    assert gdr2.check() == gdr2.OK
    assert torch.isfinite(o).all()


def test_decode_has_no_chunk_range_limit():
    gdr2.check()
    wl = workloads.DECODE_WORKLOADS["decode_256x16"]
    d = cuda(workloads.decode_inputs(wl, B=2, steps=1))
    la = torch.full_like(d["log_alpha"][0], -5.0)
    state = d["state"].clone()
    o = gdr2.decode_step(d["q"][0], d["k"][0], d["v"][0], la, d["b"][0], d["w"][0], state)
    assert gdr2.check() == gdr2.OK
    assert torch.isfinite(o).all() and torch.isfinite(state).all()


def _selftest():
    L = ctypes.CDLL(build.build_selftest())
    L.gdr2st_bounded_wait.restype = ctypes.c_int
    L.gdr2st_bounded_wait.argtypes = [ctypes.c_uint, ctypes.c_int, ctypes.c_void_p]
    L.gdr2st_index_check.restype = ctypes.c_int
    L.gdr2st_index_check.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
    return L


def test_debug_index_check_reports_without_trapping():
    """The debug build's tile-index check (compiled into the self-test library): an in-range row leaves the
    status word clean; a row past the tile sets the bounds bit (4), read back on the host, and the kernel
    returns normally. The offset is computed only; no memory is touched at the bad index."""
    L = _selftest()
    off = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert L.gdr2st_index_check(64, 3, ctypes.c_void_p(off.data_ptr())) == 0
    assert int(off.item()) == 3 * 128 + 3 * 16  # row 3, its 16-byte chunk 0 swizzled to chunk 3
    assert L.gdr2st_index_check(64, 64, ctypes.c_void_p(off.data_ptr())) == 4
    assert L.gdr2st_index_check(64, -1, ctypes.c_void_p(off.data_ptr())) == 4
    assert gdr2.check() == gdr2.OK  # the library's own status word is untouched


def test_bounded_wait_gives_up_and_reports():
    L = _selftest()
    done = torch.zeros(1, dtype=torch.int32, device="cuda")
    bits = L.gdr2st_bounded_wait(4096, 0, ctypes.c_void_p(done.data_ptr()))
    assert bits == 1 and int(done.item()) == 2  # the timeout bit, and the wait returned "gave up"
    done.zero_()
    bits = L.gdr2st_bounded_wait(4096, 1, ctypes.c_void_p(done.data_ptr()))
    assert bits == 0 and int(done.item()) == 1  # with an arrival the same wait completes
    assert gdr2.check() == gdr2.OK  # the library's own status word is untouched
