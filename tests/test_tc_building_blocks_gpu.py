"""GPU checks of the tcgen05 / TMA building blocks (libgdr2_selftest.so, B200 only).

A single M = 128 tcgen05.mma GEMM is run with every K-major / MN-major operand combination used by
the chunk kernels and compared with a torch matmul of the same bf16 values; and the shared-memory
image of a 128-byte-swizzled TMA load is compared with the tile layout the kernels assume.
"""
from __future__ import annotations

import ctypes
import itertools

import pytest
import torch

from gated_delta_rule_65_b200 import build

pytestmark = pytest.mark.gpu

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build.build_selftest())
        _lib.gdr2st_gemm.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 4
        _lib.gdr2st_gemm_f16.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 5
        _lib.gdr2st_tma_layout.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    return _lib


@pytest.mark.parametrize("N,K,a_mn,b_mn", list(itertools.product([64, 128], [64, 128], [0, 1], [0, 1])))
def test_tcgen05_gemm_layouts(N, K, a_mn, b_mn):
    g = torch.Generator(device="cuda").manual_seed(N * 1000 + K * 10 + 2 * a_mn + b_mn)
    A = torch.randn(128, K, generator=g, device="cuda").bfloat16()      # op(A) [M, K]
    Bm = torch.randn(N, K, generator=g, device="cuda").bfloat16()       # op(B) [N, K]
    A_st = (A.t() if a_mn else A).contiguous()
    B_st = (Bm.t() if b_mn else Bm).contiguous()
    D = torch.full((128, N), float("nan"), device="cuda")
    st = lib().gdr2st_gemm(A_st.data_ptr(), B_st.data_ptr(), D.data_ptr(), N, K, a_mn, b_mn)
    assert st == 0
    ref = A.float() @ Bm.float().t()
    err = (D - ref).abs().max().item()
    assert err <= 1e-4 * max(ref.abs().max().item(), 1.0), err
    assert lib().gdr2st_wait_error() == 0


@pytest.mark.parametrize("N,K,a_mn,b_mn,mode", [c + (0,) for c in itertools.product([64, 128], [64, 128], [0, 1], [0, 1])]
                         + [c[:2] + (0,) + c[2:] + (1,) for c in itertools.product([64, 128], [64, 128], [0, 1])])
def test_tcgen05_gemm_f16_layouts(N, K, a_mn, b_mn, mode):
    """fp16 operands (kind::f16 with both operands fp16); mode 1 takes the A operand from TMEM."""
    g = torch.Generator(device="cuda").manual_seed(7 + N * 1000 + K * 10 + 2 * a_mn + b_mn + 100 * mode)
    A = torch.randn(128, K, generator=g, device="cuda").half()
    Bm = torch.randn(N, K, generator=g, device="cuda").half()
    A_st = (A.t() if a_mn else A).contiguous()
    B_st = (Bm.t() if b_mn else Bm).contiguous()
    D = torch.full((128, N), float("nan"), device="cuda")
    st = lib().gdr2st_gemm_f16(A_st.data_ptr(), B_st.data_ptr(), D.data_ptr(), N, K, a_mn, b_mn, mode)
    assert st == 0
    ref = A.float() @ Bm.float().t()
    err = (D - ref).abs().max().item()
    assert err <= 1e-4 * max(ref.abs().max().item(), 1.0), err
    assert lib().gdr2st_wait_error() == 0


@pytest.mark.parametrize("rows", [64, 128])
def test_tma_swizzle_matches_tile_layout(rows):
    src = torch.arange(rows * 128, device="cuda", dtype=torch.int32).remainder(30000).to(torch.bfloat16)
    src = src.view(rows, 128).contiguous()
    out = torch.zeros(rows * 256, dtype=torch.uint8, device="cuda")
    assert lib().gdr2st_tma_layout(src.data_ptr(), out.data_ptr(), rows) == 0
    img = out.view(torch.bfloat16).cpu()
    s = src.cpu()
    for r in range(rows):
        for c in range(128):
            sub, cc = divmod(c, 64)
            off = sub * rows * 128 + r * 128 + (((cc // 8) ^ (r % 8)) * 16) + (cc % 8) * 2
            assert img[off // 2] == s[r, c], (r, c)


@pytest.mark.parametrize("N", [64, 128])
def test_tcgen05_m64_tmem_rows(N):
    """Where an M = 64 product lands in TMEM: the test finds, for every result row, the lane that holds
    it, and checks the layout the kernels may assume: row m in lane 32 * (m // 16) + m % 16."""
    lib().gdr2st_gemm_m64_dump.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 2
    g = torch.Generator(device="cuda").manual_seed(5 + N)
    A = torch.randn(64, 128, generator=g, device="cuda").bfloat16()
    Bm = torch.randn(N, 128, generator=g, device="cuda").bfloat16()
    dump = torch.zeros(128, N, device="cuda")
    assert lib().gdr2st_gemm_m64_dump(A.data_ptr(), Bm.data_ptr(), dump.data_ptr(), N, 128) == 0
    ref = (A.float() @ Bm.float().t()).cpu()
    dump = dump.cpu()
    found = {}
    for m in range(64):
        for lane in range(128):
            if torch.allclose(dump[lane], ref[m], rtol=1e-4, atol=1e-3):
                found[m] = lane
                break
    expected = {m: 32 * (m // 16) + m % 16 for m in range(64)}
    assert found == expected, f"M=64 TMEM rows -> lanes: {found}"
