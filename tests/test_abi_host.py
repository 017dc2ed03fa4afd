"""Host-side checks of the C ABI (no GPU needed: nothing here launches a kernel).

The library links the CUDA runtime statically and validates every argument before its first CUDA
call, so these calls return their status without touching device memory.
"""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from gated_delta_rule_65_b200 import gdr2

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "gdr2.h")

FAKE = 0x10000      # 16-byte aligned, never dereferenced (validation fails first)
MISALIGNED = 0x10008


def _declared_functions():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"GDR2_API\s+[\w\s\*]+?\b(gdr2_\w+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    L = gdr2.lib()
    declared = _declared_functions()
    assert len(declared) >= 6
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(gdr2.EXPORTED)


def test_debug_library_exports_every_declared_symbol():
    """libgdr2_debug.so (-DGDR2_DEBUG index checks) exports the same C ABI as the release library."""
    import ctypes

    from gated_delta_rule_65_b200 import build as gbuild
    L = ctypes.CDLL(gbuild.build_debug())
    for name in _declared_functions():
        assert hasattr(L, name), name


def test_version_and_status_strings():
    assert gdr2.lib().gdr2_version() >= 100
    for st in range(8):
        s = gdr2.status_string(st)
        assert isinstance(s, str) and s and s != "unknown status"
    assert "log-decay" in gdr2.status_string(gdr2.ERR_RANGE)
    assert "debug build" in gdr2.status_string(gdr2.ERR_BOUNDS)
    assert gdr2.status_string(99) == "unknown status"


def test_workspace_bytes():
    f = gdr2.workspace_bytes
    assert f(1, 256, 2, 64, 64, 0, 0) > 0
    assert f(1, 256, 2, 64, 64, 0, 1) > f(1, 256, 2, 64, 64, 0, 0)
    assert f(0, 256, 2, 64, 64, 0, 0) == 0
    assert f(1, 256, 2, 96, 64, 0, 0) == 0      # unsupported head size
    assert f(1, 256, 2, 64, 64, 7, 0) == 0      # bad dtype
    old = gdr2.get_chunk_path()
    try:
        gdr2.set_chunk_path(gdr2.PATH_SPLIT)
        _split_path_workspace_sizes(f)
        gdr2.set_chunk_path(gdr2.PATH_CHAIN)
        # the per-chain forward keeps everything on chip: no workspace; the backward's record is 48 KB per chunk
        assert f(8, 4096, 16, 128, 128, 1, 0) == 0 and f(1, 100, 1, 128, 128, 1, 0) == 0
        assert f(8, 4096, 16, 128, 128, 1, 1) == 8 * 16 * 64 * 48 * 1024
        assert f(1, 100, 1, 128, 128, 1, 1) == 2 * 48 * 1024
        # other shapes and dtypes are unaffected by the path setting
        assert f(1, 256, 2, 64, 64, 0, 0) > 0
        gdr2.set_chunk_path(gdr2.PATH_AUTO)
        assert f(8, 4096, 16, 128, 128, 1, 0) == 0                    # 128 chains: per-chain kernels
        assert f(8, 4096, 16, 128, 128, 1, 1) == 8 * 16 * 64 * 48 * 1024
        assert f(1, 4096, 16, 128, 128, 1, 0) > 0                     # 16 chains: chunk-parallel kernels
        # the measured cost model: chunk-parallel below about 91 chains and between 149 and 180
        assert f(4, 4096, 16, 128, 128, 1, 0) > 0                     # 64 chains
        assert f(6, 4096, 16, 128, 128, 1, 0) == 0                    # 96 chains
        assert f(10, 4096, 16, 128, 128, 1, 0) > 0                    # 160 chains
        assert f(12, 4096, 16, 128, 128, 1, 0) == 0                   # 192 chains
    finally:
        gdr2.set_chunk_path(old)
    assert gdr2.lib().gdr2_set_chunk_path(3) == gdr2.ERR_INVALID_ARG
    assert gdr2.lib().gdr2_set_chunk_path(-1) == gdr2.ERR_INVALID_ARG


def test_scan_segment_rule():
    """The chunk-level scan's segment counts on the chunk-parallel kernels, read back from the forward workspace
    (each segment adds three fp32 states per chain): the plain serial passes for many short chains (the training
    batch, and 64 chains of 64 chunks, where a combine step costs more than the segments save), 9 segments for the
    long-context case, and the counts the GPU scan tests run with."""
    f = gdr2.workspace_bytes
    old = gdr2.get_chunk_path()
    try:
        gdr2.set_chunk_path(gdr2.PATH_SPLIT)
        per_chunk = f(8, 4096, 16, 128, 128, 1, 0) // (8 * 16 * 64)

        def nseg(B, T, H):
            extra = f(B, T, H, 128, 128, 1, 0) - per_chunk * B * H * (-(-T // 64))
            return 1 if extra == 0 else extra // (3 * B * H * 128 * 128 * 4)

        assert nseg(8, 4096, 16) == 1
        assert nseg(4, 4096, 16) == 1
        assert nseg(1, 65536, 16) == 9
        assert nseg(1, 64 * 24 + 37, 2) == 5
        assert nseg(2, 64 * 128 + 19, 2) == 10
    finally:
        gdr2.set_chunk_path(old)


def _split_path_workspace_sizes(f):
    # grows linearly with the number of chunks while every chain runs as one serial pass (many chains)
    assert f(16, 4096, 16, 128, 128, 1, 1) == 2 * f(8, 4096, 16, 128, 128, 1, 1)
    # few long chains: the chunk-level scan adds fp32 states per segment (3 forward, 2 more backward)
    per_chunk = f(8, 4096, 16, 128, 128, 1, 1) // (8 * 16 * 64)
    fwd_per_chunk = f(8, 4096, 16, 128, 128, 1, 0) // (8 * 16 * 64)
    nch = 16 * 1024
    extra_fwd = f(1, 65536, 16, 128, 128, 1, 0) - fwd_per_chunk * nch
    extra_bwd = f(1, 65536, 16, 128, 128, 1, 1) - per_chunk * nch
    state = 128 * 128 * 4
    assert extra_fwd > 0 and extra_fwd % (3 * 16 * state) == 0
    nseg = extra_fwd // (3 * 16 * state)
    assert 2 <= nseg <= 16 and extra_bwd == 5 * nseg * 16 * state


def _fwd(**over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, b=FAKE, w=FAKE, s0=None, o=FAKE, st=None,
                B=1, T=64, H=1, dk=64, dv=64, dt=0, ws=FAKE, wsb=1 << 40)
    args.update(over)
    a = args
    return gdr2.lib().gdr2_chunk_fwd(a["q"], a["k"], a["v"], a["la"], a["b"], a["w"], a["s0"], a["o"], a["st"],
                                     a["B"], a["T"], a["H"], a["dk"], a["dv"], a["dt"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("over,status", [
    (dict(q=None), gdr2.ERR_INVALID_ARG),
    (dict(o=None), gdr2.ERR_INVALID_ARG),
    (dict(la=MISALIGNED), gdr2.ERR_INVALID_ARG),
    (dict(s0=MISALIGNED), gdr2.ERR_INVALID_ARG),
    (dict(B=0), gdr2.ERR_INVALID_ARG),
    (dict(T=-1), gdr2.ERR_INVALID_ARG),
    (dict(dt=2), gdr2.ERR_INVALID_ARG),
    (dict(dk=96), gdr2.ERR_UNSUPPORTED),
    (dict(dv=256), gdr2.ERR_UNSUPPORTED),
    (dict(H=70000), gdr2.ERR_UNSUPPORTED),
    (dict(ws=None), gdr2.ERR_WORKSPACE),
    (dict(wsb=16), gdr2.ERR_WORKSPACE),
    (dict(ws=MISALIGNED), gdr2.ERR_WORKSPACE),
])
def test_chunk_fwd_rejects_bad_arguments(over, status):
    assert _fwd(**over) == status


def test_chunk_bwd_rejects_bad_arguments():
    L = gdr2.lib()
    P = [FAKE] * 16
    P[6] = None   # initial_state optional
    P[7] = None   # d_o optional
    P[8] = None   # d_final_state optional
    P[15] = None  # d_initial_state optional
    good = dict(B=1, T=64, H=1, dk=64, dv=64, dt=1)

    def call(P, ws=FAKE, wsb=16, **s):
        s = {**good, **s}
        return L.gdr2_chunk_bwd(*P, s["B"], s["T"], s["H"], s["dk"], s["dv"], s["dt"], ws, wsb, None)

    assert call(P) == gdr2.ERR_WORKSPACE           # all pointers fine, workspace too small
    for i in (0, 1, 2, 3, 4, 5, 9, 10, 11, 12, 13, 14):
        Q = list(P)
        Q[i] = None
        assert call(Q) == gdr2.ERR_INVALID_ARG, i
        Q[i] = MISALIGNED
        assert call(Q) == gdr2.ERR_INVALID_ARG, i
    assert call(P, dk=32) == gdr2.ERR_UNSUPPORTED


def test_decode_rejects_bad_arguments():
    L = gdr2.lib()

    def call(P=None, **s):
        P = P or [FAKE] * 8
        d = dict(B=2, H=2, dk=128, dv=128, dt=1)
        d.update(s)
        return L.gdr2_decode_step(*P, d["B"], d["H"], d["dk"], d["dv"], d["dt"], None)

    assert call(B=0) == gdr2.ERR_INVALID_ARG
    assert call(dt=5) == gdr2.ERR_INVALID_ARG
    assert call(dk=96) == gdr2.ERR_UNSUPPORTED
    assert call(dv=96) == gdr2.ERR_UNSUPPORTED
    assert call(dv=320) == gdr2.ERR_UNSUPPORTED
    for i in range(8):
        P = [FAKE] * 8
        P[i] = None
        assert call(P) == gdr2.ERR_INVALID_ARG
        P[i] = MISALIGNED
        assert call(P) == gdr2.ERR_INVALID_ARG


def test_varlen_workspace_and_validation():
    f = gdr2.workspace_bytes_varlen
    assert f(3, 500, 2, 128, 128, 1, 1) > f(3, 500, 2, 128, 128, 1, 0) > 0
    assert f(3, 500, 2, 64, 64, 1, 0) == 0       # packed batches: tensor-core path only
    assert f(3, 500, 2, 128, 128, 0, 0) == 0     # bf16 operands only
    assert f(0, 500, 2, 128, 128, 1, 0) == 0
    assert f(70000, 500, 2, 128, 128, 1, 0) == 0
    # room for T/64 + N chunks per head: grows with N at fixed T
    assert f(9, 4096, 2, 128, 128, 1, 1) > f(3, 4096, 2, 128, 128, 1, 1)
    L = gdr2.lib()
    good = dict(N=3, T=500, H=2, dk=128, dv=128, dt=1)

    def fwd(P, ws=FAKE, wsb=1 << 40, **s):
        s = {**good, **s}
        return L.gdr2_chunk_fwd_varlen(*P, s["N"], s["T"], s["H"], s["dk"], s["dv"], s["dt"], ws, wsb, None)

    def bwd(P, ws=FAKE, wsb=16, **s):
        s = {**good, **s}
        return L.gdr2_chunk_bwd_varlen(*P, s["N"], s["T"], s["H"], s["dk"], s["dv"], s["dt"], ws, wsb, None)

    P = [FAKE] * 10
    P[6] = P[8] = None  # initial_state, final_state optional
    for i in (0, 1, 2, 3, 4, 5, 7, 9):  # q k v log_alpha b w o cu_seqlens
        Q = list(P)
        Q[i] = None
        assert fwd(Q) == gdr2.ERR_INVALID_ARG, i
        Q[i] = MISALIGNED
        assert fwd(Q) == gdr2.ERR_INVALID_ARG, i
    assert fwd(P, dk=64, dv=64) == gdr2.ERR_UNSUPPORTED
    assert fwd(P, dt=0) == gdr2.ERR_UNSUPPORTED
    assert fwd(P, N=0) == gdr2.ERR_INVALID_ARG
    assert fwd(P, ws=None) == gdr2.ERR_WORKSPACE
    assert fwd(P, wsb=16) == gdr2.ERR_WORKSPACE
    B = [FAKE] * 17
    B[6] = B[7] = B[8] = B[15] = None  # initial_state, d_o, d_final_state, d_initial_state optional
    assert bwd(B) == gdr2.ERR_WORKSPACE
    B[16] = None
    assert bwd(B) == gdr2.ERR_INVALID_ARG  # cu_seqlens


def test_gate_prologue_validation():
    L = gdr2.lib()
    f = L.gdr2_gate_prologue_workspace_bytes
    assert f(2, 100, 3, 128, 128, 1) > 0 and f(2, 100, 3, 96, 128, 1) == 0 and f(0, 100, 3, 128, 128, 1) == 0

    def fwd(P, **s):
        d = dict(B=2, T=100, H=3, dk=128, dv=128, dt=1)
        d.update(s)
        return L.gdr2_gate_prologue_fwd(*P[:7], 0, *P[7:], d["B"], d["T"], d["H"], d["dk"], d["dv"], d["dt"], None)

    for i in range(12):
        P = [FAKE] * 12
        P[i] = None
        assert fwd(P) == gdr2.ERR_INVALID_ARG, i
        P[i] = MISALIGNED
        assert fwd(P) == gdr2.ERR_INVALID_ARG, i
    assert fwd([FAKE] * 12, dk=32) == gdr2.ERR_UNSUPPORTED
    assert fwd([FAKE] * 12, T=0) == gdr2.ERR_INVALID_ARG

    def bwd(P, ws=FAKE, wsb=16):
        return L.gdr2_gate_prologue_bwd(*P[:7], 1, *P[7:], 2, 100, 3, 128, 128, 1, ws, wsb, None)

    assert bwd([FAKE] * 19) == gdr2.ERR_WORKSPACE
    assert bwd([FAKE] * 19, ws=None, wsb=1 << 40) == gdr2.ERR_WORKSPACE
    for i in range(19):
        P = [FAKE] * 19
        P[i] = None
        assert bwd(P, wsb=1 << 40) == gdr2.ERR_INVALID_ARG, i


def test_gva_validation():
    f = gdr2.workspace_bytes_gva
    assert f(2, 256, 2, 4, 128, 128, 1, 1) > f(2, 256, 2, 4, 128, 128, 1, 0) > 0
    assert f(2, 256, 2, 2, 128, 128, 1, 1) == gdr2.workspace_bytes(2, 256, 2, 128, 128, 1, 1)  # G = 1
    assert f(2, 256, 2, 3, 128, 128, 1, 0) == 0   # Hv not a multiple of H
    assert f(2, 256, 2, 4, 64, 64, 1, 0) == 0     # tensor-core path only
    assert f(2, 256, 2, 0, 128, 128, 1, 0) == 0
    # key-side arrays per key chunk, value-side per value chunk: more value heads cost less than more heads
    assert f(2, 4096, 8, 16, 128, 128, 1, 1) < f(2, 4096, 16, 16, 128, 128, 1, 1)
    L = gdr2.lib()

    def fwd(P, **s):
        d = dict(B=2, T=256, H=2, Hv=4, dk=128, dv=128, dt=1, wsb=1 << 40)
        d.update(s)
        return L.gdr2_chunk_fwd_gva(*P, d["B"], d["T"], d["H"], d["Hv"], d["dk"], d["dv"], d["dt"], FAKE, d["wsb"],
                                    None)

    P = [FAKE] * 9
    P[6] = P[8] = None
    assert fwd(P, Hv=3) == gdr2.ERR_INVALID_ARG
    assert fwd(P, Hv=0) == gdr2.ERR_INVALID_ARG
    assert fwd(P, dk=64, dv=64) == gdr2.ERR_UNSUPPORTED
    assert fwd(P, wsb=16) == gdr2.ERR_WORKSPACE
    for i in (0, 1, 2, 3, 4, 5, 7):
        Q = list(P)
        Q[i] = None
        assert fwd(Q) == gdr2.ERR_INVALID_ARG, i


def test_varlen_gva_validation():
    f = gdr2.workspace_bytes_varlen
    # group of one: the plain packed layout; more value heads: bigger than the plain packed layout of H
    assert f(5, 700, 2, 128, 128, 1, 1, Hv=2) == f(5, 700, 2, 128, 128, 1, 1)
    assert f(5, 700, 2, 128, 128, 1, 1, Hv=4) > f(5, 700, 2, 128, 128, 1, 1) > 0
    assert f(5, 700, 2, 128, 128, 1, 1, Hv=4) < f(5, 700, 4, 128, 128, 1, 1)  # key side once per group
    L = gdr2.lib()
    assert L.gdr2_workspace_bytes_varlen_gva(5, 700, 2, 3, 128, 128, 1, 0) == 0   # Hv not a multiple of H
    assert L.gdr2_workspace_bytes_varlen_gva(0, 700, 2, 4, 128, 128, 1, 0) == 0   # no sequences
    assert L.gdr2_workspace_bytes_varlen_gva(5, 700, 2, 4, 64, 64, 1, 0) == 0     # tensor-core path only

    def fwd(P, **s):
        d = dict(N=5, T=700, H=2, Hv=4, dk=128, dv=128, dt=1, wsb=1 << 40)
        d.update(s)
        return L.gdr2_chunk_fwd_varlen_gva(*P, d["N"], d["T"], d["H"], d["Hv"], d["dk"], d["dv"], d["dt"], FAKE,
                                           d["wsb"], None)

    P = [FAKE] * 10
    P[6] = P[8] = None
    assert fwd(P, Hv=3) == gdr2.ERR_INVALID_ARG
    assert fwd(P, Hv=0) == gdr2.ERR_INVALID_ARG
    assert fwd(P, N=0) == gdr2.ERR_INVALID_ARG
    assert fwd(P, dk=64, dv=64) == gdr2.ERR_UNSUPPORTED
    assert fwd(P, wsb=16) == gdr2.ERR_WORKSPACE
    for i in (0, 1, 2, 3, 4, 5, 7, 9):
        Q = list(P)
        Q[i] = None
        assert fwd(Q) == gdr2.ERR_INVALID_ARG, i


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 64, 1, 64)
    with pytest.raises(ValueError):
        gdr2.chunk_fwd(x, x, x, x, x, x, workspace=torch.zeros(16, dtype=torch.uint8))


def test_product_package_does_not_import_the_oracle():
    """The CUDA path and the oracle share no code: no module of the package names the oracle."""
    pkg = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "gated_delta_rule_65_b200")
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c", ".cpp")):
                txt = open(os.path.join(root, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "gdr2_oracle" not in txt and "oracle_gdr2" not in txt, f
