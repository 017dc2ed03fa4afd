"""GPU parity of gdr2_chunk_fwd / gdr2_chunk_bwd on the chunk-parallel kernels against the fp64 oracle (B200 only).

Small cases are compared element by element over every output. Full-size workloads run on the GPU
exactly as the benchmark launches them, and sampled (batch, head) chains -- each an independent
recurrence -- are recomputed by the oracle and compared in full.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

from gated_delta_rule_65_b200 import gdr2, workloads
from tests.parity import (assert_close, cuda, gpu_rows, oracle_bwd, oracle_fwd, select_chains)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _chunk_parallel_path():
    """These tests cover the chunk-parallel kernels (the per-chain kernels have test_chain_gpu.py): they run
    with gdr2_set_chunk_path(2), which the automatic mode picks for B*H < 64."""
    old = gdr2.get_chunk_path()
    gdr2.set_chunk_path(gdr2.PATH_SPLIT)
    yield
    gdr2.set_chunk_path(old)

GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw")
ORACLE_NAMES = {"dq": "dq", "dk": "dk", "dv": "dv", "dlog_alpha": "dlog_alpha", "db": "db", "dw": "dw"}


def _wl(name, **over):
    return dataclasses.replace(workloads.WORKLOADS[name], **over)


def _run_fwd(inp):
    g = cuda(inp)
    o, ST = gdr2.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["b"], g["w"], g["initial_state"])
    torch.cuda.synchronize()
    return o, ST


def _run_bwd(inp):
    g = cuda(inp)
    out = gdr2.chunk_bwd(g["q"], g["k"], g["v"], g["log_alpha"], g["b"], g["w"], g["initial_state"],
                         g.get("d_o"), g.get("d_final_state"))
    torch.cuda.synchronize()
    return out


def _check_fwd(inp, path, chains=None):
    o, ST = _run_fwd(inp)
    if chains is None:
        ro, rST = oracle_fwd(inp)
        assert_close("o", o, ro, path)
        assert_close("final_state", ST, rST, path)
    else:
        ro, rST = oracle_fwd(select_chains(inp, chains))
        assert_close("o", gpu_rows(o, chains), ro, path)
        assert_close("final_state", gpu_rows(ST, chains, state=True), rST, path)


def _check_bwd(inp, path, chains=None):
    out = _run_bwd(inp)
    if chains is None:
        ref = oracle_bwd(inp)
        for n in GRADS:
            assert_close(n, out[n], ref[ORACLE_NAMES[n]], path)
        assert_close("dS0", out["dS0"], ref["dS0"], path)
    else:
        ref = oracle_bwd(select_chains(inp, chains))
        for n in GRADS:
            assert_close(n, gpu_rows(out[n], chains), ref[ORACLE_NAMES[n]], path)
        assert_close("dS0", gpu_rows(out["dS0"], chains, state=True), ref["dS0"], path)


# --- the tiny fp32 workload (B=1, H=2, T=256, dk=dv=64) --------------------------------------------

def test_tiny_f32_forward():
    inp = workloads.chunk_inputs(workloads.WORKLOADS["tiny_f32"])
    _check_fwd(inp, "f32")


def test_tiny_f32_backward():
    inp = workloads.chunk_inputs(workloads.WORKLOADS["tiny_f32"])
    _check_bwd(inp, "f32")


# --- small shapes: ragged tails, every head size, both dtypes, with and without S0 -------------------

SMALL = [
    # (T, dk, dv, dtype, with_s0, neg_eig)
    (1, 64, 64, "f32", False, False),
    (63, 64, 64, "bf16", True, False),
    (65, 128, 128, "bf16", True, True),
    (100, 128, 128, "f32", True, False),
    (130, 64, 128, "bf16", False, True),
    (192, 128, 64, "f32", True, True),
    (257, 128, 128, "bf16", True, False),
]


@pytest.mark.parametrize("T,dk,dv,dtype,with_s0,neg_eig", SMALL)
def test_small_shapes_forward_backward(T, dk, dv, dtype, with_s0, neg_eig):
    wl = workloads.ChunkWorkload("small", B=2, T=T, H=3, dk=dk, dv=dv, dtype=dtype, neg_eig=neg_eig,
                                 s0_std=0.5 if with_s0 else None, backward=True, seed=7 + T)
    inp = workloads.chunk_inputs(wl)
    _check_fwd(inp, dtype)
    _check_bwd(inp, dtype)


def test_backward_with_absent_upstream_gradients():
    wl = workloads.ChunkWorkload("nograd", B=1, T=100, H=2, dk=64, dv=64, dtype="f32", s0_std=0.3,
                                 backward=True, seed=5)
    inp = workloads.chunk_inputs(wl)
    for drop in ("d_o", "d_final_state"):
        case = dict(inp)
        case[drop] = None
        _check_bwd(case, "f32")


@pytest.mark.parametrize("drop", ["d_o", "d_final_state"])
def test_backward_absent_upstream_tensor_core_path(drop):
    """bf16, dk = dv = 128 (tensor-core kernels, several chunks per CTA): a missing dO or dS_T counts as zeros."""
    wl = workloads.ChunkWorkload("nograd_tc", B=2, T=300, H=3, dk=128, dv=128, dtype="bf16", s0_std=0.3,
                                 neg_eig=True, backward=True, seed=23)
    case = dict(workloads.chunk_inputs(wl))
    case[drop] = None
    _check_bwd(case, "bf16")


def test_outputs_fully_written_and_deterministic():
    """Every output element is written (NaN canaries disappear) and two runs agree bit for bit."""
    wl = workloads.ChunkWorkload("canary", B=2, T=129, H=2, dk=128, dv=64, dtype="bf16", s0_std=0.1,
                                 backward=True, seed=11)
    g = cuda(workloads.chunk_inputs(wl))
    res = []
    for _ in range(2):
        o = torch.full((2, 129, 2, 64), float("nan"), dtype=torch.bfloat16, device="cuda")
        ST = torch.full((2, 2, 128, 64), float("nan"), device="cuda")
        gdr2.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["b"], g["w"], g["initial_state"], o=o, final_state=ST)
        out = {n: torch.full_like(g["q"], float("nan")) for n in ("dq", "dk", "db")}
        out.update({n: torch.full_like(g["v"], float("nan")) for n in ("dv", "dw")})
        out["dlog_alpha"] = torch.full_like(g["log_alpha"], float("nan"))
        out["dS0"] = torch.full_like(ST, float("nan"))
        gdr2.chunk_bwd(g["q"], g["k"], g["v"], g["log_alpha"], g["b"], g["w"], g["initial_state"], g["d_o"],
                       g["d_final_state"], out=out)
        torch.cuda.synchronize()
        for t in [o, ST, *out.values()]:
            assert torch.isfinite(t.float()).all()
        res.append([o, ST, *out.values()])
    for a, b in zip(*res):
        assert torch.equal(a, b)


@pytest.mark.parametrize("dtype,d,T", [("bf16", 128, 200), ("f32", 64, 130)])
def test_training_pair_matches_recompute(dtype, d, T):
    """gdr2_chunk_fwd_train + gdr2_chunk_bwd_saved give exactly the results of gdr2_chunk_fwd +
    gdr2_chunk_bwd (same kernels, intermediates kept instead of recomputed), and match the oracle."""
    wl = workloads.ChunkWorkload("train_pair", B=2, T=T, H=2, dk=d, dv=d, dtype=dtype, s0_std=0.2, neg_eig=True,
                                 backward=True, seed=41)
    inp = workloads.chunk_inputs(wl)
    g = cuda(inp)
    args = [g[n] for n in ("q", "k", "v", "log_alpha", "b", "w")] + [g["initial_state"]]
    o1, S1 = gdr2.chunk_fwd(*args)
    g1 = gdr2.chunk_bwd(*args, g["d_o"], g["d_final_state"])
    ws = gdr2.alloc_workspace(2, T, 2, d, d, gdr2._dtype_code(g["q"]), 1)
    o2, S2 = gdr2.chunk_fwd(*args, workspace=ws, train=True)
    g2 = gdr2.chunk_bwd(*args, g["d_o"], g["d_final_state"], workspace=ws, saved=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    for n in g1:
        assert torch.equal(g1[n], g2[n]), n
    ref = oracle_bwd(inp)
    for n in GRADS:
        assert_close(n, g2[n], ref[ORACLE_NAMES[n]], dtype)
    assert_close("dS0", g2["dS0"], ref["dS0"], dtype)


def test_split_sequence_resume():
    """fwd over T equals fwd over the first half followed by fwd over the rest from the mid state."""
    wl = workloads.ChunkWorkload("split", B=1, T=320, H=2, dk=128, dv=128, dtype="f32", s0_std=0.2, seed=3)
    inp = workloads.chunk_inputs(wl)
    g = cuda(inp)
    o_full, S_full = gdr2.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["b"], g["w"], g["initial_state"])
    cut = 131
    part = lambda t, a, b: t[:, a:b].contiguous()  # noqa: E731
    o1, S1 = gdr2.chunk_fwd(*(part(g[n], 0, cut) for n in ("q", "k", "v", "log_alpha", "b", "w")), g["initial_state"])
    o2, S2 = gdr2.chunk_fwd(*(part(g[n], cut, 320) for n in ("q", "k", "v", "log_alpha", "b", "w")), S1)
    torch.cuda.synchronize()
    ro, rST = oracle_fwd(inp)
    assert_close("o", torch.cat([o1, o2], dim=1), ro, "f32")
    assert_close("final_state", S2, rST, "f32")
    assert_close("o_full", o_full, ro, "f32")
    assert_close("final_state_full", S_full, rST, "f32")


# --- the chunk-level scan: few chains of many chunks ------------------------------------------------

def _scan_segments(B, T, H):
    """Segments per chain chosen by the library, read back from the workspace size (1: plain pass)."""
    per_chunk = gdr2.workspace_bytes(8, 4096, 16, 128, 128, gdr2.GDR2_BF16, 0) // (8 * 16 * 64)
    extra = gdr2.workspace_bytes(B, T, H, 128, 128, gdr2.GDR2_BF16, 0) - per_chunk * B * H * (-(-T // 64))
    return 1 if extra == 0 else extra // (3 * B * H * 128 * 128 * 4)


@pytest.mark.parametrize("B,T,nseg", [(1, 64 * 24 + 37, 5), (2, 64 * 128 + 19, 10)])
def test_chunk_scan_forward_backward(B, T, nseg):
    """With few (batch, head) chains the serial passes run as a chunk-level scan: segments of chunks
    are reduced to their affine transfer in parallel, combined, and rerun from their start states.
    Every output is compared with the oracle; the last segment is shorter and the last chunk partial.
    The training pair (intermediates kept) gives exactly the recompute path's results."""
    assert _scan_segments(B, T, 2) == nseg
    wl = workloads.ChunkWorkload("scan", B=B, T=T, H=2, dk=128, dv=128, dtype="bf16", s0_std=0.2, neg_eig=True,
                                 backward=True, seed=61 + B)
    inp = workloads.chunk_inputs(wl)
    _check_fwd(inp, "bf16")
    _check_bwd(inp, "bf16")
    g = cuda(inp)
    args = [g[n] for n in ("q", "k", "v", "log_alpha", "b", "w")] + [g["initial_state"]]
    o1, S1 = gdr2.chunk_fwd(*args)
    g1 = gdr2.chunk_bwd(*args, g["d_o"], g["d_final_state"])
    ws = gdr2.alloc_workspace(B, T, 2, 128, 128, gdr2.GDR2_BF16, 1)
    o2, S2 = gdr2.chunk_fwd(*args, workspace=ws, train=True)
    g2 = gdr2.chunk_bwd(*args, g["d_o"], g["d_final_state"], workspace=ws, saved=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    for n in g1:
        assert torch.equal(g1[n], g2[n]), n


# --- full-size workloads, sampled chains ----------------------------------------------------------

def test_fwd_1p3b_layer():
    """B=1, H=16, dk=dv=128, T=4096, bf16 operands: every element of o and the final state."""
    inp = workloads.chunk_inputs(workloads.WORKLOADS["fwd_1p3b"])
    _check_fwd(inp, "bf16")


def test_fwd_1p3b_layer_tied_gates():
    """Scalar decay, b = w = beta*1: the KDA / Gated DeltaNet reduction on the full layer, whole tensors."""
    inp = workloads.chunk_inputs(workloads.WORKLOADS["fwd_1p3b_tied"])
    _check_fwd(inp, "bf16")


def test_train_fwd_bwd_full_size():
    """B=8, H=16, dk=dv=128, T=4096, bf16: the benchmark's workload and launch sequence
    (gdr2_chunk_fwd_train then gdr2_chunk_bwd_saved on one workspace), run whole on the GPU."""
    wl = workloads.WORKLOADS["train_fwd_bwd"]
    inp = workloads.chunk_inputs(wl)
    g = cuda(inp)
    args = [g[n] for n in ("q", "k", "v", "log_alpha", "b", "w")] + [g["initial_state"]]
    ws = gdr2.alloc_workspace(wl.B, wl.T, wl.H, wl.dk, wl.dv, gdr2.GDR2_BF16, 1)
    o, ST = gdr2.chunk_fwd(*args, workspace=ws, train=True)
    out = gdr2.chunk_bwd(*args, g["d_o"], g["d_final_state"], workspace=ws, saved=True)
    torch.cuda.synchronize()
    chains = [(0, 0), (3, 7), (7, 15)]
    sel = select_chains(inp, chains)
    ro, rST = oracle_fwd(sel)
    assert_close("o", gpu_rows(o, chains), ro, "bf16")
    assert_close("final_state", gpu_rows(ST, chains, state=True), rST, "bf16")
    ref = oracle_bwd(sel)
    for n in GRADS:
        assert_close(n, gpu_rows(out[n], chains), ref[ORACLE_NAMES[n]], "bf16")
    assert_close("dS0", gpu_rows(out["dS0"], chains, state=True), ref["dS0"], "bf16")


def test_long_context_negative_eigenvalue():
    """B=1, H=16, T=65536, b in [0, 2], weak decay, non-zero S0, forward and backward (the chunk-level
    scan): every element of every output against the oracle."""
    inp = workloads.chunk_inputs(workloads.WORKLOADS["long_neg_eig"])
    _check_fwd(inp, "bf16")
    _check_bwd(inp, "bf16")


@pytest.mark.parametrize("neg_eig", [False, True])
def test_strong_decay_tensor_core_path(neg_eig):
    """Per-chunk cumulative log-decay between -154 and -96 in every channel (log_alpha in [-2.4, -1.5] per
    token, as Mamba-style gates with A up to 16 give): beyond e^{-80}, where absolute e^{+-G} factors leave
    fp32, but inside the tensor-core path's relative factors. Forward and backward against the oracle, and
    the device status stays clean."""
    wl = workloads.ChunkWorkload("strong", B=1, T=200, H=2, dk=128, dv=128, dtype="bf16", neg_eig=neg_eig,
                                 s0_std=0.3, backward=True, seed=41)
    inp = dict(workloads.chunk_inputs(wl))
    gen = torch.Generator().manual_seed(42)
    inp["log_alpha"] = -(1.5 + 0.9 * torch.rand(inp["log_alpha"].shape, generator=gen))
    gdr2.check()
    _check_fwd(inp, "bf16")
    _check_bwd(inp, "bf16")
    assert gdr2.check() == gdr2.OK
