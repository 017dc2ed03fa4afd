"""GPU parity of the grouped-value-head entry points (gdr2_chunk_*_gva) against the fp64 oracle.

Hv = G H value heads share each key head (review, "Headed architecture and grouped-value attention").
Small cases compare every output element by element; the group size 1 is bit-identical to the plain
entry points; the training pair is bit-identical to the recompute path; a long case runs the chunk-level
scan over value-head chains; the training-sized case is compared whole.
"""
from __future__ import annotations

import pytest
import torch

import oracle
from gated_delta_rule_65_b200 import gdr2, workloads
from tests.parity import assert_close, cuda

pytestmark = pytest.mark.gpu

TOK = ("q", "k", "v", "log_alpha", "b", "w")
GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw")


def _inputs(B, T, H, Hv, seed, neg=True):
    wl = workloads.ChunkWorkload("gva", B=B, T=T, H=Hv, dk=128, dv=128, dtype="bf16", neg_eig=neg, s0_std=0.2,
                                 backward=True, seed=seed)
    return workloads.gva_inputs(wl, H)


def _gpu(g, train=False):
    args = [g[n] for n in TOK] + [g["initial_state"]]
    if train:
        B, T, H = g["q"].shape[:3]
        Hv = g["v"].shape[2]
        ws = gdr2.alloc_workspace_gva(B, T, H, Hv, 128, 128, gdr2.GDR2_BF16, 1)
        o, ST = gdr2.chunk_fwd_gva(*args, workspace=ws, train=True)
        out = gdr2.chunk_bwd_gva(*args, g["d_o"], g["d_final_state"], workspace=ws, saved=True)
    else:
        o, ST = gdr2.chunk_fwd_gva(*args)
        out = gdr2.chunk_bwd_gva(*args, g["d_o"], g["d_final_state"])
    torch.cuda.synchronize()
    return o, ST, out


def _check(inp, o, ST, out):
    ro, rST = oracle.fwd_gva(*(inp[n] for n in TOK), inp["initial_state"])
    assert_close("o", o, ro, "bf16")
    assert_close("final_state", ST, rST, "bf16")
    ref = oracle.bwd_gva(*(inp[n] for n in TOK), inp["initial_state"], inp["d_o"], inp["d_final_state"])
    for n in GRADS:
        assert_close(n, out[n], ref[n], "bf16")
    assert_close("dS0", out["dS0"], ref["dS0"], "bf16")


@pytest.mark.parametrize("H,Hv,T", [(2, 4, 200), (2, 6, 130), (1, 4, 64)])
def test_gva_small(H, Hv, T):
    inp = _inputs(2, T, H, Hv, seed=81 + Hv)
    o, ST, out = _gpu(cuda(inp))
    _check(inp, o, ST, out)


def test_gva_group_of_one_is_the_plain_path():
    inp = _inputs(2, 150, 3, 3, seed=7)
    g = cuda(inp)
    o, ST, out = _gpu(g)
    args = [g[n] for n in TOK] + [g["initial_state"]]
    o1, S1 = gdr2.chunk_fwd(*args)
    g1 = gdr2.chunk_bwd(*args, g["d_o"], g["d_final_state"])
    torch.cuda.synchronize()
    assert torch.equal(o, o1) and torch.equal(ST, S1)
    for n in g1:
        assert torch.equal(out[n], g1[n]), n


def test_gva_training_pair_matches_recompute():
    inp = _inputs(2, 200, 2, 4, seed=9)
    g = cuda(inp)
    o1, S1, g1 = _gpu(g)
    o2, S2, g2 = _gpu(g, train=True)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    for n in g1:
        assert torch.equal(g1[n], g2[n]), n


def test_gva_long_sequence_with_scan():
    """B=1, H=2, Hv=4, T=4096 + 37: four value-head chains of 65 chunks run as a chunk-level scan."""
    T = 4096 + 37
    NT = -(-T // 64)
    arrays = (3 * 32768 + 16384 + 512) * 2 * NT + 32768 * 4 * NT  # key-side per key chunk, U per value chunk
    extra = gdr2.workspace_bytes_gva(1, T, 2, 4, 128, 128, gdr2.GDR2_BF16, 0) - arrays
    assert extra > 0 and extra % (3 * 4 * 65536) == 0  # three fp32 states per (segment, value-head chain)
    inp = _inputs(1, T, 2, 4, seed=11)
    o, ST, out = _gpu(cuda(inp), train=True)
    _check(inp, o, ST, out)


def test_gva_training_size_whole():
    """B=8, T=4096, H=8 key heads, Hv=16 value heads (the benchmark's grouped workload), training pair: every
    element of every output against the oracle."""
    wl = workloads.GVA_WORKLOADS["gva_train"]
    H = 8
    inp = workloads.gva_inputs(wl, H)
    o, ST, out = _gpu(cuda(inp), train=True)
    ro, rST = oracle.fwd_gva(*(inp[n] for n in TOK), inp["initial_state"])
    assert_close("o", o, ro, "bf16")
    assert_close("final_state", ST, rST, "bf16")
    ref = oracle.bwd_gva(*(inp[n] for n in TOK), inp["initial_state"], inp["d_o"], inp["d_final_state"])
    for n in ("dq", "dk", "dlog_alpha", "db", "dv", "dw"):
        assert_close(n, out[n], ref[n], "bf16")
    assert_close("dS0", out["dS0"], ref["dS0"], "bf16")


# ---- packed variable-length batches with grouped value heads --------------------------------------------
VL_LENGTHS = [(5, 64, 0, 130, 300), (200, 63, 65, 1)]


def _varlen_inputs(lengths, H, Hv, seed):
    """A packed batch drawn like the grouped-head case (B = 1, T = sum of lengths), with one initial state
    and one final-state gradient per (sequence, value head)."""
    wl = workloads.ChunkWorkload("vgva", B=1, T=sum(lengths), H=Hv, dk=128, dv=128, dtype="bf16", neg_eig=True,
                                 backward=True, seed=seed)
    inp = workloads.gva_inputs(wl, H)
    out = {n: inp[n][0] for n in TOK + ("d_o",)}
    gen = torch.Generator().manual_seed(seed + 1)
    out["initial_state"] = 0.2 * torch.randn(len(lengths), Hv, 128, 128, generator=gen)
    out["d_final_state"] = torch.randn(len(lengths), Hv, 128, 128, generator=gen)
    cu = [0]
    for x in lengths:
        cu.append(cu[-1] + x)
    out["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32)
    return out


def _gpu_varlen(g, train=False):
    args = [g[n] for n in TOK]
    cu = g["cu_seqlens"]
    if train:
        N, T, H, Hv = cu.numel() - 1, g["q"].shape[0], g["q"].shape[1], g["v"].shape[1]
        ws = gdr2.alloc_workspace_varlen(N, T, H, 128, 128, gdr2.GDR2_BF16, 1, Hv=Hv)
        o, ST = gdr2.chunk_fwd_varlen(*args, cu, g["initial_state"], workspace=ws, train=True)
        out = gdr2.chunk_bwd_varlen(*args, cu, g["initial_state"], g["d_o"], g["d_final_state"], workspace=ws,
                                    saved=True)
    else:
        o, ST = gdr2.chunk_fwd_varlen(*args, cu, g["initial_state"])
        out = gdr2.chunk_bwd_varlen(*args, cu, g["initial_state"], g["d_o"], g["d_final_state"])
    torch.cuda.synchronize()
    return o, ST, out


@pytest.mark.parametrize("lengths", VL_LENGTHS)
@pytest.mark.parametrize("H,Hv", [(2, 4), (1, 3)])
def test_varlen_gva_against_oracle(lengths, H, Hv):
    """Every sequence of the packed batch against the oracle's grouped-head calls on that sequence alone."""
    inp = _varlen_inputs(lengths, H, Hv, seed=301 + 7 * Hv + len(lengths))
    g = cuda(inp)
    o, ST, out = _gpu_varlen(g, train=True)
    assert gdr2.check() == gdr2.OK
    cu = inp["cu_seqlens"].tolist()
    for n, (a, e) in enumerate(zip(cu[:-1], cu[1:])):
        if e == a:  # an empty sequence passes its state and its state gradient through unchanged
            assert torch.equal(ST[n], g["initial_state"][n])
            assert torch.equal(out["dS0"][n], g["d_final_state"][n])
            continue
        one = {x: inp[x][a:e][None] for x in TOK + ("d_o",)}
        s0, dst = inp["initial_state"][n][None], inp["d_final_state"][n][None]
        ro, rST = oracle.fwd_gva(*(one[x] for x in TOK), s0)
        assert_close("o", o[a:e][None], ro, "bf16")
        assert_close("final_state", ST[n][None], rST, "bf16")
        ref = oracle.bwd_gva(*(one[x] for x in TOK), s0, one["d_o"], dst)
        for x in GRADS:
            assert_close(x, out[x][a:e][None], ref[x], "bf16")
        assert_close("dS0", out["dS0"][n][None], ref["dS0"], "bf16")


def test_varlen_gva_matches_unpacked_per_sequence():
    """Bit-identical to the grouped-head calls run on each sequence alone (B = 1, T = its length), and the
    recompute backward bit-identical to the training pair."""
    inp = _varlen_inputs(VL_LENGTHS[0], 2, 4, seed=333)
    g = cuda(inp)
    o, ST, out = _gpu_varlen(g)
    o2, S2, out2 = _gpu_varlen(g, train=True)
    assert torch.equal(o, o2) and torch.equal(ST, S2)
    for x in out:
        assert torch.equal(out[x], out2[x]), x
    cu = inp["cu_seqlens"].tolist()
    for n, (a, e) in enumerate(zip(cu[:-1], cu[1:])):
        if e == a:
            continue
        sl = [g[x][a:e][None].contiguous() for x in TOK]
        s0, dst = g["initial_state"][n:n + 1].contiguous(), g["d_final_state"][n:n + 1].contiguous()
        o1, S1 = gdr2.chunk_fwd_gva(*sl, s0)
        g1 = gdr2.chunk_bwd_gva(*sl, s0, g["d_o"][a:e][None].contiguous(), dst)
        torch.cuda.synchronize()
        assert torch.equal(o[a:e], o1[0]), n
        assert torch.equal(ST[n], S1[0]), n
        for x in GRADS:
            assert torch.equal(out[x][a:e], g1[x][0]), (n, x)
        assert torch.equal(out["dS0"][n], g1["dS0"][0]), n
