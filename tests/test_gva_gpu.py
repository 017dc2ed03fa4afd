"""GPU parity of the grouped-value-head entry points (gdr2_chunk_*_gva) against the fp64 oracle.

Hv = G H value heads share each key head (review, "Headed architecture and grouped-value attention").
Small cases compare every output element by element; the group size 1 is bit-identical to the plain
entry points; the training pair is bit-identical to the recompute path; a long case runs the chunk-level
scan over value-head chains; the training-sized case compares sampled key-head groups in full.
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


def test_gva_training_size_sampled():
    """B=8, T=4096, H=8 key heads, Hv=16 value heads (the benchmark's grouped workload); the groups of
    (batch, key head) (0, 0), (5, 3) and (7, 7) are recomputed by the oracle in full."""
    wl = workloads.GVA_WORKLOADS["gva_train"]
    H = 8
    inp = workloads.gva_inputs(wl, H)
    o, ST, out = _gpu(cuda(inp), train=True)
    G = wl.H // H
    for b, h in [(0, 0), (5, 3), (7, 7)]:
        vs = slice(h * G, (h + 1) * G)
        one = {n: inp[n][b:b + 1, :, h:h + 1] for n in ("q", "k", "log_alpha", "b")}
        one.update({n: inp[n][b:b + 1, :, vs] for n in ("v", "w", "d_o")})
        s0 = inp["initial_state"][b:b + 1, vs]
        dst = inp["d_final_state"][b:b + 1, vs]
        ro, rST = oracle.fwd_gva(*(one[n] for n in TOK), s0)
        assert_close("o", o[b:b + 1, :, vs], ro, "bf16")
        assert_close("final_state", ST[b:b + 1, vs], rST, "bf16")
        ref = oracle.bwd_gva(*(one[n] for n in TOK), s0, one["d_o"], dst)
        for n in ("dq", "dk", "dlog_alpha", "db"):
            assert_close(n, out[n][b:b + 1, :, h:h + 1], ref[n], "bf16")
        for n in ("dv", "dw"):
            assert_close(n, out[n][b:b + 1, :, vs], ref[n], "bf16")
        assert_close("dS0", out["dS0"][b:b + 1, vs], ref["dS0"], "bf16")
