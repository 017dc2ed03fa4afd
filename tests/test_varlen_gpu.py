"""GPU parity of the packed variable-length entry points (gdr2_chunk_*_varlen) against the fp64 oracle.

A packed batch holds N sequences back to back on one token axis, each with its own initial state and
chunks (review, Appendix C.6). Small batches are compared element by element over every output; they
cover an empty sequence, sequences shorter than a chunk, exactly one chunk, and ragged ends. They are
also compared bit for bit with the unpacked entry points run one sequence at a time: the kernels and
their arithmetic are the same, only the chunk table differs. The full-size packed mix is compared whole.
"""
from __future__ import annotations

import pytest
import torch

import oracle
from gated_delta_rule_65_b200 import gdr2, workloads
from tests.parity import assert_close, cuda

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw")
TOKENS = ("q", "k", "v", "log_alpha", "b", "w")

SMALL = [
    (5, 64, 0, 130, 300),       # short, one chunk, empty, ragged, several chunks
    (200, 63, 65, 128, 1, 7),   # one token, 63 / 65 around a chunk boundary
    (777,),                     # one sequence over the whole axis
]


def _wl(lengths, neg_eig=False, s0=True, seed=0):
    return workloads.VarlenWorkload("varlen_small", N=len(lengths), T=sum(lengths), H=2, neg_eig=neg_eig,
                                    s0_std=0.2 if s0 else None, lengths=tuple(lengths), seed=seed)


def _gpu_pair(g, train):
    args = [g[n] for n in TOKENS]
    cu = g["cu_seqlens"]
    N, T, H = cu.numel() - 1, g["q"].shape[0], g["q"].shape[1]
    if train:
        ws = gdr2.alloc_workspace_varlen(N, T, H, 128, 128, gdr2.GDR2_BF16, 1)
        o, ST = gdr2.chunk_fwd_varlen(*args, cu, g["initial_state"], workspace=ws, train=True)
        out = gdr2.chunk_bwd_varlen(*args, cu, g["initial_state"], g["d_o"], g["d_final_state"], workspace=ws,
                                    saved=True)
    else:
        o, ST = gdr2.chunk_fwd_varlen(*args, cu, g["initial_state"])
        out = gdr2.chunk_bwd_varlen(*args, cu, g["initial_state"], g["d_o"], g["d_final_state"])
    torch.cuda.synchronize()
    return o, ST, out


@pytest.mark.parametrize("lengths", SMALL)
@pytest.mark.parametrize("neg_eig", [False, True])
def test_varlen_small_against_oracle(lengths, neg_eig):
    inp = workloads.varlen_inputs(_wl(lengths, neg_eig=neg_eig, seed=71 + len(lengths)))
    g = cuda(inp)
    o, ST, out = _gpu_pair(g, train=False)
    cu = inp["cu_seqlens"]
    ro, rST = oracle.fwd_varlen(*(inp[n] for n in TOKENS), cu, inp["initial_state"])
    assert_close("o", o, ro, "bf16")
    assert_close("final_state", ST, rST, "bf16")
    ref = oracle.bwd_varlen(*(inp[n] for n in TOKENS), cu, inp["initial_state"], inp["d_o"], inp["d_final_state"])
    for n in GRADS:
        assert_close(n, out[n], ref[n], "bf16")
    assert_close("dS0", out["dS0"], ref["dS0"], "bf16")


@pytest.mark.parametrize("lengths", SMALL[:2])
def test_varlen_matches_unpacked_per_sequence(lengths):
    """Bit-identical to gdr2_chunk_fwd / gdr2_chunk_bwd on each sequence alone (B = 1, T = length)."""
    inp = workloads.varlen_inputs(_wl(lengths, seed=5))
    g = cuda(inp)
    o, ST, out = _gpu_pair(g, train=False)
    cu = inp["cu_seqlens"].tolist()
    for n, (a, e) in enumerate(zip(cu[:-1], cu[1:])):
        if e == a:
            assert torch.equal(ST[n], g["initial_state"][n])
            assert torch.equal(out["dS0"][n], g["d_final_state"][n])
            continue
        sl = [g[x][a:e][None].contiguous() for x in TOKENS]
        s0, dst = g["initial_state"][n:n + 1].contiguous(), g["d_final_state"][n:n + 1].contiguous()
        o1, S1 = gdr2.chunk_fwd(*sl, s0)
        g1 = gdr2.chunk_bwd(*sl, s0, g["d_o"][a:e][None].contiguous(), dst)
        torch.cuda.synchronize()
        assert torch.equal(o[a:e], o1[0]), n
        assert torch.equal(ST[n], S1[0]), n
        for x in GRADS:
            assert torch.equal(out[x][a:e], g1[x][0]), (n, x)
        assert torch.equal(out["dS0"][n], g1["dS0"][0]), n


def test_varlen_training_pair_matches_recompute():
    """gdr2_chunk_fwd_train_varlen + gdr2_chunk_bwd_saved_varlen give exactly the recompute path's results."""
    inp = workloads.varlen_inputs(_wl(SMALL[0], neg_eig=True, seed=9))
    g = cuda(inp)
    o1, S1, g1 = _gpu_pair(g, train=False)
    o2, S2, g2 = _gpu_pair(g, train=True)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    for n in g1:
        assert torch.equal(g1[n], g2[n]), n


def test_varlen_absent_optional_tensors():
    """No initial state, no d_o, no dS_T: zeros stand in for each (oracle with the same Nones)."""
    inp = workloads.varlen_inputs(_wl(SMALL[1], s0=False, seed=13))
    g = cuda(inp)
    args = [g[n] for n in TOKENS]
    cu = g["cu_seqlens"]
    out = gdr2.chunk_bwd_varlen(*args, cu, None, None, g["d_final_state"])
    torch.cuda.synchronize()
    ref = oracle.bwd_varlen(*(inp[n] for n in TOKENS), inp["cu_seqlens"], None, None, inp["d_final_state"])
    for n in GRADS:
        assert_close(n, out[n], ref[n], "bf16")
    assert_close("dS0", out["dS0"], ref["dS0"], "bf16")


def test_varlen_full_size_mix_whole():
    """16 sequences of 358..5986 tokens (32,768 in all), H = 16: the packed batch the benchmark runs, with
    the training pair; every element of every output against the oracle."""
    wl = workloads.VARLEN_WORKLOADS["varlen_mix"]
    inp = workloads.varlen_inputs(wl)
    g = cuda(inp)
    o, ST, out = _gpu_pair(g, train=True)
    ro, rST = oracle.fwd_varlen(*(inp[n] for n in TOKENS), inp["cu_seqlens"], inp["initial_state"])
    assert_close("o", o, ro, "bf16")
    assert_close("final_state", ST, rST, "bf16")
    ref = oracle.bwd_varlen(*(inp[n] for n in TOKENS), inp["cu_seqlens"], inp["initial_state"], inp["d_o"],
                            inp["d_final_state"])
    for x in GRADS:
        assert_close(x, out[x], ref[x], "bf16")
    assert_close("dS0", out["dS0"], ref["dS0"], "bf16")


def test_varlen_many_short_sequences():
    """4,500 sequences of 0..24 tokens (more than the 4,096 the index kernel orders by length, so the serial
    passes take them in their given order): sampled sequences on both sides of index 4,096, empty ones
    included, against the oracle, with the training pair."""
    gen = torch.Generator().manual_seed(4500)
    lengths = torch.randint(0, 25, (4500,), generator=gen)
    lengths[[7, 4096, 4300]] = 0
    lengths[[4095, 4097]] = torch.tensor([24, 17])
    lengths = tuple(int(x) for x in lengths)
    wl = workloads.VarlenWorkload("varlen_many", N=len(lengths), T=sum(lengths), H=1, neg_eig=True,
                                  s0_std=0.2, lengths=lengths, seed=4501)
    inp = workloads.varlen_inputs(wl)
    g = cuda(inp)
    o, ST, out = _gpu_pair(g, train=True)
    cu = inp["cu_seqlens"].tolist()
    for n in (0, 7, 4095, 4096, 4097, 4300, 4499):
        a, e = cu[n], cu[n + 1]
        if e == a:  # an empty sequence passes its state and its state gradient through unchanged
            assert torch.equal(ST[n], g["initial_state"][n])
            assert torch.equal(out["dS0"][n], g["d_final_state"][n])
            continue
        one = {x: inp[x][a:e][None] for x in TOKENS + ("d_o",)}
        s0, dst = inp["initial_state"][n][None], inp["d_final_state"][n][None]
        ro, rST = oracle.fwd(*(one[x] for x in TOKENS), s0)
        assert_close("o", o[a:e][None], ro, "bf16")
        assert_close("final_state", ST[n][None], rST, "bf16")
        ref = oracle.bwd(*(one[x] for x in TOKENS), s0, one["d_o"], dst)
        for x in GRADS:
            assert_close(x, out[x][a:e][None], ref[x], "bf16")
        assert_close("dS0", out["dS0"][n][None], ref["dS0"], "bf16")
