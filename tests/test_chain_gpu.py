"""GPU parity of the per-chain fused chunk kernels (gdr2_set_chunk_path(1)) against the fp64 oracle (B200 only).

The per-chain path walks each (batch, head) chain's chunks inside one CTA, forward in order and backward in
reverse. These tests force it on small shapes (ragged tails, several chains per CTA, initial states, negative
eigenvalues, strong decay, absent upstream gradients) and compare every output element with the oracle, for
the backward both with the forward recomputed (gdr2_chunk_bwd) and from the training pair's record
(gdr2_chunk_fwd_train + gdr2_chunk_bwd_saved); the full-size training batch is compared whole.
"""
from __future__ import annotations

import contextlib

import pytest
import torch

from gated_delta_rule_65_b200 import gdr2, workloads
from tests.parity import assert_close, cuda, oracle_bwd, oracle_fwd

pytestmark = pytest.mark.gpu


@contextlib.contextmanager
def chunk_path(path):
    old = gdr2.get_chunk_path()
    gdr2.set_chunk_path(path)
    try:
        yield
    finally:
        gdr2.set_chunk_path(old)


def _fwd(inp, path=gdr2.PATH_CHAIN):
    g = cuda(inp)
    with chunk_path(path):
        o, ST = gdr2.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["b"], g["w"], g["initial_state"])
        torch.cuda.synchronize()
    return o, ST


def _check_fwd(inp):
    gdr2.check()
    o, ST = _fwd(inp)
    assert gdr2.check() == gdr2.OK
    ro, rST = oracle_fwd(inp)
    assert_close("o", o, ro, "bf16")
    assert_close("final_state", ST, rST, "bf16")


SMALL = [
    # (B, H, T, with_s0, neg_eig)
    (1, 1, 1, False, False),
    (1, 2, 63, True, False),
    (2, 3, 64, False, True),
    (2, 3, 65, True, True),
    (1, 2, 130, True, False),
    (2, 2, 257, False, False),
    (1, 3, 700, True, True),
]


@pytest.mark.parametrize("B,H,T,with_s0,neg_eig", SMALL)
def test_chain_forward_small(B, H, T, with_s0, neg_eig):
    wl = workloads.ChunkWorkload("chain_small", B=B, T=T, H=H, dk=128, dv=128, dtype="bf16", neg_eig=neg_eig,
                                 s0_std=0.5 if with_s0 else None, seed=300 + T)
    _check_fwd(workloads.chunk_inputs(wl))


def test_chain_forward_more_chains_than_sms():
    """B*H = 300 chains on at most one CTA per SM: each CTA walks several chains."""
    wl = workloads.ChunkWorkload("chain_many", B=3, T=130, H=100, dk=128, dv=128, dtype="bf16", s0_std=0.2,
                                 seed=301)
    _check_fwd(workloads.chunk_inputs(wl))


@pytest.mark.parametrize("neg_eig", [False, True])
def test_chain_forward_strong_decay(neg_eig):
    """log_alpha in [-2.4, -1.5] per token: per-chunk cumulative decay of -154 ... -96, inside the range of
    the hi / lo relative factors of the T and A_qk product."""
    wl = workloads.ChunkWorkload("chain_strong", B=1, T=200, H=2, dk=128, dv=128, dtype="bf16", neg_eig=neg_eig,
                                 s0_std=0.3, seed=41)
    inp = dict(workloads.chunk_inputs(wl))
    gen = torch.Generator().manual_seed(42)
    inp["log_alpha"] = -(1.5 + 0.9 * torch.rand(inp["log_alpha"].shape, generator=gen))
    _check_fwd(inp)


def _format_mix(inp, case):
    """Inputs whose chunks take the hi / lo relative operands (or a mix of both formats along the chain):
    queries scaled past the single-fp16 bound (keys stay unit-norm: with b up to 2, longer keys make the
    recurrence itself diverge), queries scaled below its scale floor, or strong decay in every other
    64-token chunk."""
    inp = dict(inp)
    if case == "large_q":
        inp["q"] = (inp["q"].float() * 8.0).to(inp["q"].dtype)
    elif case == "small_q":
        inp["q"] = (inp["q"].float() * 0.01).to(inp["q"].dtype)
    else:  # alternating chunks
        T = inp["log_alpha"].shape[1]
        strong = ((torch.arange(T) // 64) % 2 == 1).view(1, T, 1, 1)
        gen = torch.Generator().manual_seed(43)
        hard = -(1.0 + 0.8 * torch.rand(inp["log_alpha"].shape, generator=gen))
        inp["log_alpha"] = torch.where(strong, hard, inp["log_alpha"])
    return inp


@pytest.mark.parametrize("case", ["large_q", "small_q", "alternating"])
def test_chain_forward_relative_formats(case):
    wl = workloads.ChunkWorkload("chain_fmt", B=2, T=300, H=2, dk=128, dv=128, dtype="bf16", s0_std=0.3,
                                 neg_eig=True, seed=44)
    _check_fwd(_format_mix(workloads.chunk_inputs(wl), case))


def test_chain_forward_tied_gates():
    """Scalar decay and b = w = beta 1 (the KDA / Gated DeltaNet reduction)."""
    wl = workloads.ChunkWorkload("chain_tied", B=2, T=300, H=2, dk=128, dv=128, dtype="bf16", tied=True,
                                 seed=302)
    _check_fwd(workloads.chunk_inputs(wl))


def test_chain_forward_training_batch_whole():
    """B=8, H=16, T=4096 (the training batch; automatic path selection picks the per-chain kernels):
    every element of o and of the final state against the oracle."""
    inp = workloads.chunk_inputs(workloads.WORKLOADS["train_fwd_bwd"])
    g = cuda(inp)
    gdr2.check()
    with chunk_path(gdr2.PATH_AUTO):
        o, ST = gdr2.chunk_fwd(g["q"], g["k"], g["v"], g["log_alpha"], g["b"], g["w"], g["initial_state"])
    torch.cuda.synchronize()
    assert gdr2.check() == gdr2.OK
    ro, rST = oracle_fwd(inp)
    assert_close("o", o, ro, "bf16")
    assert_close("final_state", ST, rST, "bf16")


GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw")


def _bwd(inp, saved, path=gdr2.PATH_CHAIN):
    g = cuda(inp)
    args = [g[n] for n in ("q", "k", "v", "log_alpha", "b", "w")] + [g["initial_state"]]
    B, T, H, dk = g["q"].shape
    with chunk_path(path):
        if saved:
            ws = gdr2.alloc_workspace(B, T, H, dk, g["v"].shape[-1], gdr2.GDR2_BF16, 1)
            o, ST = gdr2.chunk_fwd(*args, workspace=ws, train=True)
            out = gdr2.chunk_bwd(*args, g.get("d_o"), g.get("d_final_state"), workspace=ws, saved=True)
        else:
            o, ST = gdr2.chunk_fwd(*args)
            out = gdr2.chunk_bwd(*args, g.get("d_o"), g.get("d_final_state"))
        torch.cuda.synchronize()
    return o, ST, out


def _check_bwd(inp, saved):
    gdr2.check()
    o, ST, out = _bwd(inp, saved)
    assert gdr2.check() == gdr2.OK
    ro, rST = oracle_fwd(inp)
    assert_close("o", o, ro, "bf16")
    assert_close("final_state", ST, rST, "bf16")
    ref = oracle_bwd(inp)
    for n in GRADS:
        assert_close(n, out[n], ref[n], "bf16")
    assert_close("dS0", out["dS0"], ref["dS0"], "bf16")


@pytest.mark.parametrize("saved", [True, False])
@pytest.mark.parametrize("B,H,T,with_s0,neg_eig", SMALL)
def test_chain_backward_small(B, H, T, with_s0, neg_eig, saved):
    wl = workloads.ChunkWorkload("chain_small_bwd", B=B, T=T, H=H, dk=128, dv=128, dtype="bf16", neg_eig=neg_eig,
                                 s0_std=0.5 if with_s0 else None, backward=True, seed=400 + T)
    _check_bwd(workloads.chunk_inputs(wl), saved)


@pytest.mark.parametrize("drop", ["d_o", "d_final_state"])
def test_chain_backward_absent_upstream(drop):
    wl = workloads.ChunkWorkload("chain_nograd", B=2, T=300, H=3, dk=128, dv=128, dtype="bf16", s0_std=0.3,
                                 neg_eig=True, backward=True, seed=23)
    inp = dict(workloads.chunk_inputs(wl))
    inp[drop] = None
    _check_bwd(inp, True)


def test_chain_backward_more_chains_than_sms():
    wl = workloads.ChunkWorkload("chain_many_bwd", B=3, T=130, H=100, dk=128, dv=128, dtype="bf16", s0_std=0.2,
                                 backward=True, seed=302)
    _check_bwd(workloads.chunk_inputs(wl), True)


@pytest.mark.parametrize("neg_eig", [False, True])
def test_chain_backward_strong_decay(neg_eig):
    wl = workloads.ChunkWorkload("chain_strong_bwd", B=1, T=200, H=2, dk=128, dv=128, dtype="bf16",
                                 neg_eig=neg_eig, s0_std=0.3, backward=True, seed=41)
    inp = dict(workloads.chunk_inputs(wl))
    gen = torch.Generator().manual_seed(42)
    inp["log_alpha"] = -(1.5 + 0.9 * torch.rand(inp["log_alpha"].shape, generator=gen))
    _check_bwd(inp, True)


@pytest.mark.parametrize("case", ["large_q", "small_q", "alternating"])
def test_chain_backward_relative_formats(case):
    wl = workloads.ChunkWorkload("chain_fmt_bwd", B=2, T=300, H=2, dk=128, dv=128, dtype="bf16", s0_std=0.3,
                                 neg_eig=True, backward=True, seed=45)
    _check_bwd(_format_mix(workloads.chunk_inputs(wl), case), True)


def test_chain_train_pair_training_batch_whole():
    """B=8, H=16, T=4096: gdr2_chunk_fwd_train then gdr2_chunk_bwd_saved on one workspace (the benchmark's
    step), every element of every output against the oracle."""
    inp = workloads.chunk_inputs(workloads.WORKLOADS["train_fwd_bwd"])
    gdr2.check()
    o, ST, out = _bwd(inp, True)
    assert gdr2.check() == gdr2.OK
    ro, rST = oracle_fwd(inp)
    assert_close("o", o, ro, "bf16")
    assert_close("final_state", ST, rST, "bf16")
    ref = oracle_bwd(inp)
    for n in GRADS:
        assert_close(n, out[n], ref[n], "bf16")
    assert_close("dS0", out["dS0"], ref["dS0"], "bf16")
