"""GPU parity of gdr2_decode_step against the fp64 oracle (B200 only)."""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_65_b200 import gdr2, workloads
from tests.parity import assert_close, cuda, oracle_fwd

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dk,dv,dtype", [(128, 128, "bf16"), (64, 64, "f32"), (128, 256, "f32"), (64, 192, "bf16")])
def test_decode_small(dk, dv, dtype):
    wl = workloads.DecodeWorkload("small", B=3, H=5, dk=dk, dv=dv, steps=7, dtype=dtype, seed=21)
    inp = workloads.decode_inputs(wl)
    g = cuda(inp)
    S = g["state"].clone()
    Sref = inp["state"]
    path = "f32" if dtype == "f32" else "bf16"
    for t in range(wl.steps):
        o = gdr2.decode_step(g["q"][t], g["k"][t], g["v"][t], g["log_alpha"][t], g["b"][t], g["w"][t], S)
        ro, Sref = oracle.decode(inp["q"][t], inp["k"][t], inp["v"][t], inp["log_alpha"][t], inp["b"][t],
                                 inp["w"][t], Sref)
        torch.cuda.synchronize()
        assert_close(f"o[{t}]", o, ro, path)
    assert_close("state", S, Sref, path)


def test_decode_256x16_100_steps_whole():
    """Batch 256 x H=16 fp32 state, 100 consecutive steps on the full state: o of every head at every step
    and the whole final state against the oracle stepped the same way."""
    wl = workloads.DECODE_WORKLOADS["decode_256x16"]
    inp = workloads.decode_inputs(wl)
    g = cuda(inp)
    S = g["state"].clone()
    os_ = []
    for t in range(wl.steps):
        o = gdr2.decode_step(g["q"][t], g["k"][t], g["v"][t], g["log_alpha"][t], g["b"][t], g["w"][t], S)
        os_.append(o.cpu())
    torch.cuda.synchronize()
    # the 100 steps of one (sequence, head) are the token recurrence over T = 100 from the initial state: the
    # oracle's sequence form (one thread per chain) gives every step's o and the final state at once
    seq = {n: inp[n].transpose(0, 1).contiguous() for n in ("q", "k", "v", "log_alpha", "b", "w")}
    ro, Sref = oracle.fwd(seq["q"], seq["k"], seq["v"], seq["log_alpha"], seq["b"], seq["w"], inp["state"])
    for t in range(wl.steps):
        assert_close(f"o[{t}]", os_[t], ro[:, t], "bf16")
    assert_close("state", S, Sref, "bf16")


def test_prefill_then_decode():
    """Chunk forward over a prompt, then decode steps from its final state, equals the oracle run over
    the whole sequence (state hand-off between the two entry points)."""
    wl = workloads.ChunkWorkload("handoff", B=2, T=150, H=2, dk=128, dv=128, dtype="f32", s0_std=0.1, seed=31)
    inp = workloads.chunk_inputs(wl)
    g = cuda(inp)
    P = 140
    cut = {n: g[n][:, :P].contiguous() for n in ("q", "k", "v", "log_alpha", "b", "w")}
    o_p, S = gdr2.chunk_fwd(cut["q"], cut["k"], cut["v"], cut["log_alpha"], cut["b"], cut["w"], g["initial_state"])
    outs = [o_p]
    for t in range(P, 150):
        step = {n: g[n][:, t].contiguous() for n in ("q", "k", "v", "log_alpha", "b", "w")}
        outs.append(gdr2.decode_step(step["q"], step["k"], step["v"], step["log_alpha"], step["b"], step["w"],
                                     S)[:, None])
    torch.cuda.synchronize()
    ro, rST = oracle_fwd(inp)
    assert_close("o", torch.cat(outs, dim=1), ro, "f32")
    assert_close("final_state", S, rST, "f32")
