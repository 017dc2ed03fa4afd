"""GPU parity of the gate and normalisation prologue (gdr2_gate_prologue_fwd / _bwd) against the fp64
oracle (B200 only). Small shapes are compared element by element over every output, for both dtypes,
both head sizes and both ranges of the erase gate; the training-sized prologue is compared whole (one batch
element at a time), with its da / ddelta sums over all 32,768 tokens."""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_65_b200 import gdr2, workloads
from tests.parity import assert_close, cuda

pytestmark = pytest.mark.gpu

X = ("xq", "xk", "xf", "xb", "xw", "a", "delta")
FWD = {"q": "q", "k": "k", "log_alpha": "log_alpha", "b": "b", "w": "w"}
BWD = ("dxq", "dxk", "dxf", "dxb", "dxw", "da", "ddelta")


def _run(inp, neg):
    g = cuda(inp)
    fo = gdr2.gate_prologue_fwd(*(g[n] for n in X), neg_eig=neg)
    bo = gdr2.gate_prologue_bwd(*(g[n] for n in X), g["dq"], g["dk"], g["dlog_alpha"], g["db"], g["dw"], neg_eig=neg)
    torch.cuda.synchronize()
    return fo, bo


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("neg", [False, True])
def test_prologue_small(dtype, dk, dv, neg):
    wl = workloads.PrologueWorkload("small", B=2, T=77, H=3, dk=dk, dv=dv, dtype=dtype, seed=17 + dk + dv)
    inp = workloads.prologue_inputs(wl)
    fo, bo = _run(inp, neg)
    ref = oracle.prologue_fwd(*(inp[n] for n in X), neg_eig=neg)
    for n in FWD:
        assert_close(n, fo[n], ref[n], dtype)
    refb = oracle.prologue_bwd(*(inp[n] for n in X), inp["dq"], inp["dk"], inp["dlog_alpha"], inp["db"], inp["dw"],
                               neg_eig=neg)
    for n in BWD:
        assert_close(n, bo[n], refb[n], dtype)


def test_prologue_zero_rows_and_determinism():
    """A zero pre-activation row gives q = 0 with zero gradient; repeated calls give identical bits."""
    wl = workloads.PrologueWorkload("zero", B=1, T=40, H=2, dtype="f32", seed=3)
    inp = workloads.prologue_inputs(wl)
    inp["xq"][0, 5, 1] = 0.0
    fo, bo = _run(inp, False)
    assert torch.all(fo["q"][0, 5, 1] == 0) and torch.all(bo["dxq"][0, 5, 1] == 0)
    fo2, bo2 = _run(inp, False)
    for n in fo:
        assert torch.equal(fo[n], fo2[n]), n
    for n in bo:
        assert torch.equal(bo[n], bo2[n]), n


def test_prologue_training_size():
    """B=8, T=4096, H=16, d=128, bf16: every element of every output against the oracle, one batch element at a
    time (the fp64 oracle holds one element's tensors at once), and da / ddelta as the sums over all tokens."""
    wl = workloads.PROLOGUE_WORKLOADS["prologue_train"]
    inp = workloads.prologue_inputs(wl)
    fo, bo = _run(inp, False)
    da = np.zeros((wl.H, wl.dk))
    dd = np.zeros((wl.H, wl.dk))
    for b in range(wl.B):
        one = {n: (inp[n][b:b + 1] if n not in ("a", "delta") else inp[n])
               for n in list(X) + ["dq", "dk", "dlog_alpha", "db", "dw"]}
        ref = oracle.prologue_fwd(*(one[n] for n in X))
        for n in FWD:
            assert_close(n, fo[n][b:b + 1], ref[n], "bf16")
        r = oracle.prologue_bwd(*(one[n] for n in X), one["dq"], one["dk"], one["dlog_alpha"], one["db"], one["dw"])
        for n in ("dxq", "dxk", "dxf", "dxb", "dxw"):
            assert_close(n, bo[n][b:b + 1], r[n], "bf16")
        da += r["da"]
        dd += r["ddelta"]
    assert_close("da", bo["da"], da, "f32")
    assert_close("ddelta", bo["ddelta"], dd, "f32")
