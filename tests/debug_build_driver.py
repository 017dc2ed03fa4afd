"""Runs the library's entry points through the debug build (libgdr2_debug.so: the same kernels compiled with
-DGDR2_DEBUG, whose index checks report GDR2_ERR_BOUNDS through gdr2_check instead of trapping), one small
case per kernel family, and checks after each that no index check failed and that the outputs agree with the
fp64 oracle. Started by tests/test_debug_build_gpu.py in a child process with GDR2_DEBUG_BUILD=1, so that the
parent's release library is not replaced. Prints one line per case and exits non-zero on the first failure.
"""
from __future__ import annotations

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import oracle  # noqa: E402
from gated_delta_rule_65_b200 import build as gbuild, gdr2, workloads  # noqa: E402
from tests.parity import assert_close, cuda, oracle_bwd, oracle_fwd  # noqa: E402

GRADS = ("dq", "dk", "dv", "dlog_alpha", "db", "dw")
TOKENS = ("q", "k", "v", "log_alpha", "b", "w")


def status(name):
    torch.cuda.synchronize()
    st = gdr2.check()
    assert st == gdr2.OK, f"{name}: {gdr2.status_string(st)}"
    print(f"{name}: ok", flush=True)


def chunk_case(name, path, B, H, T, saved=True, **kw):
    wl = workloads.ChunkWorkload(name, B=B, T=T, H=H, dk=128, dv=128, dtype="bf16", backward=True, seed=900 + T, **kw)
    inp = workloads.chunk_inputs(wl)
    g = cuda(inp)
    args = [g[n] for n in TOKENS] + [g["initial_state"]]
    gdr2.set_chunk_path(path)
    try:
        if saved:
            ws = gdr2.alloc_workspace(B, T, H, 128, 128, gdr2.GDR2_BF16, 1)
            o, ST = gdr2.chunk_fwd(*args, workspace=ws, train=True)
            out = gdr2.chunk_bwd(*args, g["d_o"], g["d_final_state"], workspace=ws, saved=True)
        else:
            o, ST = gdr2.chunk_fwd(*args)
            out = gdr2.chunk_bwd(*args, g["d_o"], g["d_final_state"])
    finally:
        gdr2.set_chunk_path(gdr2.PATH_AUTO)
    status(name)
    ro, rST = oracle_fwd(inp)
    assert_close("o", o, ro, "bf16")
    assert_close("final_state", ST, rST, "bf16")
    ref = oracle_bwd(inp)
    for n in GRADS:
        assert_close(n, out[n], ref[n], "bf16")


def varlen_case(name, lengths, grouped):
    wl = workloads.VarlenWorkload(name, N=len(lengths), T=sum(lengths), H=2, s0_std=0.2, lengths=tuple(lengths),
                                  seed=901)
    inp = workloads.varlen_inputs(wl)
    g = cuda(inp)
    args = [g[n] for n in TOKENS]
    cu = g["cu_seqlens"]
    if grouped:  # two value heads per key head: the key-side tensors keep every other head
        args = [a[:, ::2].contiguous() if n in ("q", "k", "log_alpha", "b") else a for n, a in zip(TOKENS, args)]
    o, ST = gdr2.chunk_fwd_varlen(*args, cu, g["initial_state"])
    out = gdr2.chunk_bwd_varlen(*args, cu, g["initial_state"], g["d_o"], g["d_final_state"])
    status(name)
    if not grouped:
        ro, rST = oracle.fwd_varlen(*(inp[n] for n in TOKENS), inp["cu_seqlens"], inp["initial_state"])
        assert_close("o", o, ro, "bf16")
        assert_close("final_state", ST, rST, "bf16")
    for n in GRADS:
        assert torch.isfinite(out[n].float()).all(), f"{name}: {n} not finite"


def decode_case(name):
    wl = workloads.DecodeWorkload(name, B=5, H=3, dk=128, dv=128, steps=3, dtype="bf16", seed=902)
    inp = workloads.decode_inputs(wl)
    S = inp["state"].cuda()
    Sref = inp["state"]
    for t in range(wl.steps):
        step = {n: inp[n][t] for n in TOKENS}
        o = gdr2.decode_step(*(step[n].cuda() for n in TOKENS), S)
        ro, Sref = oracle.decode(*(step[n] for n in TOKENS), Sref)
        status(f"{name} step {t}")
        assert_close("o", o, ro, "bf16")
    assert_close("state", S, Sref, "bf16")


def main():
    assert os.environ.get("GDR2_DEBUG_BUILD") == "1"
    L = gdr2.lib()
    assert L._name == gbuild.DEBUG_LIB, L._name
    gdr2.check()
    # per-chain kernels: ragged tail, several chains per CTA, the backward with the forward recomputed
    chunk_case("per-chain", gdr2.PATH_CHAIN, B=2, H=3, T=257, s0_std=0.3, neg_eig=True)
    chunk_case("per-chain, more chains than SMs", gdr2.PATH_CHAIN, B=3, H=60, T=130, saved=False)
    # chunk-parallel kernels, and the chunk-level scan (one long chain)
    chunk_case("chunk-parallel", gdr2.PATH_SPLIT, B=2, H=3, T=257, s0_std=0.3)
    chunk_case("chunk-parallel with the scan", gdr2.PATH_SPLIT, B=1, H=1, T=64 * 40 + 17, s0_std=0.3)
    varlen_case("packed batch", (5, 64, 0, 130, 300), grouped=False)
    varlen_case("packed batch, grouped value heads", (70, 129, 64), grouped=True)
    decode_case("decode")
    print("debug build: all cases ok", flush=True)


if __name__ == "__main__":
    main()
