"""Seeded synthetic inputs for the Gated Delta Rule-2 mixer (shared by tests, smoke and bench).

This module draws random tensors with the shapes and distributions of the workloads below and
nothing else: it holds none of the mixer's arithmetic, and both the CUDA path and the CPU oracle
receive the very same tensors from it.

Distributions (the 1.3B-layer setting of "Gated DeltaNet-2: Decoupling Erase and Write in Linear
Attention": 16 heads, dk = dv = 128, i.e. 262,144 state floats per layer, 4K training length;
gates as in the review's "Gate Parameterization" section, Eqs. 11-12):
  q, k  ~ N(0, 1), then L2-normalised per (token, head)   (the block L2-normalises q and k)
  v     ~ N(0, 1)
  log_alpha = -decay_scale * softplus(N(0, 1))            (log-decay g <= 0, alpha = exp(g))
  b     = sigmoid(N(0, 1)), or 2 * sigmoid(N(0, 1)) for the negative-eigenvalue variant
  w     = sigmoid(N(0, 1))
  initial state ~ N(0, s0_std^2) or absent (zeros); upstream gradients dO, dS_T ~ N(0, 1).

For bf16 workloads every operand is drawn in fp32 and rounded to bf16 once; log_alpha is also
rounded to a bf16-representable value but kept in an fp32 tensor (the library takes fp32 decay),
so the oracle and the GPU see identical numbers. Generation uses a torch CPU generator seeded with
``seed``; the draw order is fixed (q, k, v, log_alpha, b, w, initial state, dO, dS_T).

Gate prologue inputs (the branch pre-activations of "Gate Parameterization" and "Block Design"):
x_q, x_k, x_f, x_b, x_w ~ N(0, 1); a = ln(0.1) + 0.3 N(0, 1) and delta = 0.5 N(0, 1) per (head, key
channel), so that g = -exp(a) softplus(x_f + delta) sits near the -0.1 softplus(N(0, 1)) of the mixer
workloads; upstream gradients ~ N(0, 1).

Packed variable-length batches (review, Appendix C.6) stand in for a packed pre-training batch: N
sequence lengths drawn log-uniformly over a 64x range and scaled to sum to T (at least min_len each,
seeded), the token tensors drawn as one [T, H, d] batch with the distributions above, and one initial
state and one dS_T per sequence.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclass(frozen=True)
class ChunkWorkload:
    name: str
    B: int
    T: int
    H: int
    dk: int
    dv: int
    dtype: str               # "f32" or "bf16": operand dtype of q, k, v, b, w (and of o, dq, ...)
    decay_scale: float = 0.1
    neg_eig: bool = False    # erase gate in [0, 2]
    s0_std: float | None = None
    tied: bool = False       # scalar decay and b = w = beta * 1 (KDA / Gated DeltaNet reduction)
    backward: bool = False
    seed: int = 0


@dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    H: int
    dk: int
    dv: int
    steps: int
    dtype: str
    s0_std: float = 0.02
    seed: int = 0


WORKLOADS = {
    "tiny_f32": ChunkWorkload("tiny_f32", B=1, T=256, H=2, dk=64, dv=64, dtype="f32",
                              backward=True, seed=1000),
    "fwd_1p3b": ChunkWorkload("fwd_1p3b", B=1, T=4096, H=16, dk=128, dv=128, dtype="bf16", seed=1001),
    "fwd_1p3b_tied": ChunkWorkload("fwd_1p3b_tied", B=1, T=4096, H=16, dk=128, dv=128, dtype="bf16",
                                   tied=True, seed=1011),
    "train_fwd_bwd": ChunkWorkload("train_fwd_bwd", B=8, T=4096, H=16, dk=128, dv=128, dtype="bf16",
                                   backward=True, seed=1002),
    "long_neg_eig": ChunkWorkload("long_neg_eig", B=1, T=65536, H=16, dk=128, dv=128, dtype="bf16",
                                  decay_scale=0.02, neg_eig=True, s0_std=0.02, backward=True, seed=1004),
}

@dataclass(frozen=True)
class VarlenWorkload:
    name: str
    N: int                   # sequences
    T: int                   # packed tokens
    H: int
    dtype: str = "bf16"
    min_len: int = 1
    decay_scale: float = 0.1
    neg_eig: bool = False
    s0_std: float | None = 0.02
    backward: bool = True
    lengths: tuple = ()      # explicit lengths summing to T; drawn when empty
    seed: int = 0


VARLEN_WORKLOADS = {
    # as many tokens as the 8 x 4096 training batch, in 16 sequences of mixed length
    "varlen_mix": VarlenWorkload("varlen_mix", N=16, T=32768, H=16, min_len=64, seed=1005),
}

DECODE_WORKLOADS = {
    "decode_256x16": DecodeWorkload("decode_256x16", B=256, H=16, dk=128, dv=128, steps=100,
                                    dtype="bf16", seed=1003),
}


def _round(x: torch.Tensor, dtype: str) -> torch.Tensor:
    return x.to(DTYPES[dtype])


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-12)


def chunk_inputs(wl: ChunkWorkload, *, B: int | None = None, T: int | None = None,
                 seed: int | None = None, gen_device: str = "cpu") -> dict:
    """Draw one instance of ``wl`` (optionally with B, T or seed overridden).

    Returns a dict of CPU tensors: q, k, v, b, w (operand dtype), log_alpha (fp32),
    initial_state (fp32 or None), and, when ``wl.backward``, d_o (operand dtype) and
    d_final_state (fp32).
    """
    B = wl.B if B is None else B
    T = wl.T if T is None else T
    g = torch.Generator(device=gen_device)
    g.manual_seed(wl.seed if seed is None else seed)
    H, dk, dv = wl.H, wl.dk, wl.dv

    def n(*shape):
        return torch.randn(*shape, generator=g, device=gen_device, dtype=torch.float32)

    q = _l2n(n(B, T, H, dk))
    k = _l2n(n(B, T, H, dk))
    v = n(B, T, H, dv)
    if wl.tied:
        la = (-wl.decay_scale * torch.nn.functional.softplus(n(B, T, H, 1))).expand(B, T, H, dk)
        beta = torch.sigmoid(n(B, T, H, 1))
        b = beta.expand(B, T, H, dk)
        w = beta.expand(B, T, H, dv)
    else:
        la = -wl.decay_scale * torch.nn.functional.softplus(n(B, T, H, dk))
        b = torch.sigmoid(n(B, T, H, dk))
        if wl.neg_eig:
            b = 2.0 * b
        w = torch.sigmoid(n(B, T, H, dv))
    S0 = None
    if wl.s0_std is not None:
        S0 = wl.s0_std * n(B, H, dk, dv)
    out = {
        "q": _round(q, wl.dtype).contiguous(), "k": _round(k, wl.dtype).contiguous(),
        "v": _round(v, wl.dtype).contiguous(),
        "log_alpha": _round(la, wl.dtype).float().contiguous(),
        "b": _round(b, wl.dtype).contiguous(), "w": _round(w, wl.dtype).contiguous(),
        "initial_state": None if S0 is None else S0.contiguous(),
    }
    if wl.backward:
        out["d_o"] = _round(n(B, T, H, dv), wl.dtype).contiguous()
        out["d_final_state"] = n(B, H, dk, dv).contiguous()
    return out


def decode_inputs(wl: DecodeWorkload, *, B: int | None = None, steps: int | None = None,
                  seed: int | None = None) -> dict:
    """Draw ``steps`` single-token inputs and the initial fp32 state for ``wl``.

    Returns q, k, b, log_alpha [steps, B, H, dk], v, w [steps, B, H, dv] and state [B, H, dk, dv].
    """
    B = wl.B if B is None else B
    steps = wl.steps if steps is None else steps
    g = torch.Generator()
    g.manual_seed(wl.seed if seed is None else seed)
    H, dk, dv = wl.H, wl.dk, wl.dv

    def n(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32)

    state = wl.s0_std * n(B, H, dk, dv)
    q = _l2n(n(steps, B, H, dk))
    k = _l2n(n(steps, B, H, dk))
    v = n(steps, B, H, dv)
    la = -0.1 * torch.nn.functional.softplus(n(steps, B, H, dk))
    b = torch.sigmoid(n(steps, B, H, dk))
    w = torch.sigmoid(n(steps, B, H, dv))
    return {
        "q": _round(q, wl.dtype).contiguous(), "k": _round(k, wl.dtype).contiguous(),
        "v": _round(v, wl.dtype).contiguous(),
        "log_alpha": _round(la, wl.dtype).float().contiguous(),
        "b": _round(b, wl.dtype).contiguous(), "w": _round(w, wl.dtype).contiguous(),
        "state": state.contiguous(),
    }


def varlen_lengths(wl: VarlenWorkload) -> list[int]:
    """Sequence lengths of ``wl``: explicit, or N log-uniform draws over a 64x range scaled to sum to T
    (each at least min_len; the rounding remainder goes to the first sequences)."""
    if wl.lengths:
        assert sum(wl.lengths) == wl.T and len(wl.lengths) == wl.N
        return list(wl.lengths)
    g = torch.Generator()
    g.manual_seed(wl.seed + 7)
    x = torch.exp(torch.rand(wl.N, generator=g, dtype=torch.float64) * math.log(64.0))
    free = wl.T - wl.N * wl.min_len
    lens = [wl.min_len + int(math.floor(float(v))) for v in x / x.sum() * free]
    for i in range(wl.T - sum(lens)):
        lens[i % wl.N] += 1
    return lens


def varlen_inputs(wl: VarlenWorkload, *, gen_device: str = "cpu") -> dict:
    """Draw one packed batch: token tensors [T, H, 128] (q, k, v, b, w in the operand dtype, log_alpha
    fp32), cu_seqlens int32 [N + 1], initial_state [N, H, 128, 128] (or None) and, with ``backward``,
    d_o [T, H, 128] and d_final_state [N, H, 128, 128]."""
    cw = ChunkWorkload(wl.name, B=1, T=wl.T, H=wl.H, dk=128, dv=128, dtype=wl.dtype,
                       decay_scale=wl.decay_scale, neg_eig=wl.neg_eig, backward=wl.backward, seed=wl.seed)
    inp = chunk_inputs(cw, gen_device=gen_device)
    out = {n: inp[n][0] for n in ("q", "k", "v", "log_alpha", "b", "w")}
    g = torch.Generator(device=gen_device)
    g.manual_seed(wl.seed + 1)
    out["initial_state"] = (None if wl.s0_std is None else
                            wl.s0_std * torch.randn(wl.N, wl.H, 128, 128, generator=g, device=gen_device))
    if wl.backward:
        out["d_o"] = inp["d_o"][0]
        out["d_final_state"] = torch.randn(wl.N, wl.H, 128, 128, generator=g, device=gen_device)
    lens = varlen_lengths(wl)
    cu = [0]
    for x in lens:
        cu.append(cu[-1] + x)
    out["cu_seqlens"] = torch.tensor(cu, dtype=torch.int32, device=gen_device)
    return out


@dataclass(frozen=True)
class PrologueWorkload:
    name: str
    B: int
    T: int
    H: int
    dk: int = 128
    dv: int = 128
    dtype: str = "bf16"
    neg_eig: bool = False
    seed: int = 0


PROLOGUE_WORKLOADS = {
    # the gate prologue of the training batch (B=8, H=16, T=4096)
    "prologue_train": PrologueWorkload("prologue_train", B=8, T=4096, H=16, seed=1006),
}


def prologue_inputs(wl: PrologueWorkload, *, gen_device: str = "cpu") -> dict:
    """Draw x_q, x_k, x_f, x_b [B,T,H,dk] and x_w [B,T,H,dv] (operand dtype), a and delta [H,dk] (fp32)
    and the upstream gradients dq, dk, db, dw (operand dtype) and dlog_alpha (fp32)."""
    g = torch.Generator(device=gen_device)
    g.manual_seed(wl.seed)
    B, T, H, dk, dv = wl.B, wl.T, wl.H, wl.dk, wl.dv

    def n(*shape):
        return torch.randn(*shape, generator=g, device=gen_device, dtype=torch.float32)

    out = {"xq": n(B, T, H, dk), "xk": n(B, T, H, dk), "xf": n(B, T, H, dk), "xb": n(B, T, H, dk),
           "xw": n(B, T, H, dv)}
    out = {k: _round(v, wl.dtype).contiguous() for k, v in out.items()}
    out["a"] = (math.log(0.1) + 0.3 * n(H, dk)).contiguous()
    out["delta"] = (0.5 * n(H, dk)).contiguous()
    out["dq"] = _round(n(B, T, H, dk), wl.dtype).contiguous()
    out["dk"] = _round(n(B, T, H, dk), wl.dtype).contiguous()
    out["dlog_alpha"] = n(B, T, H, dk).contiguous()
    out["db"] = _round(n(B, T, H, dk), wl.dtype).contiguous()
    out["dw"] = _round(n(B, T, H, dv), wl.dtype).contiguous()
    return out


GVA_WORKLOADS = {
    # the training batch with grouped value heads: 16 value heads (the same state as 8 x 4096 x 16 heads)
    # on 8 key heads
    "gva_train": ChunkWorkload("gva_train", B=8, T=4096, H=16, dk=128, dv=128, dtype="bf16", backward=True,
                               s0_std=0.02, seed=1007),
}


def gva_inputs(wl: ChunkWorkload, H: int, *, gen_device: str = "cpu") -> dict:
    """Grouped value heads: ``wl`` is drawn with wl.H = Hv value heads as in chunk_inputs; the key-side
    tensors (q, k, log_alpha, b) keep every (Hv / H)-th head, so H independent key heads remain."""
    inp = chunk_inputs(wl, gen_device=gen_device)
    G = wl.H // H
    assert G * H == wl.H
    for n in ("q", "k", "log_alpha", "b"):
        inp[n] = inp[n][:, :, ::G].contiguous()
    return inp
