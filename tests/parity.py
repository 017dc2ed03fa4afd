"""Parity helpers: run the CUDA path and the fp64 oracle on the same seeded inputs and compare.

Tolerances (stated by the target of this library):
  fp32-operand path : relative L2 <= 1e-4 per tensor
  bf16-operand path : relative L2 <= 5e-3 per tensor and max |err| <= 2e-2 * RMS(oracle tensor)
Relative L2 is ||x - x_ref||_2 / ||x_ref||_2 over the whole tensor.

Outputs stored in bf16 (o and dq, dk, dv, db, dw on the bf16 path) carry their own storage
rounding of up to 2^-8 |x| per element. Rounding the exact fp64 result to bf16 already breaks the
max-abs bound for heavy-tailed tensors (a dv element at 10.5 x RMS gives 0.031 x RMS), so for
bf16-stored tensors the max-abs bound applies to the error beyond that rounding:
max(|x - x_ref| - 2^-8 |x_ref|) <= 2e-2 * RMS. Relative L2 is checked as stated, rounding included.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL = {"f32": dict(rel=1e-4, maxabs_rms=None), "bf16": dict(rel=5e-3, maxabs_rms=2e-2)}


def to_np(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.astype(np.float64)
    return t.detach().to("cpu").double().numpy()


def metrics(got, ref):
    got, ref = to_np(got), to_np(ref)
    err = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / nref if nref > 0 else np.linalg.norm(err)
    rms = np.sqrt(np.mean(ref * ref)) if ref.size else 0.0
    maxabs = np.max(np.abs(err)) if err.size else 0.0
    return float(rel), float(maxabs), float(rms)


BF16_STORAGE_ROUNDING = 2.0 ** -8


def assert_close(name, got, ref, path, report=None):
    stored_bf16 = hasattr(got, "dtype") and str(got.dtype) == "torch.bfloat16"
    got_np, ref_np = to_np(got), to_np(ref)
    assert got_np.shape == ref_np.shape, (name, got_np.shape, ref_np.shape)
    assert np.all(np.isfinite(got_np)), f"{name}: non-finite values"
    rel, maxabs, rms = metrics(got_np, ref_np)
    if stored_bf16:
        maxabs = float(np.max(np.abs(got_np - ref_np) - BF16_STORAGE_ROUNDING * np.abs(ref_np))) if got_np.size else 0.0
    tol = TOL[path]
    if report is not None:
        report[name] = dict(rel_l2=rel, max_abs=maxabs, rms=rms)
    assert rel <= tol["rel"], f"{name}: relative L2 {rel:.3e} > {tol['rel']:.0e}"
    if tol["maxabs_rms"] is not None and rms > 0:
        assert maxabs <= tol["maxabs_rms"] * rms, f"{name}: max abs {maxabs:.3e} > {tol['maxabs_rms']} * rms {rms:.3e}"


def cuda(inputs):
    return {k: (None if v is None else v.cuda()) for k, v in inputs.items()}


def select_chains(inputs, chains):
    """Stack the (b, h) chains listed in `chains` as a batch of single-head sequences."""
    out = {}
    for key, t in inputs.items():
        if t is None:
            out[key] = None
        elif key in ("initial_state", "d_final_state"):
            out[key] = torch.stack([t[b, h] for b, h in chains])[:, None]
        else:
            out[key] = torch.stack([t[b, :, h] for b, h in chains])[:, :, None]
    return out


def gpu_rows(t, chains, state=False):
    """The same chains cut out of a full-size GPU result ([B,T,H,d] or [B,H,dk,dv])."""
    if t is None:
        return None
    t = t.detach().cpu()
    if state:
        return torch.stack([t[b, h] for b, h in chains])[:, None]
    return torch.stack([t[b, :, h] for b, h in chains])[:, :, None]


def oracle_fwd(inp):
    return oracle.fwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], inp.get("initial_state"))


def oracle_bwd(inp):
    return oracle.bwd(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["b"], inp["w"], inp.get("initial_state"),
                      inp.get("d_o"), inp.get("d_final_state"))
