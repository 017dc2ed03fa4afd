"""fp64 CPU oracle for the Gated Delta Rule-2 mixer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
this package. The CUDA library (``gated_delta_rule_65_b200``) never imports it, and it imports
nothing from that package.

The arithmetic lives in ``gdr2_oracle.c`` (plain C, double precision, one serial token loop per
(batch, head) chain). The formulas follow "Gated DeltaNet-2: Decoupling Erase and Write in Linear
Attention", review page section "The Gated Delta Rule-2 State Update", Steps 1-5 / Eq. 10; the
backward is the explicit token-by-token adjoint of those steps (the verification protocol of the
review's Appendix D.6 paragraph). This module only compiles the C file, marshals numpy arrays and
checks shapes.

Pins (tests/test_oracle_pins.py) tie the oracle to facts other than itself: the KDA and Gated
DeltaNet reductions, the linear-attention prefix sum, the k^T S = z projector property, the
reflection norm for b = 2, explicit transition-matrix products, a hand-worked Eq. 10 example, finite
differences of the loss, an independent chunkwise (WY) restatement, value-column independence, the
segment composition S_end = M S_start + N behind the chunk-level scan, and for the packed-batch helpers
(fwd_varlen / bwd_varlen, review Appendix C.6) equal lengths = the batch, and the state reset.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_gdr2.so")
_lib = None
_lock = threading.Lock()

_DP = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    """Compile gdr2_oracle.c into liboracle_gdr2.so next to it (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off",
                               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            for name in ("oracle_gdr2_fwd", "oracle_gdr2_bwd", "oracle_gdr2_decode"):
                getattr(lib, name).restype = ctypes.c_int
            lib.oracle_gdr2_fwd.argtypes = [_DP] * 9 + [ctypes.c_int] * 6
            lib.oracle_gdr2_bwd.argtypes = [_DP] * 16 + [ctypes.c_int] * 6
            lib.oracle_gdr2_decode.argtypes = [_DP] * 8 + [ctypes.c_int] * 4
            _lib = lib
    return _lib


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_DP)


def _check(name, a, shape):
    if a is not None and tuple(a.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(a.shape)}")


def fwd(q, k, v, log_alpha, b, w, initial_state=None, nthreads: int = 0):
    """Token recurrence in fp64. Returns (o [B,T,H,dv], final_state [B,H,dk,dv])."""
    q, k, v, la, b, w, S0 = map(_f64, (q, k, v, log_alpha, b, w, initial_state))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for n, a, s in (("k", k, q.shape), ("log_alpha", la, q.shape), ("b", b, q.shape),
                    ("w", w, v.shape), ("v", v, (B, T, H, dv)), ("initial_state", S0, (B, H, dk, dv))):
        _check(n, a, s)
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))
    rc = _load().oracle_gdr2_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(w), _ptr(S0),
                                 _ptr(o), _ptr(ST), B, T, H, dk, dv, int(nthreads))
    if rc != 0:
        raise MemoryError(f"oracle_gdr2_fwd returned {rc}")
    return o, ST


def bwd(q, k, v, log_alpha, b, w, initial_state=None, d_o=None, d_final_state=None, nthreads: int = 0):
    """Adjoint recurrence in fp64. Returns dict dq, dk, dv, dlog_alpha, db, dw, dS0."""
    q, k, v, la, b, w, S0, dO, dST = map(_f64, (q, k, v, log_alpha, b, w, initial_state, d_o, d_final_state))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    for n, a, s in (("k", k, q.shape), ("log_alpha", la, q.shape), ("b", b, q.shape),
                    ("w", w, v.shape), ("d_o", dO, v.shape), ("initial_state", S0, (B, H, dk, dv)),
                    ("d_final_state", dST, (B, H, dk, dv))):
        _check(n, a, s)
    out = {n: np.zeros(q.shape) for n in ("dq", "dk", "dlog_alpha", "db")}
    out.update({n: np.zeros(v.shape) for n in ("dv", "dw")})
    out["dS0"] = np.zeros((B, H, dk, dv))
    rc = _load().oracle_gdr2_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(w), _ptr(S0),
                                 _ptr(dO), _ptr(dST), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                 _ptr(out["dlog_alpha"]), _ptr(out["db"]), _ptr(out["dw"]),
                                 _ptr(out["dS0"]), B, T, H, dk, dv, int(nthreads))
    if rc != 0:
        raise MemoryError(f"oracle_gdr2_bwd returned {rc}")
    return out


def decode(q, k, v, log_alpha, b, w, state):
    """One token per (b, h). Returns (o [B,H,dv], new_state [B,H,dk,dv]); the input is not modified."""
    q, k, v, la, b, w = map(_f64, (q, k, v, log_alpha, b, w))
    S = _f64(state).copy()
    B, H, dk = q.shape
    dv = v.shape[-1]
    for n, a, s in (("k", k, q.shape), ("log_alpha", la, q.shape), ("b", b, q.shape),
                    ("w", w, v.shape), ("state", S, (B, H, dk, dv))):
        _check(n, a, s)
    o = np.zeros((B, H, dv))
    rc = _load().oracle_gdr2_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(w), _ptr(S),
                                    _ptr(o), B, H, dk, dv)
    if rc != 0:
        raise MemoryError(f"oracle_gdr2_decode returned {rc}")
    return o, S


def _sequences(cu_seqlens, T):
    cu = [int(x) for x in np.asarray(cu_seqlens.detach().cpu() if hasattr(cu_seqlens, "detach") else cu_seqlens)]
    if cu[0] != 0 or cu[-1] != T or any(b < a for a, b in zip(cu[:-1], cu[1:])):
        raise ValueError("cu_seqlens must rise from 0 to T")
    return list(zip(cu[:-1], cu[1:]))


def fwd_varlen(q, k, v, log_alpha, b, w, cu_seqlens, initial_state=None, nthreads: int = 0):
    """Packed variable-length batch (review, Appendix C.6 "Variable-length sequences"): the token axis
    holds N sequences back to back, sequence n on tokens [cu[n], cu[n+1]), and the recurrence restarts
    from that sequence's own initial state at each boundary. Token tensors [T,H,d]; states
    [N,H,dk,dv]. Each sequence is the token recurrence of fwd() on its slice.
    Returns (o [T,H,dv], final_state [N,H,dk,dv])."""
    q, k, v, la, b, w, S0 = map(_f64, (q, k, v, log_alpha, b, w, initial_state))
    T, H, dk = q.shape
    dv = v.shape[-1]
    seqs = _sequences(cu_seqlens, T)
    o = np.zeros((T, H, dv))
    ST = np.zeros((len(seqs), H, dk, dv))
    for n, (a, e) in enumerate(seqs):
        s0 = None if S0 is None else S0[n:n + 1]
        if e == a:  # an empty sequence leaves its state unchanged
            ST[n] = 0.0 if s0 is None else s0[0]
            continue
        on, Sn = fwd(*(x[None, a:e] for x in (q, k, v, la, b, w)), s0, nthreads=nthreads)
        o[a:e] = on[0]
        ST[n] = Sn[0]
    return o, ST


def bwd_varlen(q, k, v, log_alpha, b, w, cu_seqlens, initial_state=None, d_o=None, d_final_state=None,
               nthreads: int = 0):
    """Adjoint of fwd_varlen: every sequence is the adjoint recurrence of bwd() on its slice, from its
    own dS_T; gradients of tokens [T,H,d], dS0 [N,H,dk,dv]."""
    q, k, v, la, b, w, S0, dO, dST = map(_f64, (q, k, v, log_alpha, b, w, initial_state, d_o, d_final_state))
    T, H, dk = q.shape
    dv = v.shape[-1]
    seqs = _sequences(cu_seqlens, T)
    out = {n: np.zeros((T, H, dk)) for n in ("dq", "dk", "dlog_alpha", "db")}
    out.update({n: np.zeros((T, H, dv)) for n in ("dv", "dw")})
    out["dS0"] = np.zeros((len(seqs), H, dk, dv))
    for n, (a, e) in enumerate(seqs):
        dst = None if dST is None else dST[n:n + 1]
        if e == a:  # the gradient of an empty sequence's state passes through
            out["dS0"][n] = 0.0 if dst is None else dst[0]
            continue
        g = bwd(*(x[None, a:e] for x in (q, k, v, la, b, w)), None if S0 is None else S0[n:n + 1],
                None if dO is None else dO[None, a:e], dst, nthreads=nthreads)
        for name in ("dq", "dk", "dlog_alpha", "db", "dv", "dw"):
            out[name][a:e] = g[name][0]
        out["dS0"][n] = g["dS0"][0]
    return out


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def prologue_fwd(xq, xk, xf, xb, xw, a, delta, neg_eig=False):
    """Gate and normalisation prologue in fp64 (review, "Gate Parameterization", Eqs. 11-12, and
    "Block Design", steps 2-3). Pre-activations [B,T,H,d]; a, delta [H,dk].
      q = xq / ||xq||, k = xk / ||xk|| over each head's channels (a zero vector stays zero)
      log_alpha = -exp(a) * softplus(xf + delta);  b = sigmoid(xb) (x2 if neg_eig);  w = sigmoid(xw)
    Returns a dict q, k, log_alpha, b, w."""
    xq, xk, xf, xb, xw, a, delta = map(_f64, (xq, xk, xf, xb, xw, a, delta))
    out = {}
    for name, x in (("q", xq), ("k", xk)):
        n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
        out[name] = np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0)
    out["log_alpha"] = -np.exp(a) * np.logaddexp(0.0, xf + delta)
    out["b"] = (2.0 if neg_eig else 1.0) * _sigmoid(xb)
    out["w"] = _sigmoid(xw)
    return out


def prologue_bwd(xq, xk, xf, xb, xw, a, delta, dq, dk, dlog_alpha, db, dw, neg_eig=False):
    """Chain rule through prologue_fwd: returns dxq, dxk, dxf, dxb, dxw and da, ddelta [H,dk] (sums over
    every batch element and token)."""
    xq, xk, xf, xb, xw, a, delta, dq, dk, dg, db, dw = map(
        _f64, (xq, xk, xf, xb, xw, a, delta, dq, dk, dlog_alpha, db, dw))
    out = {}
    for name, x, dy in (("dxq", xq, dq), ("dxk", xk, dk)):
        n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
        safe = np.where(n > 0, n, 1.0)
        u = x / safe
        out[name] = np.where(n > 0, (dy - u * np.sum(u * dy, axis=-1, keepdims=True)) / safe, 0.0)
    z = xf + delta
    g = -np.exp(a) * np.logaddexp(0.0, z)
    out["dxf"] = dg * (-np.exp(a)) * _sigmoid(z)
    out["da"] = np.sum(dg * g, axis=(0, 1))
    out["ddelta"] = np.sum(out["dxf"], axis=(0, 1))
    sb = _sigmoid(xb)
    out["dxb"] = db * (2.0 if neg_eig else 1.0) * sb * (1.0 - sb)
    sw = _sigmoid(xw)
    out["dxw"] = dw * sw * (1.0 - sw)
    return out


def fwd_gva(q, k, v, log_alpha, b, w, initial_state=None, nthreads: int = 0):
    """Grouped value heads (review, "Headed architecture and grouped-value attention"): Hv = G H value
    heads; the key-side tensors q, k, log_alpha, b [B,T,H,dk] are repeated across each group of G value
    heads (value head j reads key head j // G), v, w [B,T,Hv,dv] and the states [B,Hv,dk,dv] are per
    value head. Returns (o [B,T,Hv,dv], final_state [B,Hv,dk,dv])."""
    q, k, la, b = map(_f64, (q, k, log_alpha, b))
    G = _f64(v).shape[2] // q.shape[2]
    rep = lambda x: np.repeat(x, G, axis=2)  # noqa: E731
    return fwd(rep(q), rep(k), v, rep(la), rep(b), w, initial_state, nthreads=nthreads)


def bwd_gva(q, k, v, log_alpha, b, w, initial_state=None, d_o=None, d_final_state=None, nthreads: int = 0):
    """Adjoint of fwd_gva: the gradient of a key-side tensor is the sum of the gradients of its copies
    over the value-head group. Returns dq, dk, dlog_alpha, db [B,T,H,dk], dv, dw [B,T,Hv,dv], dS0."""
    q, k, la, b = map(_f64, (q, k, log_alpha, b))
    B, T, H, dk = q.shape
    G = _f64(v).shape[2] // H
    rep = lambda x: np.repeat(x, G, axis=2)  # noqa: E731
    g = bwd(rep(q), rep(k), v, rep(la), rep(b), w, initial_state, d_o, d_final_state, nthreads=nthreads)
    for name in ("dq", "dk", "dlog_alpha", "db"):
        g[name] = g[name].reshape(B, T, H, G, dk).sum(axis=3)
    return g
