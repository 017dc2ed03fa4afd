"""Thin ctypes binding of libgdr2.so (the C ABI declared in include/gdr2.h).

Argument marshalling only: every computation happens in the library's CUDA kernels. PyTorch is used
to hold device memory and to name the current CUDA stream. If the library cannot be loaded the
calls raise; there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

GDR2_F32, GDR2_BF16 = 0, 1
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_RANGE, ERR_BOUNDS = range(8)

EXPORTED = ("gdr2_version", "gdr2_status_string", "gdr2_check", "gdr2_workspace_bytes", "gdr2_chunk_fwd",
            "gdr2_chunk_bwd", "gdr2_decode_step", "gdr2_chunk_fwd_noalloc", "gdr2_profile_enable",
            "gdr2_profile_collect", "gdr2_chunk_fwd_train", "gdr2_chunk_bwd_saved", "gdr2_workspace_bytes_varlen",
            "gdr2_chunk_fwd_varlen", "gdr2_chunk_fwd_train_varlen", "gdr2_chunk_bwd_varlen",
            "gdr2_chunk_bwd_saved_varlen", "gdr2_gate_prologue_workspace_bytes", "gdr2_gate_prologue_fwd",
            "gdr2_gate_prologue_bwd", "gdr2_workspace_bytes_gva", "gdr2_chunk_fwd_gva", "gdr2_chunk_fwd_train_gva",
            "gdr2_chunk_bwd_gva", "gdr2_chunk_bwd_saved_gva", "gdr2_workspace_bytes_varlen_gva",
            "gdr2_chunk_fwd_varlen_gva", "gdr2_chunk_fwd_train_varlen_gva", "gdr2_chunk_bwd_varlen_gva",
            "gdr2_chunk_bwd_saved_varlen_gva", "gdr2_set_chunk_path", "gdr2_get_chunk_path")

_lib = None
_lock = threading.Lock()
_VP = ctypes.c_void_p
_I = ctypes.c_int


class GDR2Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed with status {status}: {status_string(status)}")


def lib(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libgdr2.so from the package directory (building it first when missing or stale). With the
    environment variable GDR2_DEBUG_BUILD=1 the process loads libgdr2_debug.so instead: the same kernels with
    the index checks of -DGDR2_DEBUG, reported by check() as ERR_BOUNDS."""
    global _lib
    with _lock:
        if _lib is None:
            debug = os.environ.get("GDR2_DEBUG_BUILD") == "1"
            path = _build.DEBUG_LIB if debug else _build.LIB
            if build_if_missing:
                path = _build.build_debug() if debug else _build.build()
            if not os.path.exists(path):
                raise RuntimeError(f"libgdr2.so not found at {path}; run gated_delta_rule_65_b200.build")
            L = ctypes.CDLL(path)
            L.gdr2_version.restype = _I
            L.gdr2_version.argtypes = []
            L.gdr2_status_string.restype = ctypes.c_char_p
            L.gdr2_status_string.argtypes = [_I]
            L.gdr2_check.restype = _I
            L.gdr2_check.argtypes = [_VP]
            L.gdr2_workspace_bytes.restype = ctypes.c_size_t
            L.gdr2_workspace_bytes.argtypes = [_I] * 7
            L.gdr2_set_chunk_path.restype = _I
            L.gdr2_set_chunk_path.argtypes = [_I]
            L.gdr2_get_chunk_path.restype = _I
            L.gdr2_get_chunk_path.argtypes = []
            L.gdr2_chunk_fwd.restype = _I
            L.gdr2_chunk_fwd.argtypes = [_VP] * 9 + [_I] * 6 + [_VP, ctypes.c_size_t, _VP]
            L.gdr2_chunk_bwd.restype = _I
            L.gdr2_chunk_bwd.argtypes = [_VP] * 16 + [_I] * 6 + [_VP, ctypes.c_size_t, _VP]
            L.gdr2_chunk_fwd_train.restype = _I
            L.gdr2_chunk_fwd_train.argtypes = [_VP] * 9 + [_I] * 6 + [_VP, ctypes.c_size_t, _VP]
            L.gdr2_chunk_bwd_saved.restype = _I
            L.gdr2_chunk_bwd_saved.argtypes = [_VP] * 16 + [_I] * 6 + [_VP, ctypes.c_size_t, _VP]
            L.gdr2_workspace_bytes_varlen.restype = ctypes.c_size_t
            L.gdr2_workspace_bytes_varlen.argtypes = [_I] * 7
            for fn in (L.gdr2_chunk_fwd_varlen, L.gdr2_chunk_fwd_train_varlen):
                fn.restype = _I
                fn.argtypes = [_VP] * 10 + [_I] * 6 + [_VP, ctypes.c_size_t, _VP]
            for fn in (L.gdr2_chunk_bwd_varlen, L.gdr2_chunk_bwd_saved_varlen):
                fn.restype = _I
                fn.argtypes = [_VP] * 17 + [_I] * 6 + [_VP, ctypes.c_size_t, _VP]
            L.gdr2_workspace_bytes_varlen_gva.restype = ctypes.c_size_t
            L.gdr2_workspace_bytes_varlen_gva.argtypes = [_I] * 8
            for fn in (L.gdr2_chunk_fwd_varlen_gva, L.gdr2_chunk_fwd_train_varlen_gva):
                fn.restype = _I
                fn.argtypes = [_VP] * 10 + [_I] * 7 + [_VP, ctypes.c_size_t, _VP]
            for fn in (L.gdr2_chunk_bwd_varlen_gva, L.gdr2_chunk_bwd_saved_varlen_gva):
                fn.restype = _I
                fn.argtypes = [_VP] * 17 + [_I] * 7 + [_VP, ctypes.c_size_t, _VP]
            L.gdr2_workspace_bytes_gva.restype = ctypes.c_size_t
            L.gdr2_workspace_bytes_gva.argtypes = [_I] * 8
            for fn in (L.gdr2_chunk_fwd_gva, L.gdr2_chunk_fwd_train_gva):
                fn.restype = _I
                fn.argtypes = [_VP] * 9 + [_I] * 7 + [_VP, ctypes.c_size_t, _VP]
            for fn in (L.gdr2_chunk_bwd_gva, L.gdr2_chunk_bwd_saved_gva):
                fn.restype = _I
                fn.argtypes = [_VP] * 16 + [_I] * 7 + [_VP, ctypes.c_size_t, _VP]
            L.gdr2_gate_prologue_workspace_bytes.restype = ctypes.c_size_t
            L.gdr2_gate_prologue_workspace_bytes.argtypes = [_I] * 6
            L.gdr2_gate_prologue_fwd.restype = _I
            L.gdr2_gate_prologue_fwd.argtypes = [_VP] * 7 + [_I] + [_VP] * 5 + [_I] * 6 + [_VP]
            L.gdr2_gate_prologue_bwd.restype = _I
            L.gdr2_gate_prologue_bwd.argtypes = ([_VP] * 7 + [_I] + [_VP] * 12 + [_I] * 6 +
                                                 [_VP, ctypes.c_size_t, _VP])
            L.gdr2_decode_step.restype = _I
            L.gdr2_decode_step.argtypes = [_VP] * 8 + [_I] * 5 + [_VP]
            L.gdr2_chunk_fwd_noalloc.restype = _I
            L.gdr2_chunk_fwd_noalloc.argtypes = [_VP] * 9 + [_I] * 6 + [_VP]
            L.gdr2_profile_enable.restype = _I
            L.gdr2_profile_enable.argtypes = [_I]
            L.gdr2_profile_collect.restype = _I
            L.gdr2_profile_collect.argtypes = [ctypes.c_char_p, _I, ctypes.POINTER(_I),
                                               ctypes.POINTER(ctypes.c_double), _I, ctypes.POINTER(_I)]
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gdr2_status_string(int(status)).decode()


def check(stream=None) -> int:
    """gdr2_check: synchronise ``stream`` (default: the current stream), then read and clear the device
    status words. Returns OK, ERR_TIMEOUT (a bounded wait expired), ERR_RANGE (a chunk's cumulative
    log-decay left [-160, 160] on the tensor-core path, [-80, 80] on the fp32 path, or an fp16 operand of the
    per-chain path passed 65504), ERR_BOUNDS (debug build only: a kernel index check failed) or ERR_CUDA; the
    outputs of the calls since the last check are valid only with OK."""
    return int(lib().gdr2_check(_stream(stream)))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GDR2_F32
    if t.dtype == torch.bfloat16:
        return GDR2_BF16
    raise TypeError(f"unsupported operand dtype {t.dtype}; use float32 or bfloat16")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("gdr2: tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("gdr2: tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn, st):
    if st != OK:
        raise GDR2Error(fn, st)


PATH_AUTO, PATH_CHAIN, PATH_SPLIT = 0, 1, 2


def set_chunk_path(path: int) -> None:
    """gdr2_set_chunk_path: 0 automatic, 1 per-chain fused kernels, 2 chunk-parallel kernels (process-wide)."""
    _check("gdr2_set_chunk_path", lib().gdr2_set_chunk_path(int(path)))


def get_chunk_path() -> int:
    return int(lib().gdr2_get_chunk_path())


def workspace_bytes(B, T, H, dk, dv, dtype_code, for_bwd) -> int:
    return int(lib().gdr2_workspace_bytes(B, T, H, dk, dv, dtype_code, int(for_bwd)))


def alloc_workspace(B, T, H, dk, dv, dtype_code, for_bwd, device=None) -> torch.Tensor:
    n = workspace_bytes(B, T, H, dk, dv, dtype_code, for_bwd)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device or "cuda")


def chunk_fwd(q, k, v, log_alpha, b, w, initial_state=None, *, output_final_state=True,
              o=None, final_state=None, workspace=None, stream=None, train=False):
    """gdr2_chunk_fwd, or gdr2_chunk_fwd_train when train=True (then `workspace` must be the
    backward-sized buffer that gdr2_chunk_bwd_saved will read). Returns (o, final_state or None)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if output_final_state and final_state is None:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if not output_final_state:
        final_state = None
    if workspace is None:
        if train:
            raise ValueError("train=True needs the workspace that the backward will read")
        workspace = alloc_workspace(B, T, H, dk, dv, dt, 0, q.device)
    fn = lib().gdr2_chunk_fwd_train if train else lib().gdr2_chunk_fwd
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(initial_state),
                              _ptr(o), _ptr(final_state), B, T, H, dk, dv, dt, _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _check("gdr2_chunk_fwd_train" if train else "gdr2_chunk_fwd", st)
    return o, final_state


def chunk_fwd_noalloc(q, k, v, log_alpha, b, w, initial_state=None, *, output_final_state=True,
                      o=None, final_state=None, stream=None):
    """gdr2_chunk_fwd_noalloc: the forward with the library's fixed scratch instead of a workspace,
    for callers that cannot allocate device memory (the outputs here are still allocated by torch
    when not given). Returns (o, final_state or None)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if output_final_state and final_state is None:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    if not output_final_state:
        final_state = None
    st = lib().gdr2_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w),
                                      _ptr(initial_state), _ptr(o), _ptr(final_state), B, T, H, dk, dv,
                                      _dtype_code(q), _stream(stream))
    _check("gdr2_chunk_fwd_noalloc", st)
    return o, final_state


def chunk_bwd(q, k, v, log_alpha, b, w, initial_state=None, d_o=None, d_final_state=None, *,
              want_d_initial_state=True, out=None, workspace=None, stream=None, saved=False):
    """gdr2_chunk_bwd, or gdr2_chunk_bwd_saved when saved=True (then `workspace` is the buffer a
    chunk_fwd(..., train=True) call with the same inputs filled). Returns a dict dq, dk, dv,
    dlog_alpha, db, dw, dS0 (dS0 None if not wanted)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    if out is None:
        out = {n: torch.empty_like(q) for n in ("dq", "dk", "db")}
        out.update({n: torch.empty_like(v) for n in ("dv", "dw")})
        out["dlog_alpha"] = torch.empty((B, T, H, dk), dtype=torch.float32, device=q.device)
        out["dS0"] = (torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
                      if want_d_initial_state else None)
    if workspace is None:
        if saved:
            raise ValueError("saved=True needs the workspace filled by chunk_fwd(..., train=True)")
        workspace = alloc_workspace(B, T, H, dk, dv, dt, 1, q.device)
    fn = lib().gdr2_chunk_bwd_saved if saved else lib().gdr2_chunk_bwd
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(initial_state),
                              _ptr(d_o), _ptr(d_final_state), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                              _ptr(out["dlog_alpha"]), _ptr(out["db"]), _ptr(out["dw"]), _ptr(out.get("dS0")),
                              B, T, H, dk, dv, dt, _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _check("gdr2_chunk_bwd_saved" if saved else "gdr2_chunk_bwd", st)
    return out


def workspace_bytes_gva(B, T, H, Hv, dk, dv, dtype_code, for_bwd) -> int:
    return int(lib().gdr2_workspace_bytes_gva(B, T, H, Hv, dk, dv, dtype_code, int(for_bwd)))


def alloc_workspace_gva(B, T, H, Hv, dk, dv, dtype_code, for_bwd, device=None) -> torch.Tensor:
    n = workspace_bytes_gva(B, T, H, Hv, dk, dv, dtype_code, for_bwd)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device or "cuda")


def chunk_fwd_gva(q, k, v, log_alpha, b, w, initial_state=None, *, output_final_state=True, o=None,
                  final_state=None, workspace=None, stream=None, train=False):
    """gdr2_chunk_fwd_gva (or the _train variant): grouped value heads. q, k, log_alpha, b [B,T,H,dk];
    v, w [B,T,Hv,dv] with Hv a multiple of H; states [B,Hv,dk,dv]. Returns (o [B,T,Hv,dv], final_state)."""
    B, T, H, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    dt = _dtype_code(q)
    if o is None:
        o = torch.empty((B, T, Hv, dv), dtype=q.dtype, device=q.device)
    if output_final_state and final_state is None:
        final_state = torch.empty((B, Hv, dk, dv), dtype=torch.float32, device=q.device)
    if not output_final_state:
        final_state = None
    if workspace is None:
        if train:
            raise ValueError("train=True needs the workspace that the backward will read")
        workspace = alloc_workspace_gva(B, T, H, Hv, dk, dv, dt, 0, q.device)
    fn = lib().gdr2_chunk_fwd_train_gva if train else lib().gdr2_chunk_fwd_gva
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(initial_state), _ptr(o),
            _ptr(final_state), B, T, H, Hv, dk, dv, dt, _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream))
    _check("gdr2_chunk_fwd_train_gva" if train else "gdr2_chunk_fwd_gva", st)
    return o, final_state


def chunk_bwd_gva(q, k, v, log_alpha, b, w, initial_state=None, d_o=None, d_final_state=None, *,
                  want_d_initial_state=True, out=None, workspace=None, stream=None, saved=False):
    """gdr2_chunk_bwd_gva (or the _saved variant): returns a dict dq, dk, dlog_alpha, db [B,T,H,dk],
    dv, dw [B,T,Hv,dv], dS0 [B,Hv,dk,dv] (or None)."""
    B, T, H, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    dt = _dtype_code(q)
    if out is None:
        out = {n: torch.empty_like(q) for n in ("dq", "dk", "db")}
        out.update({n: torch.empty_like(v) for n in ("dv", "dw")})
        out["dlog_alpha"] = torch.empty((B, T, H, dk), dtype=torch.float32, device=q.device)
        out["dS0"] = (torch.empty((B, Hv, dk, dv), dtype=torch.float32, device=q.device)
                      if want_d_initial_state else None)
    if workspace is None:
        if saved:
            raise ValueError("saved=True needs the workspace filled by chunk_fwd_gva(..., train=True)")
        workspace = alloc_workspace_gva(B, T, H, Hv, dk, dv, dt, 1, q.device)
    fn = lib().gdr2_chunk_bwd_saved_gva if saved else lib().gdr2_chunk_bwd_gva
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(initial_state), _ptr(d_o),
            _ptr(d_final_state), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dlog_alpha"]),
            _ptr(out["db"]), _ptr(out["dw"]), _ptr(out.get("dS0")), B, T, H, Hv, dk, dv, dt, _ptr(workspace),
            workspace.numel() * workspace.element_size(), _stream(stream))
    _check("gdr2_chunk_bwd_saved_gva" if saved else "gdr2_chunk_bwd_gva", st)
    return out


def workspace_bytes_varlen(N, T, H, dk, dv, dtype_code, for_bwd, Hv=None) -> int:
    """gdr2_workspace_bytes_varlen, or gdr2_workspace_bytes_varlen_gva when Hv (value heads) != H."""
    if Hv is not None and Hv != H:
        return int(lib().gdr2_workspace_bytes_varlen_gva(N, T, H, Hv, dk, dv, dtype_code, int(for_bwd)))
    return int(lib().gdr2_workspace_bytes_varlen(N, T, H, dk, dv, dtype_code, int(for_bwd)))


def alloc_workspace_varlen(N, T, H, dk, dv, dtype_code, for_bwd, device=None, Hv=None) -> torch.Tensor:
    n = workspace_bytes_varlen(N, T, H, dk, dv, dtype_code, for_bwd, Hv)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device or "cuda")


def _packed_shape(q, cu_seqlens):
    if q.dim() == 4:
        if q.shape[0] != 1:
            raise ValueError("packed token tensors are [T, H, d] or [1, T, H, d]")
        q = q[0]
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens must be a 1-D int32 device tensor of N + 1 offsets")
    T, H, dk = q.shape
    return cu_seqlens.numel() - 1, T, H, dk


def chunk_fwd_varlen(q, k, v, log_alpha, b, w, cu_seqlens, initial_state=None, *, output_final_state=True,
                     o=None, final_state=None, workspace=None, stream=None, train=False):
    """gdr2_chunk_fwd_varlen (or the _train variant): packed token tensors [T, H, d] (or [1, T, H, d]),
    cu_seqlens int32 [N + 1] on the device, states [N, Hv, dk, dv]. v and w with more heads than q (Hv =
    G H value heads) select gdr2_chunk_fwd_varlen_gva. Returns (o shaped like v, final_state)."""
    N, T, H, dk = _packed_shape(q, cu_seqlens)
    dv, Hv = v.shape[-1], v.shape[-2]
    dt = _dtype_code(q)
    if o is None:
        o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    if output_final_state and final_state is None:
        final_state = torch.empty((N, Hv, dk, dv), dtype=torch.float32, device=q.device)
    if not output_final_state:
        final_state = None
    if workspace is None:
        if train:
            raise ValueError("train=True needs the workspace that the backward will read")
        workspace = alloc_workspace_varlen(N, T, H, dk, dv, dt, 0, q.device, Hv)
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(initial_state), _ptr(o),
            _ptr(final_state), _ptr(cu_seqlens), N, T, H]
    tail = [dk, dv, dt, _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)]
    if Hv != H:
        name = "gdr2_chunk_fwd_train_varlen_gva" if train else "gdr2_chunk_fwd_varlen_gva"
        st = getattr(lib(), name)(*args, Hv, *tail)
    else:
        name = "gdr2_chunk_fwd_train_varlen" if train else "gdr2_chunk_fwd_varlen"
        st = getattr(lib(), name)(*args, *tail)
    _check(name, st)
    return o, final_state


def chunk_bwd_varlen(q, k, v, log_alpha, b, w, cu_seqlens, initial_state=None, d_o=None, d_final_state=None, *,
                     want_d_initial_state=True, out=None, workspace=None, stream=None, saved=False):
    """gdr2_chunk_bwd_varlen (or the _saved variant after chunk_fwd_varlen(..., train=True) on the same
    workspace); v and w with more heads than q select the _gva entry points. Returns a dict dq, dk, dv,
    dlog_alpha, db, dw, dS0 ([N, Hv, dk, dv] or None)."""
    N, T, H, dk = _packed_shape(q, cu_seqlens)
    dv, Hv = v.shape[-1], v.shape[-2]
    dt = _dtype_code(q)
    if out is None:
        out = {n: torch.empty_like(q) for n in ("dq", "dk", "db")}
        out.update({n: torch.empty_like(v) for n in ("dv", "dw")})
        out["dlog_alpha"] = torch.empty(log_alpha.shape, dtype=torch.float32, device=q.device)
        out["dS0"] = (torch.empty((N, Hv, dk, dv), dtype=torch.float32, device=q.device)
                      if want_d_initial_state else None)
    if workspace is None:
        if saved:
            raise ValueError("saved=True needs the workspace filled by chunk_fwd_varlen(..., train=True)")
        workspace = alloc_workspace_varlen(N, T, H, dk, dv, dt, 1, q.device, Hv)
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(initial_state), _ptr(d_o),
            _ptr(d_final_state), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dlog_alpha"]),
            _ptr(out["db"]), _ptr(out["dw"]), _ptr(out.get("dS0")), _ptr(cu_seqlens), N, T, H]
    tail = [dk, dv, dt, _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)]
    if Hv != H:
        name = "gdr2_chunk_bwd_saved_varlen_gva" if saved else "gdr2_chunk_bwd_varlen_gva"
        st = getattr(lib(), name)(*args, Hv, *tail)
    else:
        name = "gdr2_chunk_bwd_saved_varlen" if saved else "gdr2_chunk_bwd_varlen"
        st = getattr(lib(), name)(*args, *tail)
    _check(name, st)
    return out


def gate_prologue_fwd(xq, xk, xf, xb, xw, a, delta, *, neg_eig=False, out=None, stream=None):
    """gdr2_gate_prologue_fwd: q, k (L2-normalised), log_alpha (fp32), b, w from the pre-activations
    [B,T,H,d] and a, delta [H,dk]. Returns a dict q, k, log_alpha, b, w."""
    B, T, H, dk = xq.shape
    dv = xw.shape[-1]
    if out is None:
        out = {"q": torch.empty_like(xq), "k": torch.empty_like(xk), "b": torch.empty_like(xb),
               "w": torch.empty_like(xw),
               "log_alpha": torch.empty((B, T, H, dk), dtype=torch.float32, device=xq.device)}
    st = lib().gdr2_gate_prologue_fwd(_ptr(xq), _ptr(xk), _ptr(xf), _ptr(xb), _ptr(xw), _ptr(a), _ptr(delta),
                                      int(neg_eig), _ptr(out["q"]), _ptr(out["k"]), _ptr(out["log_alpha"]),
                                      _ptr(out["b"]), _ptr(out["w"]), B, T, H, dk, dv, _dtype_code(xq),
                                      _stream(stream))
    _check("gdr2_gate_prologue_fwd", st)
    return out


def gate_prologue_bwd(xq, xk, xf, xb, xw, a, delta, dq, dk, dlog_alpha, db, dw, *, neg_eig=False, out=None,
                      workspace=None, stream=None):
    """gdr2_gate_prologue_bwd: returns a dict dxq, dxk, dxf, dxb, dxw, da, ddelta."""
    B, T, H, dk_ = xq.shape
    dv = xw.shape[-1]
    dt = _dtype_code(xq)
    if out is None:
        out = {"dxq": torch.empty_like(xq), "dxk": torch.empty_like(xk), "dxf": torch.empty_like(xf),
               "dxb": torch.empty_like(xb), "dxw": torch.empty_like(xw),
               "da": torch.empty((H, dk_), dtype=torch.float32, device=xq.device),
               "ddelta": torch.empty((H, dk_), dtype=torch.float32, device=xq.device)}
    if workspace is None:
        n = int(lib().gdr2_gate_prologue_workspace_bytes(B, T, H, dk_, dv, dt))
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=xq.device)
    st = lib().gdr2_gate_prologue_bwd(_ptr(xq), _ptr(xk), _ptr(xf), _ptr(xb), _ptr(xw), _ptr(a), _ptr(delta),
                                      int(neg_eig), _ptr(dq), _ptr(dk), _ptr(dlog_alpha), _ptr(db), _ptr(dw),
                                      _ptr(out["dxq"]), _ptr(out["dxk"]), _ptr(out["dxf"]), _ptr(out["dxb"]),
                                      _ptr(out["dxw"]), _ptr(out["da"]), _ptr(out["ddelta"]), B, T, H, dk_, dv, dt,
                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream(stream))
    _check("gdr2_gate_prologue_bwd", st)
    return out


def decode_step(q, k, v, log_alpha, b, w, state, o=None, *, stream=None):
    """gdr2_decode_step: updates `state` in place and returns o [B,H,dv]."""
    B, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, H, dv), dtype=q.dtype, device=q.device)
    st = lib().gdr2_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b), _ptr(w), _ptr(state), _ptr(o),
                                B, H, dk, dv, _dtype_code(q), _stream(stream))
    _check("gdr2_decode_step", st)
    return o


def profile_enable(on: bool = True) -> None:
    """Turn per-kernel event timing on or off for later launches (benchmark support)."""
    lib().gdr2_profile_enable(int(bool(on)))


def profile_collect(max_entries: int = 64) -> dict:
    """Wait for recorded launches and return {kernel name: (launches, total ms)}; clears the record."""
    stride = 64
    names = ctypes.create_string_buffer(stride * max_entries)
    launches = (_I * max_entries)()
    ms = (ctypes.c_double * max_entries)()
    dropped = _I(0)
    n = lib().gdr2_profile_collect(names, stride, launches, ms, max_entries, ctypes.byref(dropped))
    if n < 0:
        raise GDR2Error("gdr2_profile_collect", -n)
    out = {}
    for i in range(n):
        nm = names.raw[i * stride:(i + 1) * stride].split(b"\0", 1)[0].decode()
        out[nm] = (int(launches[i]), float(ms[i]))
    if dropped.value:
        out["<dropped>"] = (int(dropped.value), 0.0)
    return out
