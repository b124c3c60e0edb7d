"""ctypes binding of libgdn2.so: argument marshalling only.

Every function here takes torch CUDA tensors, checks dtypes/devices, turns
them into raw pointers and calls the C entry point of the same name.  All
arithmetic runs in the library's CUDA kernels; nothing here computes.  If the
library cannot be loaded, every call raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn2.so")

GDN2_OK = 0
STATUS_NAMES = {0: "GDN2_OK", -1: "GDN2_ERR_NULL", -2: "GDN2_ERR_SHAPE", -3: "GDN2_ERR_DTYPE",
                -4: "GDN2_ERR_ALIGN", -5: "GDN2_ERR_WORKSPACE", -6: "GDN2_ERR_CUDA",
                -7: "GDN2_ERR_TIMEOUT", -8: "GDN2_ERR_UNSUPPORTED", -9: "GDN2_ERR_TOO_LARGE",
                -10: "GDN2_ERR_SEQLENS"}
GDN2_F32, GDN2_BF16 = 0, 1
EXPORTS = ("gdn2_chunk_fwd", "gdn2_decode_step", "gdn2_chunk_bwd", "gdn2_workspace_size",
           "gdn2_strerror", "gdn2_sync_status", "gdn2_chunk_bwd_noalloc", "gdn2_chunk_fwd_varlen",
           "gdn2_chunk_bwd_varlen", "gdn2_chunk_fwd_gated", "gdn2_chunk_bwd_gated", "gdn2_decode_step_gated",
           "gdn2_workspace_size_gated", "gdn2_prologue", "gdn2_chunk_fwd_save", "gdn2_chunk_bwd_saved",
           "gdn2_chunk_fwd_host", "gdn2_selftest_timeout")
# gate layout flags (gdn2_gate_flags in include/gdn2.h)
DECAY_SCALAR, ERASE_SCALAR, WRITE_SCALAR, DECAY_NONE, ERASE_NONE, WRITE_NONE = 1, 2, 4, 8, 16, 32
# input prologue: q, k L2-normalised in the call; b, w given as logits (sigmoid in the call)
QK_L2NORM, BW_LOGITS = 64, 128
# Size of the library's static scratch array used by gdn2_chunk_bwd_noalloc
# (GDN2_NOALLOC_MAX_SCRATCH_BYTES in include/gdn2.h).
NOALLOC_MAX_SCRATCH_BYTES = 32 << 20

_lib = None


class Gdn2Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = raw().gdn2_strerror(status).decode() if _lib is not None else ""
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}: {msg}")


def load(path: str | None = None):
    """Load libgdn2.so (raises OSError if it is missing: build it first)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise OSError(f"{path} not found: run gated_delta_rule_78_b200/build.py (or __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.gdn2_chunk_fwd.argtypes = [i] * 6 + [vp] * 10 + [sz, vp]
    lib.gdn2_chunk_fwd.restype = i
    lib.gdn2_decode_step.argtypes = [i] * 5 + [vp] * 8 + [vp]
    lib.gdn2_decode_step.restype = i
    lib.gdn2_chunk_bwd.argtypes = [i] * 6 + [vp] * 17 + [sz, vp]
    lib.gdn2_chunk_bwd.restype = i
    lib.gdn2_chunk_bwd_noalloc.argtypes = [i] * 6 + [vp] * 16 + [vp]
    lib.gdn2_chunk_bwd_noalloc.restype = i
    lib.gdn2_chunk_fwd_varlen.argtypes = [i] * 6 + [vp] * 11 + [sz, vp]
    lib.gdn2_chunk_fwd_varlen.restype = i
    lib.gdn2_chunk_bwd_varlen.argtypes = [i] * 6 + [vp] * 18 + [sz, vp]
    lib.gdn2_chunk_bwd_varlen.restype = i
    lib.gdn2_chunk_fwd_gated.argtypes = [i] * 7 + [vp] * 10 + [sz, vp]
    lib.gdn2_chunk_fwd_gated.restype = i
    lib.gdn2_chunk_bwd_gated.argtypes = [i] * 7 + [vp] * 17 + [sz, vp]
    lib.gdn2_chunk_bwd_gated.restype = i
    lib.gdn2_decode_step_gated.argtypes = [i] * 6 + [vp] * 9 + [sz, vp]
    lib.gdn2_decode_step_gated.restype = i
    lib.gdn2_chunk_fwd_host.argtypes = [i] * 6 + [vp] * 10 + [sz, vp]
    lib.gdn2_chunk_fwd_host.restype = i
    lib.gdn2_chunk_fwd_save.argtypes = [i] * 6 + [vp] * 10 + [sz, vp]
    lib.gdn2_chunk_fwd_save.restype = i
    lib.gdn2_chunk_bwd_saved.argtypes = [i] * 6 + [vp] * 17 + [sz, vp]
    lib.gdn2_chunk_bwd_saved.restype = i
    lib.gdn2_prologue.argtypes = [i] * 5 + [vp] * 8 + [vp]
    lib.gdn2_prologue.restype = i
    lib.gdn2_workspace_size_gated.argtypes = [i] * 8
    lib.gdn2_workspace_size_gated.restype = sz
    lib.gdn2_workspace_size.argtypes = [i] * 7
    lib.gdn2_workspace_size.restype = sz
    lib.gdn2_strerror.argtypes = [i]
    lib.gdn2_strerror.restype = ctypes.c_char_p
    lib.gdn2_sync_status.argtypes = [vp]
    lib.gdn2_sync_status.restype = i
    lib.gdn2_selftest_timeout.argtypes = [i, vp]
    lib.gdn2_selftest_timeout.restype = i
    _lib = lib
    return lib


def raw():
    """The loaded ctypes library object (C names, raw pointers)."""
    return load()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GDN2_F32
    if t.dtype == torch.bfloat16:
        return GDN2_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _check(fn: str, st: int):
    if st != GDN2_OK:
        raise Gdn2Error(fn, st)


def _cuda_contig(name, t, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def gdn2_workspace_size(which: int, dtype: torch.dtype, B: int, T: int, H: int, Dk: int, Dv: int) -> int:
    dt = GDN2_F32 if dtype == torch.float32 else GDN2_BF16
    return int(raw().gdn2_workspace_size(which, dt, B, T, H, Dk, Dv))


def gdn2_chunk_fwd(q, k, v, log_alpha, b, w, S0=None, *, o=None, S_T=None, want_state=True,
                   workspace=None, stream=None):
    """Chunkwise forward.  Returns (o, S_T); S_T is None when want_state is False."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    for n, t in (("q", q), ("k", k), ("v", v), ("b", b), ("w", w)):
        _cuda_contig(n, t, q.dtype)
    _cuda_contig("log_alpha", log_alpha, torch.float32)
    _cuda_contig("S0", S0, torch.float32)
    if o is None:
        o = torch.empty(B, T, H, Dv, dtype=q.dtype, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty(B, H, Dk, Dv, dtype=torch.float32, device=q.device)
    ws = workspace
    if ws is None:  # few long chains run as a chunk-parallel scan, which needs a workspace
        nb = gdn2_workspace_size(0, q.dtype, B, T, H, Dk, Dv)
        ws = torch.empty(nb, dtype=torch.uint8, device=q.device) if nb > 0 else None
    st = raw().gdn2_chunk_fwd(dt, B, T, H, Dk, Dv, _p(q), _p(k), _p(v), _p(log_alpha), _p(b), _p(w),
                              _p(S0), _p(o), _p(S_T), _p(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                              _stream(stream))
    _check("gdn2_chunk_fwd", st)
    return o, S_T


def gdn2_decode_step(q, k, v, log_alpha, b, w, S, *, o=None, stream=None):
    """One decode step; S [N,H,Dk,Dv] fp32 is updated in place.  Returns o [N,H,Dv]."""
    N, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    for n, t in (("q", q), ("k", k), ("v", v), ("b", b), ("w", w)):
        _cuda_contig(n, t, q.dtype)
    _cuda_contig("log_alpha", log_alpha, torch.float32)
    _cuda_contig("S", S, torch.float32)
    if o is None:
        o = torch.empty(N, H, Dv, dtype=q.dtype, device=q.device)
    st = raw().gdn2_decode_step(dt, N, H, Dk, Dv, _p(q), _p(k), _p(v), _p(log_alpha), _p(b), _p(w),
                                _p(S), _p(o), _stream(stream))
    _check("gdn2_decode_step", st)
    return o


def gdn2_chunk_fwd_host(q, k, v, log_alpha, b, w, S0=None, *, o=None, S_T=None, workspace=None, stream=None,
                        device=None):
    """The forward on host (CPU) tensors: inputs copied in and o, S_T copied out inside the call,
    pipelined by batch rows.  Pinned host tensors let the copies overlap.  Returns (o, S_T) as
    host tensors; ``workspace`` is device staging of gdn2_workspace_size(4, ...) bytes."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    for n, t in (("q", q), ("k", k), ("v", v), ("b", b), ("w", w), ("log_alpha", log_alpha)):
        if t.device.type != "cpu" or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous host tensor")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if o is None:
        o = torch.empty(B, T, H, Dv, dtype=q.dtype, pin_memory=True)
    if S_T is None:
        S_T = torch.empty(B, H, Dk, Dv, dtype=torch.float32, pin_memory=True)
    if workspace is None:
        nbytes = gdn2_workspace_size(4, q.dtype, B, T, H, Dk, Dv)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    st = raw().gdn2_chunk_fwd_host(dt, B, T, H, Dk, Dv, _p(q), _p(k), _p(v), _p(log_alpha), _p(b), _p(w),
                                   _p(S0), _p(o), _p(S_T), _p(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check("gdn2_chunk_fwd_host", st)
    return o, S_T


def gdn2_chunk_fwd_save(q, k, v, log_alpha, b, w, S0=None, *, workspace=None, o=None, S_T=None, stream=None):
    """The forward that also records the chunk-boundary states into the backward's workspace.
    Returns (o, S_T, workspace); pass the workspace to gdn2_chunk_bwd_saved."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    for n, t in (("q", q), ("k", k), ("v", v), ("b", b), ("w", w)):
        _cuda_contig(n, t, q.dtype)
    _cuda_contig("log_alpha", log_alpha, torch.float32)
    _cuda_contig("S0", S0, torch.float32)
    if o is None:
        o = torch.empty(B, T, H, Dv, dtype=q.dtype, device=q.device)
    if S_T is None:
        S_T = torch.empty(B, H, Dk, Dv, dtype=torch.float32, device=q.device)
    if workspace is None:
        nbytes = gdn2_workspace_size(1, q.dtype, B, T, H, Dk, Dv)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    st = raw().gdn2_chunk_fwd_save(dt, B, T, H, Dk, Dv, _p(q), _p(k), _p(v), _p(log_alpha), _p(b), _p(w),
                                   _p(S0), _p(o), _p(S_T), _p(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check("gdn2_chunk_fwd_save", st)
    return o, S_T, workspace


def gdn2_chunk_bwd_saved(q, k, v, log_alpha, b, w, S0, d_o, dS_T=None, *, workspace, out=None, stream=None):
    """gdn2_chunk_bwd on the states gdn2_chunk_fwd_save recorded into ``workspace``."""
    return gdn2_chunk_bwd(q, k, v, log_alpha, b, w, S0, d_o, dS_T, workspace=workspace, out=out, stream=stream,
                          _saved=True)


def gdn2_chunk_bwd(q, k, v, log_alpha, b, w, S0, d_o, dS_T=None, *, workspace=None, out=None, stream=None,
                   _saved=False):
    """Gate-aware backward.  Returns dict(dq, dk, dv, dlog_alpha, db, dw, dS0)."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    for n, t in (("q", q), ("k", k), ("v", v), ("b", b), ("w", w), ("d_o", d_o)):
        _cuda_contig(n, t, q.dtype)
    _cuda_contig("log_alpha", log_alpha, torch.float32)
    _cuda_contig("S0", S0, torch.float32)
    _cuda_contig("dS_T", dS_T, torch.float32)
    if out is None:
        out = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
               "dlog_alpha": torch.empty_like(log_alpha), "db": torch.empty_like(b),
               "dw": torch.empty_like(w),
               "dS0": torch.empty(B, H, Dk, Dv, dtype=torch.float32, device=q.device)}
    if workspace is None:
        nbytes = gdn2_workspace_size(1, q.dtype, B, T, H, Dk, Dv)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q.device)
    fn = raw().gdn2_chunk_bwd_saved if _saved else raw().gdn2_chunk_bwd
    st = fn(dt, B, T, H, Dk, Dv, _p(q), _p(k), _p(v), _p(log_alpha), _p(b), _p(w),
            _p(S0), _p(d_o), _p(dS_T), _p(out["dq"]), _p(out["dk"]), _p(out["dv"]),
            _p(out["dlog_alpha"]), _p(out["db"]), _p(out["dw"]), _p(out["dS0"]),
            _p(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check("gdn2_chunk_bwd_saved" if _saved else "gdn2_chunk_bwd", st)
    return out


def gdn2_chunk_bwd_noalloc(q, k, v, log_alpha, b, w, S0, d_o, dS_T=None, *, out, stream=None):
    """The backward with the library's static scratch array instead of a workspace.

    ``out`` holds caller-allocated gradient tensors (keys as returned by
    gdn2_chunk_bwd); nothing is allocated here or in the library.  Problems
    whose workspace would exceed NOALLOC_MAX_SCRATCH_BYTES raise
    GDN2_ERR_TOO_LARGE.  Calls that overlap on the GPU share the array and race.
    """
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    for n, t in (("q", q), ("k", k), ("v", v), ("b", b), ("w", w), ("d_o", d_o)):
        _cuda_contig(n, t, q.dtype)
    _cuda_contig("log_alpha", log_alpha, torch.float32)
    _cuda_contig("S0", S0, torch.float32)
    _cuda_contig("dS_T", dS_T, torch.float32)
    for n in ("dq", "dk", "dv", "db", "dw"):
        _cuda_contig(n, out[n], q.dtype)
    _cuda_contig("dlog_alpha", out["dlog_alpha"], torch.float32)
    _cuda_contig("dS0", out["dS0"], torch.float32)
    st = raw().gdn2_chunk_bwd_noalloc(dt, B, T, H, Dk, Dv, _p(q), _p(k), _p(v), _p(log_alpha), _p(b),
                                      _p(w), _p(S0), _p(d_o), _p(dS_T), _p(out["dq"]), _p(out["dk"]),
                                      _p(out["dv"]), _p(out["dlog_alpha"]), _p(out["db"]),
                                      _p(out["dw"]), _p(out["dS0"]), _stream(stream))
    _check("gdn2_chunk_bwd_noalloc", st)
    return out


def _packed(t):
    """[total_T, H, D] view of a packed token tensor given as [total_T, H, D] or [1, total_T, H, D]."""
    if t.dim() == 4:
        if t.shape[0] != 1:
            raise ValueError("packed tensors are [total_T, H, D] (or [1, total_T, H, D])")
        return t[0]
    return t


def gdn2_chunk_fwd_varlen(q, k, v, log_alpha, b, w, cu_seqlens, S0=None, *, o=None, S_T=None, want_state=True,
                          workspace=None, stream=None):
    """Forward over N packed sequences (cu_seqlens int32 [N+1] on the device).
    Returns (o [total_T, H, Dv], S_T [N, H, Dk, Dv] or None)."""
    q3, k3, v3, g3, b3, w3 = (_packed(t) for t in (q, k, v, log_alpha, b, w))
    total_T, H, Dk = q3.shape
    Dv = v3.shape[-1]
    N = cu_seqlens.numel() - 1
    dt = _dt(q3)
    for n, t in (("q", q3), ("k", k3), ("v", v3), ("b", b3), ("w", w3)):
        _cuda_contig(n, t, q3.dtype)
    _cuda_contig("log_alpha", g3, torch.float32)
    _cuda_contig("cu_seqlens", cu_seqlens, torch.int32)
    _cuda_contig("S0", S0, torch.float32)
    if o is None:
        o = torch.empty(total_T, H, Dv, dtype=q3.dtype, device=q3.device)
    if S_T is None and want_state:
        S_T = torch.empty(N, H, Dk, Dv, dtype=torch.float32, device=q3.device)
    ws = workspace
    st = raw().gdn2_chunk_fwd_varlen(dt, N, total_T, H, Dk, Dv, _p(cu_seqlens), _p(q3), _p(k3), _p(v3), _p(g3),
                                     _p(b3), _p(w3), _p(S0), _p(o), _p(S_T), _p(ws),
                                     0 if ws is None else ws.numel() * ws.element_size(), _stream(stream))
    _check("gdn2_chunk_fwd_varlen", st)
    return o, S_T


def gdn2_chunk_bwd_varlen(q, k, v, log_alpha, b, w, cu_seqlens, S0, d_o, dS_T=None, *, workspace=None, out=None,
                          stream=None):
    """Backward over N packed sequences.  Returns dict(dq, dk, dv, dlog_alpha, db, dw, dS0)."""
    q3, k3, v3, g3, b3, w3, do3 = (_packed(t) for t in (q, k, v, log_alpha, b, w, d_o))
    total_T, H, Dk = q3.shape
    Dv = v3.shape[-1]
    N = cu_seqlens.numel() - 1
    dt = _dt(q3)
    for n, t in (("q", q3), ("k", k3), ("v", v3), ("b", b3), ("w", w3), ("d_o", do3)):
        _cuda_contig(n, t, q3.dtype)
    _cuda_contig("log_alpha", g3, torch.float32)
    _cuda_contig("cu_seqlens", cu_seqlens, torch.int32)
    _cuda_contig("S0", S0, torch.float32)
    _cuda_contig("dS_T", dS_T, torch.float32)
    if out is None:
        out = {"dq": torch.empty_like(q3), "dk": torch.empty_like(k3), "dv": torch.empty_like(v3),
               "dlog_alpha": torch.empty_like(g3), "db": torch.empty_like(b3), "dw": torch.empty_like(w3),
               "dS0": torch.empty(N, H, Dk, Dv, dtype=torch.float32, device=q3.device)}
    if workspace is None:
        nbytes = gdn2_workspace_size(3, q3.dtype, N, total_T, H, Dk, Dv)
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=q3.device)
    st = raw().gdn2_chunk_bwd_varlen(dt, N, total_T, H, Dk, Dv, _p(cu_seqlens), _p(q3), _p(k3), _p(v3), _p(g3),
                                     _p(b3), _p(w3), _p(S0), _p(do3), _p(dS_T), _p(out["dq"]), _p(out["dk"]),
                                     _p(out["dv"]), _p(out["dlog_alpha"]), _p(out["db"]), _p(out["dw"]),
                                     _p(out["dS0"]), _p(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream))
    _check("gdn2_chunk_bwd_varlen", st)
    return out


def gdn2_workspace_size_gated(which: int, flags: int, dtype: torch.dtype, B: int, T: int, H: int, Dk: int,
                              Dv: int) -> int:
    dt = GDN2_F32 if dtype == torch.float32 else GDN2_BF16
    return int(raw().gdn2_workspace_size_gated(which, flags, dt, B, T, H, Dk, Dv))


def _ws(workspace, nbytes, device):
    if workspace is None and nbytes > 0:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace, (0 if workspace is None else workspace.numel() * workspace.element_size())


def gdn2_chunk_fwd_gated(q, k, v, log_alpha, b, w, S0=None, *, flags, o=None, S_T=None, want_state=True,
                         workspace=None, stream=None):
    """Forward with gate layouts given by `flags` (scalar gates are [B, T, H]; absent ones may be None)."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    for n, t in (("q", q), ("k", k), ("v", v)):
        _cuda_contig(n, t, q.dtype)
    for n, t in (("b", b), ("w", w)):
        _cuda_contig(n, t, q.dtype)
    _cuda_contig("log_alpha", log_alpha, torch.float32)
    _cuda_contig("S0", S0, torch.float32)
    if o is None:
        o = torch.empty(B, T, H, Dv, dtype=q.dtype, device=q.device)
    if S_T is None and want_state:
        S_T = torch.empty(B, H, Dk, Dv, dtype=torch.float32, device=q.device)
    ws, nb = _ws(workspace, gdn2_workspace_size_gated(0, flags, q.dtype, B, T, H, Dk, Dv), q.device)
    st = raw().gdn2_chunk_fwd_gated(flags, dt, B, T, H, Dk, Dv, _p(q), _p(k), _p(v), _p(log_alpha), _p(b), _p(w),
                                    _p(S0), _p(o), _p(S_T), _p(ws), nb, _stream(stream))
    _check("gdn2_chunk_fwd_gated", st)
    return o, S_T


def gdn2_chunk_bwd_gated(q, k, v, log_alpha, b, w, S0, d_o, dS_T=None, *, flags, workspace=None, out=None,
                         stream=None):
    """Backward with gate layouts given by `flags`; gate gradients come back in the gates' layouts
    (None for absent gates)."""
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    for n, t in (("q", q), ("k", k), ("v", v), ("d_o", d_o), ("b", b), ("w", w)):
        _cuda_contig(n, t, q.dtype)
    _cuda_contig("log_alpha", log_alpha, torch.float32)
    _cuda_contig("S0", S0, torch.float32)
    _cuda_contig("dS_T", dS_T, torch.float32)
    if out is None:
        out = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
               "dlog_alpha": None if log_alpha is None else torch.empty_like(log_alpha),
               "db": None if b is None else torch.empty_like(b), "dw": None if w is None else torch.empty_like(w),
               "dS0": torch.empty(B, H, Dk, Dv, dtype=torch.float32, device=q.device)}
    ws, nb = _ws(workspace, gdn2_workspace_size_gated(1, flags, q.dtype, B, T, H, Dk, Dv), q.device)
    st = raw().gdn2_chunk_bwd_gated(flags, dt, B, T, H, Dk, Dv, _p(q), _p(k), _p(v), _p(log_alpha), _p(b), _p(w),
                                    _p(S0), _p(d_o), _p(dS_T), _p(out["dq"]), _p(out["dk"]), _p(out["dv"]),
                                    _p(out["dlog_alpha"]), _p(out["db"]), _p(out["dw"]), _p(out["dS0"]), _p(ws), nb,
                                    _stream(stream))
    _check("gdn2_chunk_bwd_gated", st)
    return out


def gdn2_decode_step_gated(q, k, v, log_alpha, b, w, S, *, flags, o=None, workspace=None, stream=None):
    """Decode step with gate layouts given by `flags` (scalar gates are [N, H])."""
    N, H, Dk = q.shape
    Dv = v.shape[-1]
    dt = _dt(q)
    for n, t in (("q", q), ("k", k), ("v", v), ("b", b), ("w", w)):
        _cuda_contig(n, t, q.dtype)
    _cuda_contig("log_alpha", log_alpha, torch.float32)
    _cuda_contig("S", S, torch.float32)
    if o is None:
        o = torch.empty(N, H, Dv, dtype=q.dtype, device=q.device)
    ws, nb = _ws(workspace, gdn2_workspace_size_gated(2, flags, q.dtype, N, 1, H, Dk, Dv), q.device)
    st = raw().gdn2_decode_step_gated(flags, dt, N, H, Dk, Dv, _p(q), _p(k), _p(v), _p(log_alpha), _p(b), _p(w),
                                      _p(S), _p(o), _p(ws), nb, _stream(stream))
    _check("gdn2_decode_step_gated", st)
    return o


def gdn2_prologue(q, k, b, w, *, flags, out=None, stream=None):
    """The input prologue alone: returns dict(q, k, b, w) with q, k normalised (QK_L2NORM) and
    b, w through the sigmoid (BW_LOGITS); parts the flags do not ask for come back as None.
    q, k: [..., H, D]; b, w: [..., H, D] or, with ERASE_SCALAR / WRITE_SCALAR, [..., H]."""
    H, D = q.shape[-2], q.shape[-1]
    N = q.numel() // (H * D)
    dt = _dt(q)
    norm = bool(flags & QK_L2NORM)
    sig_b = bool(flags & BW_LOGITS) and not flags & ERASE_NONE
    sig_w = bool(flags & BW_LOGITS) and not flags & WRITE_NONE
    for n, t, used in (("q", q, norm), ("k", k, norm), ("b", b, sig_b), ("w", w, sig_w)):
        if used:
            _cuda_contig(n, t, q.dtype)
    if out is None:
        out = {"q": torch.empty_like(q) if norm else None, "k": torch.empty_like(k) if norm else None,
               "b": torch.empty_like(b) if sig_b else None, "w": torch.empty_like(w) if sig_w else None}
    st = raw().gdn2_prologue(flags, dt, N, H, D, _p(q if norm else None), _p(k if norm else None),
                             _p(b if sig_b else None), _p(w if sig_w else None), _p(out["q"]), _p(out["k"]),
                             _p(out["b"]), _p(out["w"]), _stream(stream))
    _check("gdn2_prologue", st)
    return out


def gdn2_sync_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the kernel status word."""
    return int(raw().gdn2_sync_status(_stream(stream)))


def gdn2_selftest_timeout(limit_us: int = 2000, stream=None):
    """Failure-detection self-test: enqueue one bounded wait on a barrier phase nothing
    completes; the next gdn2_sync_status() returns GDN2_ERR_TIMEOUT (-7)."""
    _check("gdn2_selftest_timeout", raw().gdn2_selftest_timeout(int(limit_us), _stream(stream)))


def gdn2_strerror(status: int) -> str:
    return raw().gdn2_strerror(status).decode()
