"""fp64 CPU oracle for the Gated DeltaNet-2 recurrence.

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  It shares no code with
the CUDA path (``gated_delta_rule_78_b200``) and never imports it.

* ``ref_fwd`` / ``ref_bwd`` / ``ref_decode`` call the C token recurrence in
  ``gdn2_ref.c`` (threads over (batch, head)).
* ``oracle.checks`` holds separately written NumPy forms used to pin it:
  KDA, Gated DeltaNet and DeltaNet recurrences, the b = 0 closed form, the
  chunkwise (WY) forward and its hand-derived backward.

Every function here is pinned by a ``-m "not gpu"`` test; none is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.gdn2_ref_fwd.argtypes = [i, i, i, i, i] + [dp] * 9 + [i]
        lib.gdn2_ref_fwd.restype = i
        lib.gdn2_ref_bwd.argtypes = [i, i, i, i, i] + [dp] * 16 + [i]
        lib.gdn2_ref_bwd.restype = i
        lib.gdn2_ref_decode.argtypes = [i, i, i, i] + [dp] * 8 + [i]
        lib.gdn2_ref_decode.restype = i
        _LIB = lib
    return _LIB


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return ctypes.POINTER(ctypes.c_double)()
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def ref_fwd(q, k, v, g, b, w, S0=None, nthreads=None):
    """Token recurrence forward.  Returns (o [B,T,H,Dv], S_T [B,H,Dk,Dv]) in fp64."""
    q, k, v, g, b, w, S0 = map(_f64, (q, k, v, g, b, w, S0))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    o = np.empty((B, T, H, Dv))
    ST = np.empty((B, H, Dk, Dv))
    rc = _lib().gdn2_ref_fwd(B, T, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b),
                             _ptr(w), _ptr(S0), _ptr(o), _ptr(ST), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"gdn2_ref_fwd failed ({rc})")
    return o, ST


def ref_bwd(q, k, v, g, b, w, S0, do, dST=None, nthreads=None):
    """Reverse-mode gradients of <o, do> + <S_T, dST>.  Returns a dict of fp64 arrays."""
    q, k, v, g, b, w, S0, do, dST = map(_f64, (q, k, v, g, b, w, S0, do, dST))
    B, T, H, Dk = q.shape
    Dv = v.shape[-1]
    out = {n: np.zeros_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dg", g),
                                            ("db", b), ("dw", w))}
    out["dS0"] = np.zeros((B, H, Dk, Dv))
    rc = _lib().gdn2_ref_bwd(B, T, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b),
                             _ptr(w), _ptr(S0), _ptr(do), _ptr(dST), _ptr(out["dq"]),
                             _ptr(out["dk"]), _ptr(out["dv"]), _ptr(out["dg"]), _ptr(out["db"]),
                             _ptr(out["dw"]), _ptr(out["dS0"]), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"gdn2_ref_bwd failed ({rc})")
    return out


def ref_decode(q, k, v, g, b, w, S, nthreads=None, inplace=False):
    """One decode step: inputs [N,H,D], S [N,H,Dk,Dv].  Returns (o, S_new) in fp64.  With
    inplace=True, S must be a C-contiguous fp64 array; it is updated in place and returned."""
    q, k, v, g, b, w = map(_f64, (q, k, v, g, b, w))
    if inplace:
        if not (isinstance(S, np.ndarray) and S.dtype == np.float64 and S.flags["C_CONTIGUOUS"]):
            raise ValueError("inplace ref_decode needs a C-contiguous fp64 state")
    else:
        S = _f64(S).copy()
    N, H, Dk = q.shape
    Dv = v.shape[-1]
    o = np.empty((N, H, Dv))
    rc = _lib().gdn2_ref_decode(N, H, Dk, Dv, _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b),
                                _ptr(w), _ptr(S), _ptr(o), nthreads or default_threads())
    if rc != 0:
        raise RuntimeError(f"gdn2_ref_decode failed ({rc})")
    return o, S


# ---------------------------------------------------------------- input prologue
# The aixai.ru post's architecture paragraph ("Как это реализуется на практике"): queries and
# keys are L2-normalised before the recurrent update, the erase and write gates come from
# their own projections (logits through the logistic sigmoid, gates in [0, 1]), and log alpha
# is computed outside the kernel (so it is an input of every function below).
NORM_EPS = 1e-6


def ref_prologue(q, k, b, w, norm=True, sigmoid=True):
    """q, k -> x / sqrt(sum_c x^2 + NORM_EPS) per (token, head) over the last axis;
    b, w -> 1 / (1 + exp(-x)) elementwise (any layout; None passes through).  fp64."""
    q, k = _f64(q), _f64(k)
    if norm:
        q = q / np.sqrt((q * q).sum(-1, keepdims=True) + NORM_EPS)
        k = k / np.sqrt((k * k).sum(-1, keepdims=True) + NORM_EPS)
    if sigmoid:
        b = None if b is None else 1.0 / (1.0 + np.exp(-_f64(b)))
        w = None if w is None else 1.0 / (1.0 + np.exp(-_f64(w)))
    return q, k, (None if b is None else _f64(b)), (None if w is None else _f64(w))


def ref_fwd_prologue(q, k, v, g, b, w, S0=None, norm=True, sigmoid=True, nthreads=None):
    """The forward on raw q, k and gate logits: ref_fwd after ref_prologue."""
    qn, kn, bs, ws = ref_prologue(q, k, b, w, norm, sigmoid)
    return ref_fwd(qn, kn, v, g, bs, ws, S0, nthreads)


def ref_bwd_prologue(q, k, v, g, b, w, S0, do, dST=None, norm=True, sigmoid=True, nthreads=None):
    """Gradients with respect to the raw q, k and the gate logits: ref_bwd at the normalised /
    activated inputs, then the two derivatives of the prologue.  For x_n = x r with
    r = (|x|^2 + eps)^-1/2, d x_n / d x = r (I - x_n x_n^T), so dx = r (dx_n - x_n (x_n . dx_n));
    the sigmoid's derivative is s (1 - s)."""
    qn, kn, bs, ws = ref_prologue(q, k, b, w, norm, sigmoid)
    out = ref_bwd(qn, kn, v, g, bs, ws, S0, do, dST, nthreads)
    if norm:
        for x, key in ((_f64(q), "dq"), (_f64(k), "dk")):
            r = 1.0 / np.sqrt((x * x).sum(-1, keepdims=True) + NORM_EPS)
            xn = x * r
            dxn = out[key]
            out[key] = r * (dxn - xn * (xn * dxn).sum(-1, keepdims=True))
    if sigmoid:
        out["db"] = out["db"] * bs * (1.0 - bs)
        out["dw"] = out["dw"] * ws * (1.0 - ws)
    return out
