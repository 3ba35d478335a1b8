"""fp64 CPU oracle of the selective state-space recurrence (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
reference arm may import this package.  The product path
(``state_space_model_07_b200``) never imports it, and this package imports
nothing from the product path: the two share no code.

The arithmetic lives in ``ssd_oracle.c`` (a literal token-by-token loop in
double precision, see the header there for the definition and its sources) and
``ssd_oracle_bwd.c`` (the gradient of that loop: the adjoint reverse sweep).
This module only marshals numpy arrays to them.

Every input is taken as the exact values the GPU sees: bf16 / fp32 tensors are
widened to float64 without rounding before the call.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_SRC_BWD = os.path.join(_HERE, "ssd_oracle_bwd.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compiles ssd_oracle.c and ssd_oracle_bwd.c into libssd_oracle.so (plain
    gcc, no fast-math, no FMA contraction, so the loops are evaluated exactly as
    written)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_BWD))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-pthread", _SRC, _SRC_BWD, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_softplus.restype = ctypes.c_double
        lib.oracle_softplus.argtypes = [ctypes.c_double]
        lib.oracle_ssd_scan.restype = ctypes.c_int
        lib.oracle_ssd_scan.argtypes = [_i64] * 7 + [_D] * 8 + [_I32, _D, _D, ctypes.c_int]
        lib.oracle_state_update.restype = ctypes.c_int
        lib.oracle_state_update.argtypes = [_i64] * 5 + [_D] * 9
        lib.oracle_ssd_scan_bwd.restype = ctypes.c_int
        lib.oracle_ssd_scan_bwd.argtypes = [_i64] * 7 + [_D] * 8 + [_I32] + [_D] * 10
        _lib = lib
    return _lib


def _f64(a):
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor: widen exactly on the CPU
        a = a.detach().to("cpu")
        import torch
        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a, typ=_D):
    return None if a is None else a.ctypes.data_as(typ)


def softplus(z: float) -> float:
    return _load().oracle_softplus(float(z))


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def ssd_scan(x, dt, A, B, C, dt_bias=None, D=None, init_state=None, seq_idx=None,
             nseqs=None, nthreads=None, want_final=True):
    """Token-by-token fp64 recurrence.

    Shapes: x (b, L, H, P); dt (b, L, H); A (H,); B, C (b, L, G, N);
    dt_bias, D (H,) or None; init_state (S, H, N, P) or None;
    seq_idx (b=1, L) int or None.  S = nseqs with seq_idx, else b.
    Returns (y (b, L, H, P), final_state (S, H, N, P) or None) as float64.
    """
    x, dt, A, B, C = (_f64(v) for v in (x, dt, A, B, C))
    dt_bias, D, init_state = _f64(dt_bias), _f64(D), _f64(init_state)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt.shape == (b, L, H) and A.shape == (H,)
    assert B.shape == (b, L, G, N) and C.shape == (b, L, G, N)
    si = None
    if seq_idx is not None:
        if hasattr(seq_idx, "detach"):
            seq_idx = seq_idx.detach().to("cpu").numpy()
        si = np.ascontiguousarray(np.asarray(seq_idx, dtype=np.int32).reshape(-1))
        assert b == 1 and si.shape == (L,)
        if nseqs is None:
            nseqs = int(si[-1]) + 1 if L > 0 else 0
        S = nseqs
    else:
        nseqs = b
        S = b
    if init_state is not None:
        assert init_state.shape == (S, H, N, P), init_state.shape
    y = np.zeros((b, L, H, P), dtype=np.float64)
    fs = np.zeros((S, H, N, P), dtype=np.float64) if want_final else None
    rc = _load().oracle_ssd_scan(
        b, L, H, P, N, G, nseqs, _ptr(x), _ptr(dt), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C),
        _ptr(D), _ptr(init_state), _ptr(si, _I32), _ptr(y), _ptr(fs),
        int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError(f"oracle_ssd_scan rejected its arguments (rc={rc})")
    return y, fs


def state_update(state, x, dt, A, B, C, dt_bias=None, D=None):
    """One fp64 decode step.  state (b, H, N, P) is copied, not modified.
    Returns (new_state, y (b, H, P))."""
    st = _f64(state).copy()
    x, dt, A, B, C = (_f64(v) for v in (x, dt, A, B, C))
    dt_bias, D = _f64(dt_bias), _f64(D)
    b, H, N, P = st.shape
    G = B.shape[1]
    assert x.shape == (b, H, P) and dt.shape == (b, H) and B.shape == (b, G, N)
    y = np.zeros((b, H, P), dtype=np.float64)
    rc = _load().oracle_state_update(b, H, P, N, G, _ptr(st), _ptr(x), _ptr(dt), _ptr(dt_bias),
                                     _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y))
    if rc != 0:
        raise ValueError(f"oracle_state_update rejected its arguments (rc={rc})")
    return st, y


def ssd_scan_bwd(x, dt, A, B, C, dy, dt_bias=None, D=None, init_state=None, seq_idx=None,
                 nseqs=None, dfinal=None):
    """Gradient of J = sum(dy * y) + sum(dfinal * final_state) through the scan.

    Same inputs and shapes as ``ssd_scan``; dy (b, L, H, P); dfinal (S, H, N, P)
    or None.  Returns a dict of float64 arrays: x, dt, dt_bias, A, B, C, D,
    init_state (the last is the gradient for the initial state, zero or not).
    """
    x, dt, A, B, C, dy = (_f64(v) for v in (x, dt, A, B, C, dy))
    dt_bias, D, init_state, dfinal = _f64(dt_bias), _f64(D), _f64(init_state), _f64(dfinal)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    si = None
    if seq_idx is not None:
        if hasattr(seq_idx, "detach"):
            seq_idx = seq_idx.detach().to("cpu").numpy()
        si = np.ascontiguousarray(np.asarray(seq_idx, dtype=np.int32).reshape(-1))
        assert b == 1 and si.shape == (L,)
        if nseqs is None:
            nseqs = int(si[-1]) + 1 if L > 0 else 0
        S = nseqs
    else:
        nseqs = b
        S = b
    assert dy.shape == x.shape
    out = {"x": np.zeros_like(x), "dt": np.zeros((b, L, H)), "dt_bias": np.zeros(H), "A": np.zeros(H),
           "B": np.zeros((b, L, G, N)), "C": np.zeros((b, L, G, N)), "D": np.zeros(H),
           "init_state": np.zeros((S, H, N, P))}
    rc = _load().oracle_ssd_scan_bwd(
        b, L, H, P, N, G, nseqs, _ptr(x), _ptr(dt), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
        _ptr(init_state), _ptr(si, _I32), _ptr(dy), _ptr(dfinal),
        *(_ptr(out[k]) for k in ("x", "dt", "dt_bias", "A", "B", "C", "D", "init_state")))
    if rc != 0:
        raise ValueError(f"oracle_ssd_scan_bwd rejected its arguments (rc={rc})")
    return out
