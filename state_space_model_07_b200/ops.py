"""Python face of libssd.so: the same two calls, argument marshalling only.

torch is used for device memory and the current stream; every step of the
computation runs in the library's CUDA kernels.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib
from ._lib import SsdDims, SsdError  # noqa: F401  (re-export)

_DT = {torch.float32: _lib.SSD_F32, torch.bfloat16: _lib.SSD_BF16}


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, name, dtype=None, ndim=None, device=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def chunk_scan_fwd(x, dt, A, B, C, *, dt_bias=None, D=None, init_state=None, seq_idx=None,
                   nseqs: Optional[int] = None, chunk: int = 256, y=None, final_state=None,
                   want_final: bool = True, stream=None):
    """SSD chunked scan forward.  Returns (y, final_state or None).

    x (b,L,H,P), dt (b,L,H), B/C (b,L,G,N) in float32 or bfloat16 (all the same);
    A, dt_bias, D (H,) float32; init_state (S,H,N,P) float32; seq_idx (1,L) or (L,)
    int32 with batch 1 (then pass nseqs, or it is read from seq_idx[-1] with a sync).
    """
    _need(x, "x", ndim=4)
    dev = x.device
    if x.dtype not in _DT:
        raise ValueError(f"x dtype {x.dtype} not supported")
    for t, n, nd in ((dt, "dt", 3), (B, "B", 4), (C, "C", 4)):
        _need(t, n, dtype=x.dtype, ndim=nd, device=dev)
    _need(A, "A", torch.float32, 1, dev)
    _need(dt_bias, "dt_bias", torch.float32, 1, dev)
    _need(D, "D", torch.float32, 1, dev)
    _need(init_state, "init_state", torch.float32, 4, dev)
    _need(seq_idx, "seq_idx", torch.int32, None, dev)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if seq_idx is not None:
        if nseqs is None:
            nseqs = int(seq_idx.reshape(-1)[-1].item()) + 1 if L > 0 else 0
        S = nseqs
    else:
        S = b
    if y is None:
        y = torch.empty_like(x)
    else:
        _need(y, "y", x.dtype, 4, dev)
    if final_state is None and want_final:
        final_state = torch.empty((S, H, N, P), dtype=torch.float32, device=dev)
    elif final_state is not None:
        _need(final_state, "final_state", torch.float32, 4, dev)
    dims = SsdDims(b, L, H, P, N, G, S if seq_idx is not None else 0, _DT[x.dtype])
    with torch.cuda.device(dev):
        rc = _lib.lib().ssd_chunk_scan_fwd(
            ctypes.byref(dims), _p(x), _p(dt), _p(dt_bias), _p(A), _p(B), _p(C), _p(D),
            _p(init_state), _p(seq_idx), int(chunk), _p(y), _p(final_state), _stream(stream, dev))
    _lib.check(rc)
    return y, final_state


def chunk_scan_bwd(x, dt, A, B, C, dy, *, dt_bias=None, D=None, init_state=None, seq_idx=None,
                   nseqs: Optional[int] = None, chunk: int = 256, dfinal=None, stream=None):
    """Gradient of J = sum(dy * y) + sum(dfinal * final_state) through the scan.

    Inputs as for ``chunk_scan_fwd``; dy (b,L,H,P) in x's dtype; dfinal (S,H,N,P)
    float32 or None.  Returns a dict of gradients: x, dt, B, C (dtype of x), dt_bias,
    A, D (H,) float32, init_state (S,H,N,P) float32.
    """
    _need(x, "x", ndim=4)
    dev = x.device
    if x.dtype not in _DT:
        raise ValueError(f"x dtype {x.dtype} not supported")
    for t, n, nd in ((dt, "dt", 3), (B, "B", 4), (C, "C", 4), (dy, "dy", 4)):
        _need(t, n, dtype=x.dtype, ndim=nd, device=dev)
    _need(A, "A", torch.float32, 1, dev)
    _need(dt_bias, "dt_bias", torch.float32, 1, dev)
    _need(D, "D", torch.float32, 1, dev)
    _need(init_state, "init_state", torch.float32, 4, dev)
    _need(dfinal, "dfinal", torch.float32, 4, dev)
    _need(seq_idx, "seq_idx", torch.int32, None, dev)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if seq_idx is not None:
        if nseqs is None:
            nseqs = int(seq_idx.reshape(-1)[-1].item()) + 1 if L > 0 else 0
        S = nseqs
    else:
        S = b
    out = {"x": torch.empty_like(x), "dt": torch.empty_like(dt), "B": torch.empty_like(B),
           "C": torch.empty_like(C), "dt_bias": torch.empty(H, dtype=torch.float32, device=dev),
           "A": torch.empty(H, dtype=torch.float32, device=dev),
           "D": torch.empty(H, dtype=torch.float32, device=dev),
           "init_state": torch.empty((S, H, N, P), dtype=torch.float32, device=dev)}
    dims = SsdDims(b, L, H, P, N, G, S if seq_idx is not None else 0, _DT[x.dtype])
    with torch.cuda.device(dev):
        rc = _lib.lib().ssd_chunk_scan_bwd(
            ctypes.byref(dims), _p(x), _p(dt), _p(dt_bias), _p(A), _p(B), _p(C), _p(D), _p(init_state),
            _p(seq_idx), int(chunk), _p(dy), _p(dfinal), _p(out["x"]), _p(out["dt"]), _p(out["dt_bias"]),
            _p(out["A"]), _p(out["B"]), _p(out["C"]), _p(out["D"]), _p(out["init_state"]),
            _stream(stream, dev))
    _lib.check(rc)
    return out


def state_update(state, x, dt, A, B, C, *, D=None, dt_bias=None, y=None, stream=None):
    """One decode step, in place on ``state`` (b,H,N,P) float32.  Returns y (b,H,P)."""
    _need(state, "state", torch.float32, 4)
    dev = state.device
    _need(x, "x", None, 3, dev)
    if x.dtype not in _DT:
        raise ValueError(f"x dtype {x.dtype} not supported")
    for t, n, nd in ((dt, "dt", 2), (B, "B", 3), (C, "C", 3)):
        _need(t, n, dtype=x.dtype, ndim=nd, device=dev)
    _need(A, "A", torch.float32, 1, dev)
    _need(D, "D", torch.float32, 1, dev)
    _need(dt_bias, "dt_bias", torch.float32, 1, dev)
    b, H, N, P = state.shape
    G = B.shape[1]
    if y is None:
        y = torch.empty_like(x)
    else:
        _need(y, "y", x.dtype, 3, dev)
    dims = SsdDims(b, 1, H, P, N, G, 0, _DT[x.dtype])
    with torch.cuda.device(dev):
        rc = _lib.lib().ssd_state_update(ctypes.byref(dims), _p(state), _p(x), _p(dt), _p(A), _p(B),
                                         _p(C), _p(D), _p(y), _stream(stream, dev), _p(dt_bias))
    _lib.check(rc)
    return y
