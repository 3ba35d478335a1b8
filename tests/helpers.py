"""Shared helpers for the GPU parity tests (GPU result vs the fp64 oracle)."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Accuracy bounds: |gpu - ref| <= tol * (1 + |ref|) elementwise, for y and
# final_state.  bf16 inputs with fp32 state/accumulation: 1e-2; fp32 inputs: 1e-4.
TOL = {torch.bfloat16: 1e-2, torch.float32: 1e-4}


def rel_err(got, ref):
    if isinstance(got, torch.Tensor):
        got = got.detach().double().cpu().numpy()
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if got.size == 0:
        return 0.0, None
    err = np.abs(got - ref) / (1.0 + np.abs(ref))
    i = int(np.nanargmax(err)) if not np.isnan(err).any() else int(np.argmax(np.isnan(err)))
    worst = float(err.reshape(-1)[i]) if not np.isnan(err).any() else float("nan")
    return worst, np.unravel_index(i, err.shape)


def assert_close(got, ref, tol, what=""):
    worst, where = rel_err(got, ref)
    assert worst <= tol, f"{what}: max |d|/(1+|ref|) = {worst:.3e} > {tol:.1e} at {where}"
    return worst


def oracle_scan(d, **kw):
    """Oracle on a make_inputs() dict (any device; widened exactly to fp64)."""
    return oracle.ssd_scan(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_bias=d["dt_bias"], D=d["D"],
                           init_state=d["init_state"], seq_idx=d["seq_idx"], nseqs=d["nseqs"], **kw)


def head_slice(d, h, H, G, seq=None):
    """Inputs of one head (its group's B, C) as an H = G = 1 problem.

    With ``seq`` (packed input) only that sequence's tokens are kept."""
    g = h // (H // G)
    out = {
        "x": d["x"][:, :, h:h + 1], "dt": d["dt"][:, :, h:h + 1], "B": d["B"][:, :, g:g + 1],
        "C": d["C"][:, :, g:g + 1], "A": d["A"][h:h + 1], "D": d["D"][h:h + 1],
        "dt_bias": d["dt_bias"][h:h + 1],
        "init_state": None if d["init_state"] is None else d["init_state"][:, h:h + 1],
        "seq_idx": None, "nseqs": d["nseqs"],
    }
    if seq is not None:
        lens = np.asarray(d["lengths"])
        t0 = int(lens[:seq].sum())
        t1 = t0 + int(lens[seq])
        for k in ("x", "dt", "B", "C"):
            out[k] = out[k][:, t0:t1]
        if out["init_state"] is not None:
            out["init_state"] = out["init_state"][seq:seq + 1]
        out["nseqs"] = 1
        out["span"] = (t0, t1)
    return out


def to_cpu(d):
    return {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
