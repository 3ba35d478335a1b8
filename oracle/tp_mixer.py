"""fp64 CPU oracle of the head-sharded (tensor-parallel) mixer (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` may import this module; it imports
nothing from the product path.

"5.3 Tensor Parallelism support and large-cluster training", section 4.1, partitions the layer
over Tp devices: the input projection by columns (each device computes its own heads' x, B, C and
dt from the whole input; section 3.3: B, C and dt come from the input by their own linear maps),
the scan over the device's heads, a group norm whose groups divide among the devices, and the
output projection by rows, so the output is the sum over devices of their partial products (the
layer's one all-reduce).  "Scaling State-Space Models on Multiple GPUs with Tensor Parallelism"
(abstract) quantises that all-reduce.  The pages fix neither the norm's exact form nor the
quantisation; the readings taken here:
  * group norm: per token, mean and biased variance over each group's channels, then per-channel
    gamma and beta (eps 1e-5); groups = the SSM groups, each the channels of H / G heads;
  * quantisation: symmetric int8 per block of 64 consecutive columns of a row, scale = amax / 127,
    code = rint(x * (127 / amax)) (round half to even), all in float32 -- the precision in which the
    codes are decided, so that they can be compared code for code;
  * the quantised all-reduce: a reduce-scatter on codes (every rank's partial quantised, the codes
    of column chunk j dequantised and summed in float32 in rank order, the sum quantised again) and
    an all-gather of those codes, dequantised;
  * in bf16 mode every tensor handed from one step to the next is bf16, as the scan's own contract
    has it (bf16 x, B, C, dt in; y out in the input's type): with ``bf16_between_steps`` the oracle
    rounds the projections, the scan's output and the norm's output to bf16 (round to nearest even)
    at those hand-offs and computes everything else in fp64.  Those roundings alone move the layer's
    output by up to ~3% of 1 + |z| on the small test layer (dt enters the decay exponentially), so
    a comparison with the unrounded layer would measure them, not the kernels.
"""
from __future__ import annotations

import numpy as np

from . import ssd_scan

QBLOCK = 64
EPS = 1e-5


def _bf16(a):
    """Round to bf16 (nearest even) and widen back to fp64."""
    import torch
    return torch.from_numpy(np.asarray(a, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def _f64(t):
    if hasattr(t, "detach"):
        t = t.detach().float().cpu().numpy()
    return np.asarray(t, dtype=np.float64)


def group_norm(x, gamma, beta, ngroups, eps=EPS):
    """x (rows, C) -> (rows, C): each row's C channels in ngroups consecutive groups, normalised by
    the group's mean and biased variance, then scaled by gamma and shifted by beta (fp64)."""
    x = _f64(x)
    rows, C = x.shape
    g = x.reshape(rows, ngroups, C // ngroups)
    mean = g.mean(axis=2, keepdims=True)
    var = ((g - mean) ** 2).mean(axis=2, keepdims=True)
    n = ((g - mean) / np.sqrt(var + eps)).reshape(rows, C)
    return n * _f64(gamma) + _f64(beta)


def shard_weights(w, rank, ranks):
    """Rank `rank`'s part of the layer's weights (fp64): its H / ranks heads and G / ranks groups --
    columns of the input projections, rows of the output projection."""
    H = _f64(w["A"]).shape[0]
    P = _f64(w["W_x"]).shape[1] // H
    GN = _f64(w["W_B"]).shape[1]
    Hr = H // ranks
    h0, h1 = rank * Hr, (rank + 1) * Hr
    g0, g1 = rank * GN // ranks, (rank + 1) * GN // ranks
    return {
        "W_x": _f64(w["W_x"])[:, h0 * P:h1 * P], "W_B": _f64(w["W_B"])[:, g0:g1], "W_C": _f64(w["W_C"])[:, g0:g1],
        "W_dt": _f64(w["W_dt"])[:, h0:h1], "dt_bias": _f64(w["dt_bias"])[h0:h1], "A": _f64(w["A"])[h0:h1],
        "D": _f64(w["D"])[h0:h1], "gamma": _f64(w["gamma"])[h0 * P:h1 * P], "beta": _f64(w["beta"])[h0 * P:h1 * P],
        "W_out": _f64(w["W_out"])[h0 * P:h1 * P, :],
    }


def local_output(u, s, ngroups, dstate, headdim, bf16_between_steps=False):
    """One rank's local work in fp64: projections, scan of its heads (zero initial state), group
    norm of its groups.  Returns (b L, heads P)."""
    r = _bf16 if bf16_between_steps else (lambda a: a)
    u = _f64(u)
    b, L, Dm = u.shape
    P, N = headdim, dstate
    Hr = s["A"].shape[0]
    x = r(u @ s["W_x"]).reshape(b, L, Hr, P)
    B = r(u @ s["W_B"]).reshape(b, L, -1, N)
    C = r(u @ s["W_C"]).reshape(b, L, -1, N)
    dt = r(u @ s["W_dt"])
    y, _ = ssd_scan(x, dt, s["A"], B, C, dt_bias=s["dt_bias"], D=s["D"], want_final=False)
    return r(group_norm(r(y).reshape(b * L, Hr * P), s["gamma"], s["beta"], ngroups))


def partial_output(u, w, rank, ranks, ngroups, dstate, headdim, bf16_between_steps=False):
    """Rank `rank`'s partial product of the output projection, (b L, d_model) fp64."""
    s = shard_weights(w, rank, ranks)
    return local_output(u, s, ngroups // ranks, dstate, headdim, bf16_between_steps) @ s["W_out"]


def mixer(u, w, ngroups, dstate, headdim, bf16_between_steps=False):
    """The whole layer on one device (fp64): (b L, d_model)."""
    return partial_output(u, w, 0, 1, ngroups, dstate, headdim, bf16_between_steps)


def quantize(x):
    """float32 (T, D) -> int8 codes (T, D) and float32 scales (T, D / 64); see the module header."""
    x = np.asarray(x, dtype=np.float32)
    T, D = x.shape
    xb = x.reshape(T, D // QBLOCK, QBLOCK)
    amax = np.max(np.abs(xb), axis=2).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, np.float32(127.0) / amax, np.float32(0.0)).astype(np.float32)
    codes = np.clip(np.rint(xb * inv[:, :, None]), -127, 127).astype(np.int8).reshape(T, D)
    return codes, (amax / np.float32(127.0)).astype(np.float32)


def dequantize(codes, scales):
    """Codes (T, D) and scales (T, D / 64) -> float32 (T, D), one rounding per value."""
    T, D = codes.shape
    c = codes.reshape(T, D // QBLOCK, QBLOCK).astype(np.float32)
    return (c * np.asarray(scales, dtype=np.float32)[:, :, None]).astype(np.float32).reshape(T, D)


def quant_allreduce(partials):
    """The quantised all-reduce of float32 partials (one (T, D) array per rank): reduce-scatter on
    codes over D / ranks column chunks, then all-gather of the re-quantised sums.  Returns float32
    (T, D)."""
    ranks = len(partials)
    T, D = partials[0].shape
    Dc = D // ranks
    q = [quantize(p) for p in partials]
    out = np.empty((T, D), dtype=np.float32)
    for j in range(ranks):
        cols = slice(j * Dc, (j + 1) * Dc)
        blocks = slice(j * Dc // QBLOCK, (j + 1) * Dc // QBLOCK)
        acc = np.zeros((T, Dc), dtype=np.float32)
        for r in range(ranks):
            acc = (acc + dequantize(q[r][0][:, cols], q[r][1][:, blocks])).astype(np.float32)
        out[:, cols] = dequantize(*quantize(acc))
    return out


def quant_allreduce_bound(partials):
    """Per-element bound on |quant_allreduce - exact sum| implied by the scheme: half a step of each
    rank's block scale plus half a step of the summed block's scale (with a little room for the
    float32 products and sums)."""
    ranks = len(partials)
    T, D = partials[0].shape
    exact = np.sum([np.asarray(p, dtype=np.float64) for p in partials], axis=0)
    step = np.zeros((T, D // QBLOCK))
    for p in partials:
        step += quantize(p)[1] / 2
    amax = np.max(np.abs(exact.reshape(T, D // QBLOCK, QBLOCK)), axis=2) + step
    step += amax / 127 / 2
    return np.repeat(step, QBLOCK, axis=1) * (1 + 1e-5) + 1e-6 * np.abs(exact)
