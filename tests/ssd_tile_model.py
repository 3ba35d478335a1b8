"""A numpy model of the tile algebra the tensor-core scan kernel evaluates.

Written from "5.3 Tensor Parallelism support and large-cluster training",
section 3.2 (block decomposition) and the recurrence of section 2.1, with the
kernel's own choices spelled out so that they can be checked against the fp64
oracle on the CPU:

* 128-token tiles; decays as base-2 exponents, cs_j = sum_{k <= j in tile} d_k A log2(e);
* the causal mask S[j, i] = (C_j . B_i) 2^(cs_j - cs_i) d_i (i <= j) split per
  16-token column block b: blocks left of the row's 32-row lane quarter use the
  rank-1 form 2^(cs_j - cs_m) * (2^(cs_m - cs_i) d_i) with pivot m = the block's
  last token; the two blocks of the row's own quarter use the direct form;
  D rides on the diagonal of S;
* w_i = d_i 2^(cs_last - cs_i); the tile's own state term s = B^T (w o x);
* y = S x + C' h_prev with C' = rows of C scaled by 2^cs_j;
* h <- 2^cs_last h + s, carried in fp32 between tiles.

``rounding`` chooses what the kernel rounds: None keeps everything in fp64
(the form must then equal the oracle up to fp64 rounding); "kernel" rounds the
tensor-core operands the way the kernel does (fp16 S, x, w o x, h_prev, B, C,
C'; fp32 accumulation and state; bf16 y); "bf16_operands" rounds S, w o x and
h_prev to bf16 instead, the alternative the kernel rejects.
"""
from __future__ import annotations

import numpy as np
import torch

LOG2E = 1.4426950408889634
T = 128


def _round(a, kind):
    if kind is None:
        return a
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    dt = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[kind]
    return t.to(dt).to(torch.float64).numpy()


_FP8 = {"e4m3": (torch.float8_e4m3fn, 448.0), "e5m2": (torch.float8_e5m2, 57344.0)}


# Microscaled fp8 (the OCP MX formats that the sm_100 block-scaled MMAs take): one power-of-two
# scale per 32 consecutive elements along the contracted dimension, 2^(floor(log2 amax) - emax)
# with emax the element format's largest exponent (8 for e4m3, 15 for e5m2); elements that land
# above the format's largest value saturate to it.
_MX = {"mxe4m3": ("e4m3", 8), "mxe5m2": ("e5m2", 15)}


def _round_mx(a, kind, axis):
    fmt, emax = _MX[kind]
    dt, top = _FP8[fmt]
    m = np.moveaxis(np.asarray(a, dtype=np.float64), axis, -1)
    k = m.shape[-1]
    pad = (-k) % 32
    if pad:
        m = np.concatenate([m, np.zeros(m.shape[:-1] + (pad,))], axis=-1)
    blk = m.reshape(m.shape[:-1] + (-1, 32))
    amax = np.max(np.abs(blk), axis=-1, keepdims=True)
    e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - emax, 0.0)
    scale = np.exp2(e)
    q = np.clip(blk / scale, -top, top)
    t = torch.from_numpy(np.ascontiguousarray(q, dtype=np.float32)).to(dt).to(torch.float64).numpy()
    out = (t * scale).reshape(m.shape)[..., :k]
    return np.moveaxis(out, -1, axis)


def _round_op(a, kind, axis):
    """Rounds one GEMM operand.  fp8 kinds carry one scale per slice along `axis` (the
    contracted dimension: a row of A, a column of B), as a scaled fp8 MMA would: the scales
    multiply back in its epilogue.  mx kinds carry one power-of-two scale per 32 elements of
    that slice (block scaling)."""
    if kind in _MX:
        return _round_mx(a, kind, axis)
    if kind not in _FP8:
        return _round(a, kind)
    dt, top = _FP8[kind]
    amax = np.max(np.abs(a), axis=axis, keepdims=True)
    scale = np.where(amax > 0, top / np.where(amax > 0, amax, 1.0), 1.0)
    t = torch.from_numpy(np.ascontiguousarray(a * scale, dtype=np.float32))
    return t.to(dt).to(torch.float64).numpy() / scale


def _softplus(z):
    return np.where(z > 0, z + np.log1p(np.exp(-np.abs(z))), np.log1p(np.exp(np.minimum(z, 0))))


def _mask(CB, cs, d, Dh, q):
    """S for one tile, block by block as the kernel forms it (exact identities)."""
    S = np.zeros_like(CB)
    for j in range(T):
        quarter = j // 32
        for b in range(8):
            cols = np.arange(16 * b, 16 * b + 16)
            if b < 2 * quarter:                              # left of the row's quarter: rank-1
                m = 16 * b + 15
                rf = np.exp2(cs[j] - cs[m])
                colfac = np.exp2(cs[m] - cs[cols]) * d[cols]
                S[j, cols] = CB[j, cols] * (colfac * rf)
            elif b <= 2 * quarter + 1:                       # the row's own quarter: direct
                f = np.exp2(cs[j] - cs[cols]) * d[cols]
                S[j, cols] = np.where(cols <= j, CB[j, cols] * f, 0.0)
        S[j, j] += Dh
    return S


def tile_form(x, dt, A, B, C, dt_bias=None, D=None, init_state=None, rounding=None, operands=None, stats=None):
    """x (b,L,H,P), dt (b,L,H), B/C (b,L,G,N), A/dt_bias/D (H,), init_state (b,H,N,P).

    `operands` (with rounding="kernel") overrides the operand type of single GEMMs: keys "cb"
    (C B^T), "state" (B^T (w o x)), "out" (C' h_prev), "diag" (S x); values "f16", "bf16",
    "e4m3", "e5m2" (fp8 with one scale per row of A and per column of B), "mxe4m3", "mxe5m2" (fp8
    with one power-of-two scale per 32 elements along the contracted dimension).

    `stats` (a dict) collects the largest magnitude of each thread-made tensor-core operand
    ("S", "h_prev", "wx", "Cp"), to check their fp16 range.

    Returns (y, final_state) as fp64 arrays."""
    ops = dict(operands or {})
    x, dt, B, C = (np.asarray(v, dtype=np.float64) for v in (x, dt, B, C))
    A = np.asarray(A, dtype=np.float64)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    bias = np.zeros(H) if dt_bias is None else np.asarray(dt_bias, dtype=np.float64)
    Dv = np.zeros(H) if D is None else np.asarray(D, dtype=np.float64)
    k16 = "f16" if rounding == "kernel" else ("bf16" if rounding == "bf16_operands" else None)
    kop = "f16" if rounding in ("kernel", "bf16_operands") else None   # x, B, C, C' always fp16 in the kernel
    k32 = "f32" if rounding else None
    y = np.zeros((b, L, H, P))
    fs = np.zeros((b, H, N, P))
    for bb in range(b):
        for h in range(H):
            g = h // (H // G)
            hst = np.zeros((N, P)) if init_state is None else np.asarray(init_state, np.float64)[bb, h].copy()
            for t0 in range(0, L, T):
                q = min(T, L - t0)
                d = np.zeros(T)
                d[:q] = _softplus(dt[bb, t0:t0 + q, h] + bias[h])
                d = _round(d, k32)
                cs = np.cumsum(d * A[h] * LOG2E)
                cs = _round(cs, k32)
                xt = np.zeros((T, P))
                xt[:q] = x[bb, t0:t0 + q, h]
                Bt = np.zeros((T, N))
                Bt[:q] = B[bb, t0:t0 + q, g]
                Ct = np.zeros((T, N))
                Ct[:q] = C[bb, t0:t0 + q, g]
                Braw, Craw, xraw = Bt, Ct, xt
                Bt, Ct, x16 = _round(Bt, kop), _round(Ct, kop), _round(xt, kop)
                if "cb" in ops:
                    CB = _round(_round_op(Craw, ops["cb"], 1) @ _round_op(Braw, ops["cb"], 1).T, k32)
                else:
                    CB = _round(Ct @ Bt.T, k32)
                S = _mask(CB, cs, d, Dv[h], q)
                w = d * np.exp2(cs[q - 1] - cs)
                if stats is not None:
                    for k, v in (("S", S), ("h_prev", hst), ("wx", w[:, None] * xraw),
                                 ("Cp", np.exp2(cs)[:, None] * Craw)):
                        stats[k] = max(stats.get(k, 0.0), float(np.max(np.abs(v))))
                if "state" in ops:
                    s_tile = _round(_round_op(Braw, ops["state"], 0).T @ _round_op(w[:, None] * xraw, ops["state"], 0), k32)
                else:
                    s_tile = _round(Bt.T @ _round(w[:, None] * x16, k16), k32)
                if "out" in ops:
                    Yo = _round_op(np.exp2(cs)[:, None] * Craw, ops["out"], 1) @ _round_op(hst, ops["out"], 0)
                else:
                    Yo = _round(np.exp2(cs)[:, None] * Ct, kop) @ _round(hst, k16)
                if "diag" in ops:
                    Yd = _round_op(S, ops["diag"], 1) @ _round_op(xraw, ops["diag"], 0)
                else:
                    Yd = _round(S, k16) @ x16
                Y = Yd + Yo
                yt = _round(Y, "bf16") if rounding else Y
                y[bb, t0:t0 + q, h] = yt[:q]
                hst = _round(np.exp2(cs[q - 1]) * hst + s_tile, k32)
            fs[bb, h] = hst
    return y, fs


def segment_split_form(x, dt, A, B, C, dt_bias=None, D=None, init_state=None, segments=2):
    """The sequence-split scheme for long sequences with few heads, in fp64.

    Pass 1 runs every segment independently from a zero state (segment 0 from the
    real initial state), giving y and each segment's final state; pass 2 chains
    the segment states, h_in(k) = 2^(total decay of segment k-1) h_in(k-1) +
    final(k-1); pass 3 adds 2^(cs_j) C_j h_in(k) to y of every segment k >= 1,
    with cs_j the cumulative decay from the segment's start to token j."""
    x, dt, B, C = (np.asarray(v, dtype=np.float64) for v in (x, dt, B, C))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    bias = np.zeros(H) if dt_bias is None else np.asarray(dt_bias, dtype=np.float64)
    bounds = np.linspace(0, L, segments + 1).astype(int)
    y = np.zeros((b, L, H, P))
    h_in = np.zeros((b, H, N, P)) if init_state is None else np.asarray(init_state, np.float64).copy()
    for k in range(segments):
        s0, s1 = bounds[k], bounds[k + 1]
        h0 = h_in if k == 0 else None
        yk, fk = tile_form(x[:, s0:s1], dt[:, s0:s1], A, B[:, s0:s1], C[:, s0:s1], dt_bias, D, h0)  # pass 1
        if k > 0:                                                                                     # pass 3
            for bb in range(b):
                for h in range(H):
                    g = h // (H // G)
                    d = _softplus(dt[bb, s0:s1, h] + bias[h])
                    cs = np.cumsum(d * np.asarray(A, np.float64)[h] * LOG2E)
                    yk[bb, :, h] += (np.exp2(cs)[:, None] * C[bb, s0:s1, g]) @ h_in[bb, h]
        y[:, s0:s1] = yk
        # pass 2: the state entering segment k + 1
        for bb in range(b):
            for h in range(H):
                d = _softplus(dt[bb, s0:s1, h] + bias[h])
                total = np.exp2(np.sum(d * np.asarray(A, np.float64)[h] * LOG2E))
                h_in[bb, h] = fk[bb, h] + (0.0 if k == 0 else total * h_in[bb, h])
    return y, h_in


def segment_rerun_form(x, dt, A, B, C, dt_bias=None, D=None, init_state=None, segments=3, seg_len=None):
    """The long-sequence split that reruns the scan instead of correcting y, in fp64.

    Segments of `seg_len` tokens (default ceil(L / segments)); the last one takes the rest.
    Pass 1 scans segments 0 .. K-2 independently: segment 0 from the real initial state (its y
    is final), the others from zero (only their final states are used).  The chain gives the
    state entering segment k >= 1: h_in(1) = final(0), h_in(k) = exp(sum of d A over segment
    k - 1) h_in(k - 1) + final(k - 1).  Pass 2 rescans segments 1 .. K-1 from h_in(k), giving
    their y and, from the last one, the final state."""
    x, dt, B, C = (np.asarray(v, dtype=np.float64) for v in (x, dt, B, C))
    A = np.asarray(A, dtype=np.float64)
    b, L, H, P = x.shape
    N = B.shape[3]
    bias = np.zeros(H) if dt_bias is None else np.asarray(dt_bias, dtype=np.float64)
    Ls = seg_len or -(-L // segments)
    bounds = [min(k * Ls, L) for k in range(segments)] + [L]
    assert all(bounds[k] < bounds[k + 1] for k in range(segments)), "every segment needs tokens"
    seg = lambda v, k: v[:, bounds[k]:bounds[k + 1]]
    y = np.zeros((b, L, H, P))
    finals = []
    for k in range(segments - 1):                                                      # pass 1
        h0 = init_state if k == 0 else None
        yk, fk = tile_form(seg(x, k), seg(dt, k), A, seg(B, k), seg(C, k), dt_bias, D, h0)
        if k == 0:
            y[:, bounds[0]:bounds[1]] = yk
        finals.append(fk)
    h_in = [None, finals[0]]                                                           # chain
    for k in range(2, segments):
        total = np.exp(np.sum(_softplus(seg(dt, k - 1) + bias) * A, axis=1))           # (b, H)
        h_in.append(total[:, :, None, None] * h_in[k - 1] + finals[k - 1])
    fs = None
    for k in range(1, segments):                                                       # pass 2
        yk, fs = tile_form(seg(x, k), seg(dt, k), A, seg(B, k), seg(C, k), dt_bias, D, h_in[k])
        y[:, bounds[k]:bounds[k + 1]] = yk
    return y, fs
