"""The gradient of the scan in chunked (block-decomposed) form, in numpy fp64.

This is the backward counterpart of ``tests/ssd_blocks_ref.py``.  The forward is the block
decomposition of "5.3 Tensor Parallelism support and large-cluster training", section 3.2.
Inside a chunk, with a_i = d_i A (natural log-decay), chunk-local cs_j = sum_{k<=j} a_k,
e_j = exp(cs_j), E = exp(cs_last) and u_i = exp(cs_last - cs_i) d_i:
    y_j   = sum_{i<=j} (C_j . B_i) exp(cs_j - cs_i) d_i x_i + e_j C_j^T h_prev + D x_j
    h_end = E h_prev + sum_i u_i B_i x_i^T
The gradient of J = sum <dy, y> + <dfinal, final_state> is derived from it by the chain rule,
one chunk at a time from the last:
  * reverse state passing: dh_prev = E dh_end + sum_j e_j C_j dy_j^T, with dh_end of the last
    chunk = dfinal and dh_end of chunk c = dh_prev of chunk c + 1;
  * x, B, C from the masked quadratic form and the two state terms;
  * the decays: J depends on cs through every exponential above; dJ/dcs_k is gathered term by
    term, dJ/da_m = sum_{k>=m} dJ/dcs_k (a reverse cumulative sum inside the chunk), and
    dJ/dd_m = (direct terms) + A dJ/da_m, dA += d_m dJ/da_m, dz = dJ/dd sigmoid(z).
This is the algorithm a chunked backward kernel evaluates (per chunk: quadratic terms on the
tensor core, the state terms as GEMMs against h_prev and dh_end, the reverse scan over chunks);
``tests/test_oracle_bwd.py`` checks it against the token-by-token gradient oracle.
"""
from __future__ import annotations

import numpy as np


def _softplus(z):
    return np.where(z > 0, z + np.log1p(np.exp(-np.abs(z))), np.log1p(np.exp(np.minimum(z, 0))))


def _sigmoid(z):
    return np.where(z >= 0, 1.0 / (1.0 + np.exp(-np.abs(z))), np.exp(-np.abs(z)) / (1.0 + np.exp(-np.abs(z))))


def chunked_bwd(x, dt, A, B, C, dy, dt_bias=None, D=None, init_state=None, dfinal=None, Q=16, operands=None,
                grouped=False):
    """x, dy (b,L,H,P); dt (b,L,H); B, C (b,L,G,N); A, dt_bias, D (H,); init_state, dfinal
    (b,H,N,P) or None.  Returns the same dict of gradients as the oracle.

    `grouped` takes two terms the way the tensor-core gradient kernel does: K^T C of dB and K B of
    dC once per (chunk, group) from K summed over the group's heads (C and B are the group's), and
    Y_j = C_j^T h_prev dy_j as sum_n C_jn (dy h_prev^T)_jn, the product dC's state term uses.

    `operands` ("f16" or "bf16") rounds both operands of every matrix product (the work a
    tensor-core kernel would do) to that type, with products and sums kept in fp32; the
    decay arithmetic stays in fp64.  None: everything fp64."""
    if operands is None:
        rd = lambda a: a
        mm = lambda a, b: a @ b
    else:
        import torch
        dt_ = {"f16": torch.float16, "bf16": torch.bfloat16}[operands]
        rd = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dt_).double().numpy()
        f32 = lambda a: np.asarray(a, dtype=np.float32).astype(np.float64)
        mm = lambda a, b: f32(rd(a) @ rd(b))
    x, dt, B, C, dy = (np.asarray(v, dtype=np.float64) for v in (x, dt, B, C, dy))
    A = np.asarray(A, dtype=np.float64)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    bias = np.zeros(H) if dt_bias is None else np.asarray(dt_bias, dtype=np.float64)
    Dv = np.zeros(H) if D is None else np.asarray(D, dtype=np.float64)
    h0 = np.zeros((b, H, N, P)) if init_state is None else np.asarray(init_state, dtype=np.float64)
    dfin = np.zeros((b, H, N, P)) if dfinal is None else np.asarray(dfinal, dtype=np.float64)
    out = {"x": np.zeros_like(x), "dt": np.zeros((b, L, H)), "dt_bias": np.zeros(H), "A": np.zeros(H),
           "B": np.zeros_like(B), "C": np.zeros_like(C), "D": np.zeros(H), "init_state": np.zeros((b, H, N, P))}
    starts = list(range(0, L, Q))
    ksum = {}   # grouped: (batch row, chunk, group) -> K summed over the group's heads
    for bb in range(b):
        for h in range(H):
            g = h // (H // G)
            z = dt[bb, :, h] + bias[h]
            d = _softplus(z)
            # forward over chunks: the state entering each chunk
            h_prev = [h0[bb, h].copy()]
            for t0 in starts:
                t1 = min(t0 + Q, L)
                cs = np.cumsum(d[t0:t1] * A[h])
                u = np.exp(cs[-1] - cs) * d[t0:t1]
                h_prev.append(np.exp(cs[-1]) * h_prev[-1] + mm((B[bb, t0:t1, g] * u[:, None]).T, x[bb, t0:t1, h]))
            # backward over chunks, last first
            dh_end = dfin[bb, h].copy()
            for c in reversed(range(len(starts))):
                t0 = starts[c]
                t1 = min(t0 + Q, L)
                dc, xc, Bc, Cc, dyc = d[t0:t1], x[bb, t0:t1, h], B[bb, t0:t1, g], C[bb, t0:t1, g], dy[bb, t0:t1, h]
                hp = h_prev[c]
                cs = np.cumsum(dc * A[h])
                e = np.exp(cs)
                E = np.exp(cs[-1])
                u = np.exp(cs[-1] - cs) * dc
                q = t1 - t0
                mask = np.tril(np.ones((q, q), dtype=bool))
                Lm = np.where(mask, np.exp(np.where(mask, cs[:, None] - cs[None, :], 0.0)), 0.0)  # [j, i]
                CB = mm(Cc, Bc.T)                                # [j, i]
                W = CB * Lm * dc[None, :]
                dyx = mm(dyc, xc.T)                              # [j, i] = dy_j . x_i
                # x, B, C, D
                dx = Dv[h] * dyc + mm(W.T, dyc) + u[:, None] * mm(Bc, dh_end)
                K = Lm * dyx * dc[None, :]                       # [j, i]
                dyhp = mm(dyc, hp.T)                             # [j, n] = dy_j . h_prev[n]
                if grouped:
                    ksum[(bb, c, g)] = ksum.get((bb, c, g), 0.0) + K
                    dB = u[:, None] * mm(xc, dh_end.T)
                    dC = e[:, None] * dyhp
                else:
                    dB = mm(K.T, Cc) + u[:, None] * mm(xc, dh_end.T)
                    dC = mm(K, Bc) + e[:, None] * dyhp
                out["x"][bb, t0:t1, h] += dx
                out["B"][bb, t0:t1, g] += dB
                out["C"][bb, t0:t1, g] += dC
                out["D"][h] += np.sum(dyc * xc)
                # decays: direct d_i terms and dJ/dcs_k
                R = CB * dyx * Lm                                # [j, i] = (C_j.B_i)(dy_j.x_i) exp(cs_j - cs_i)
                Z = np.einsum("in,np,ip->i", Bc, dh_end, xc)     # B_i^T dh_end x_i
                if grouped:
                    Yoff = np.sum(Cc * dyhp, axis=1)             # C_j^T h_prev dy_j
                else:
                    Yoff = np.einsum("jn,np,jp->j", Cc, hp, dyc)
                ddir = R.sum(axis=0) + np.exp(cs[-1] - cs) * Z
                Rd = R * dc[None, :]
                dcs = Rd.sum(axis=1) - Rd.sum(axis=0) + e * Yoff
                dcs[-1] += E * np.sum(dh_end * hp) + np.sum(u * Z)
                dcs -= u * Z
                da = np.cumsum(dcs[::-1])[::-1]                  # dJ/da_m = sum_{k>=m} dJ/dcs_k
                dd = ddir + A[h] * da
                out["A"][h] += np.sum(dc * da)
                dz = dd * _sigmoid(z[t0:t1])
                out["dt"][bb, t0:t1, h] += dz
                out["dt_bias"][h] += np.sum(dz)
                # reverse state passing
                dh_end = E * dh_end + mm((Cc * e[:, None]).T, dyc)
            out["init_state"][bb, h] = dh_end
    for (bb, c, g), Ks in ksum.items():
        t0 = starts[c]
        t1 = min(t0 + Q, L)
        out["B"][bb, t0:t1, g] += mm(Ks.T, C[bb, t0:t1, g])
        out["C"][bb, t0:t1, g] += mm(Ks, B[bb, t0:t1, g])
    return out
