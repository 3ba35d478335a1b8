"""Independent fp64 forms of the SSD computation, used only to pin the oracle.

Neither function shares code with ``oracle/`` (a token loop in C) nor with the
CUDA path; both are written from the pages' statements:

* ``semiseparable_matrix_form`` -- "5.3 Tensor Parallelism support and
  large-cluster training", section 3.1: with A_t = a_t I the whole scan is one
  causal (lower-triangular) semiseparable matrix M applied to X, Y = M X, where
  M[j, i] = (C_j . B_i) d_i exp(sum_{k=i+1..j} d_k A) for i <= j.  The initial
  state adds C_j exp(sum_{k<=j} d_k A) h0 and the skip adds D x_j.

* ``block_decomposition_form`` -- same page, section 3.2: cut the sequence into
  chunks of length Q; diagonal blocks are computed as the quadratic (attention
  like) form inside the chunk, off-diagonal blocks through the N x P state
  handed from one chunk to the next (low rank).
"""
from __future__ import annotations

import numpy as np


def softplus(z):
    z = np.asarray(z, dtype=np.float64)
    return np.where(z > 0, z + np.log1p(np.exp(-np.abs(z))), np.log1p(np.exp(np.minimum(z, 0))))


def _per_head(x, dt, A, B, C, dt_bias, D, init_state):
    x, dt, B, C = (np.asarray(v, dtype=np.float64) for v in (x, dt, B, C))
    A = np.asarray(A, dtype=np.float64)
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    bias = np.zeros(H) if dt_bias is None else np.asarray(dt_bias, dtype=np.float64)
    Dv = np.zeros(H) if D is None else np.asarray(D, dtype=np.float64)
    h0 = None if init_state is None else np.asarray(init_state, dtype=np.float64)
    return x, dt, A, B, C, bias, Dv, h0, (b, L, H, P, G, N)


def semiseparable_matrix_form(x, dt, A, B, C, dt_bias=None, D=None, init_state=None):
    """Materialises the L x L matrix M per (batch, head); O(L^2) memory."""
    x, dt, A, B, C, bias, Dv, h0, (b, L, H, P, G, N) = _per_head(x, dt, A, B, C, dt_bias, D, init_state)
    y = np.zeros((b, L, H, P))
    final = np.zeros((b, H, N, P))
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            d = softplus(dt[bi, :, h] + bias[h])
            logdec = np.cumsum(d * A[h])                 # sum_{k<=j} d_k A
            seg = logdec[:, None] - logdec[None, :]      # sum_{k=i+1..j} d_k A
            causal = np.tril(np.ones((L, L), dtype=bool))
            decay = np.where(causal, np.exp(np.where(causal, seg, 0.0)), 0.0)
            CB = C[bi, :, g, :] @ B[bi, :, g, :].T       # (L, L): C_j . B_i
            M = CB * decay * d[None, :]
            y[bi, :, h, :] = M @ x[bi, :, h, :] + Dv[h] * x[bi, :, h, :]
            # final state: sum_i exp(sum_{k=i+1..L-1} d_k A) d_i B_i x_i^T
            w = np.exp(logdec[-1] - logdec) * d if L else d
            final[bi, h] = (B[bi, :, g, :] * w[:, None]).T @ x[bi, :, h, :]
            if h0 is not None:
                y[bi, :, h, :] += np.exp(logdec)[:, None] * (C[bi, :, g, :] @ h0[bi, h])
                if L:
                    final[bi, h] += np.exp(logdec[-1]) * h0[bi, h]
                else:
                    final[bi, h] += h0[bi, h]
    return y, final


def block_decomposition_form(x, dt, A, B, C, Q, dt_bias=None, D=None, init_state=None):
    """Chunked form: quadratic inside each chunk, N x P state between chunks."""
    x, dt, A, B, C, bias, Dv, h0, (b, L, H, P, G, N) = _per_head(x, dt, A, B, C, dt_bias, D, init_state)
    y = np.zeros((b, L, H, P))
    final = np.zeros((b, H, N, P))
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            d_all = softplus(dt[bi, :, h] + bias[h])
            state = np.zeros((N, P)) if h0 is None else h0[bi, h].copy()
            for c0 in range(0, L, Q):
                c1 = min(c0 + Q, L)
                d = d_all[c0:c1]
                cs = np.cumsum(d * A[h])                  # chunk-local cumulative log decay
                Xc, Bc, Cc = x[bi, c0:c1, h, :], B[bi, c0:c1, g, :], C[bi, c0:c1, g, :]
                q = c1 - c0
                tri = np.tril(np.ones((q, q), dtype=bool))
                Lmat = np.where(tri, np.exp(np.where(tri, cs[:, None] - cs[None, :], 0.0)), 0.0)
                # diagonal block: (C B^T o L) diag(d) X
                y_diag = ((Cc @ Bc.T) * Lmat * d[None, :]) @ Xc
                # off-diagonal blocks through the carried state
                y_off = np.exp(cs)[:, None] * (Cc @ state)
                y[bi, c0:c1, h, :] = y_diag + y_off + Dv[h] * Xc
                # chunk state and hand-over to the next chunk
                w = d * np.exp(cs[-1] - cs)
                state = np.exp(cs[-1]) * state + (Bc * w[:, None]).T @ Xc
            final[bi, h] = state
    return y, final
