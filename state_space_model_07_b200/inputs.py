"""Seeded synthetic inputs for the SSD scan and the decode state update.

This module only draws random numbers; it holds none of the method's
arithmetic.  Both the CUDA path and the fp64 oracle consume exactly the bytes
produced here (the oracle widens them to float64 without rounding).

Recipe (one ``numpy.random.default_rng(seed)`` stream per workload, draws in
float32, then rounded to bf16 round-to-nearest-even by torch for bf16 fields):
  x, B, C        ~ N(0, 1)
  dt (raw)       ~ N(0, 1); the method applies softplus(dt + dt_bias)
  dt_bias        = -2 for every head (tiny fp32 workload), else
                   ~ U(ln 1e-3, ln 1e-1) per head (float32)
  A_h            = -exp(U(0, ln 16))  -> A in [-16, -1] (float32)
  D_h            ~ N(0, 1) (float32)
  init_state     zero, or ~ N(0, 0.1^2) (float32) where the workload has one
  packed lengths rng.integers(512, 8193, nseqs) (upper bound exclusive)

The workloads are the shapes of Mamba / Mamba-2 LLM layers named in the
pages' setting; no dataset is involved.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int
    chunk: int
    dtype: str            # "f32" or "bf16"
    seed: int
    init_state: bool      # random initial state ~ N(0, 0.1^2)
    dt_bias_const: Optional[float] = None   # fixed bias for every head, else U(ln1e-3, ln1e-1)
    packed_nseqs: int = 0                    # >0: one packed row of that many sequences
    decode_steps: int = 0                    # decode steps following the prefill

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


WORKLOADS = {
    "tiny_fp32": Workload("tiny_fp32", 1, 64, 2, 16, 16, 1, 16, "f32", 0, False, dt_bias_const=-2.0),
    "mamba2_2.7b_layer": Workload("mamba2_2.7b_layer", 8, 4096, 80, 64, 128, 1, 256, "bf16", 1, False),
    "long_context": Workload("long_context", 1, 131072, 64, 64, 128, 8, 256, "bf16", 2, True),
    "prefill_decode": Workload("prefill_decode", 64, 2048, 64, 64, 128, 1, 256, "bf16", 3, False,
                               decode_steps=256),
    "packed_varlen": Workload("packed_varlen", 1, 0, 128, 64, 256, 4, 128, "bf16", 4, True,
                              packed_nseqs=16),
}


def scaled(w: Workload, **over) -> Workload:
    """Same distributions, other sizes (used for oracle-sized parity cases)."""
    return dataclasses.replace(w, **over)


def packed_lengths(rng: np.random.Generator, nseqs: int, lo: int = 512, hi: int = 8192) -> np.ndarray:
    return rng.integers(lo, hi + 1, nseqs)


def _bf16_or_f32(a: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(dtype) if dtype != torch.float32 else t


def make_inputs(w: Workload, device="cpu", lengths=None):
    """Returns a dict of tensors for one scan call (and, if the workload has
    decode steps, per-step decode inputs are made by ``make_decode_inputs``).

    Keys: x (b,L,H,P), dt (b,L,H), dt_bias (H) f32, A (H) f32, B, C (b,L,G,N),
    D (H) f32, init_state (S,H,N,P) f32 or None, seq_idx (1,L) int32 or None,
    nseqs, lengths (packed only), chunk.
    """
    rng = np.random.default_rng(w.seed)
    dt_ = w.torch_dtype
    H, P, N, G = w.nheads, w.headdim, w.dstate, w.ngroups
    seq_idx = None
    if w.packed_nseqs:
        if lengths is None:
            lengths = packed_lengths(rng, w.packed_nseqs)
        lengths = np.asarray(lengths, dtype=np.int64)
        b, L = 1, int(lengths.sum())
        seq_idx = np.repeat(np.arange(len(lengths), dtype=np.int32), lengths).reshape(1, L)
        S = len(lengths)
    else:
        b, L = w.batch, w.seqlen
        S = b
    x = rng.standard_normal((b, L, H, P), dtype=np.float32)
    dt = rng.standard_normal((b, L, H), dtype=np.float32)
    B = rng.standard_normal((b, L, G, N), dtype=np.float32)
    C = rng.standard_normal((b, L, G, N), dtype=np.float32)
    if w.dt_bias_const is not None:
        dt_bias = np.full((H,), w.dt_bias_const, dtype=np.float32)
    else:
        dt_bias = rng.uniform(math.log(1e-3), math.log(1e-1), H).astype(np.float32)
    A = (-np.exp(rng.uniform(0.0, math.log(16.0), H))).astype(np.float32)
    D = rng.standard_normal(H, dtype=np.float32)
    init = None
    if w.init_state:
        init = (0.1 * rng.standard_normal((S, H, N, P), dtype=np.float32)).astype(np.float32)
    out = {
        "x": _bf16_or_f32(x, dt_).to(device),
        "dt": _bf16_or_f32(dt, dt_).to(device),
        "dt_bias": torch.from_numpy(dt_bias).to(device),
        "A": torch.from_numpy(A).to(device),
        "B": _bf16_or_f32(B, dt_).to(device),
        "C": _bf16_or_f32(C, dt_).to(device),
        "D": torch.from_numpy(D).to(device),
        "init_state": None if init is None else torch.from_numpy(init).to(device),
        "seq_idx": None if seq_idx is None else torch.from_numpy(seq_idx).to(device),
        "nseqs": S,
        "lengths": None if lengths is None else np.asarray(lengths),
        "chunk": w.chunk,
    }
    return out


def make_decode_inputs(w: Workload, step: int, batch: int, device="cpu"):
    """Fresh per-step decode inputs (x (b,H,P), dt (b,H), B, C (b,G,N)) from
    the workload's distributions; the stream for step k is seeded by
    (seed, 1000 + k) so any step can be regenerated on its own."""
    rng = np.random.default_rng([w.seed, 1000 + step])
    dt_ = w.torch_dtype
    H, P, N, G = w.nheads, w.headdim, w.dstate, w.ngroups
    x = rng.standard_normal((batch, H, P), dtype=np.float32)
    dt = rng.standard_normal((batch, H), dtype=np.float32)
    B = rng.standard_normal((batch, G, N), dtype=np.float32)
    C = rng.standard_normal((batch, G, N), dtype=np.float32)
    return {
        "x": _bf16_or_f32(x, dt_).to(device),
        "dt": _bf16_or_f32(dt, dt_).to(device),
        "B": _bf16_or_f32(B, dt_).to(device),
        "C": _bf16_or_f32(C, dt_).to(device),
    }


# ---- Head-sharded mixer (tensor parallelism): synthetic layer weights and input -------------
#
# Shapes of a Mamba-2-2.7B-like layer with the SSM groups raised to 8 so that they divide among
# up to 8 devices: d_model 2560, 80 heads of 64, d_state 128.  Recipe (one default_rng(seed)
# stream, float32 draws, bf16 RNE for the matrices and the input):
#   u              ~ N(0, 1)                              (b, L, d_model)
#   W_x, W_B, W_C  ~ N(0, 1 / d_model)                    (d_model, H P), (d_model, G N) x 2
#   W_dt           ~ N(0, 1 / d_model)                    (d_model, H)
#   dt_bias, A, D  as for the scan (per head, float32)
#   gamma ~ 1 + N(0, 0.1^2), beta ~ N(0, 0.1^2)           (H P) float32
#   W_out          ~ N(0, 1 / (H P))                      (H P, d_model)

@dataclasses.dataclass(frozen=True)
class MixerConfig:
    name: str
    batch: int
    seqlen: int
    d_model: int
    nheads: int
    headdim: int
    dstate: int
    ngroups: int          # SSM groups (B, C) and also the group-norm groups
    chunk: int
    seed: int


MIXERS = {
    "mixer_2.7b": MixerConfig("mixer_2.7b", 8, 4096, 2560, 80, 64, 128, 8, 256, 5),
    "mixer_small": MixerConfig("mixer_small", 2, 300, 256, 8, 64, 128, 4, 128, 6),
}


def make_mixer(cfg: MixerConfig, device="cpu"):
    """Returns (u, weights dict) for one layer; matrices and u in bf16, vectors float32."""
    rng = np.random.default_rng(cfg.seed)
    Dm, H, P, N, G = cfg.d_model, cfg.nheads, cfg.headdim, cfg.dstate, cfg.ngroups
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16).to(device)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)
    u = rng.standard_normal((cfg.batch, cfg.seqlen, Dm), dtype=np.float32)
    sd = np.float32(1.0 / math.sqrt(Dm))
    w = {
        "W_x": bf(rng.standard_normal((Dm, H * P), dtype=np.float32) * sd),
        "W_B": bf(rng.standard_normal((Dm, G * N), dtype=np.float32) * sd),
        "W_C": bf(rng.standard_normal((Dm, G * N), dtype=np.float32) * sd),
        "W_dt": bf(rng.standard_normal((Dm, H), dtype=np.float32) * sd),
        "dt_bias": f32(rng.uniform(math.log(1e-3), math.log(1e-1), H)),
        "A": f32(-np.exp(rng.uniform(0.0, math.log(16.0), H))),
        "D": f32(rng.standard_normal(H, dtype=np.float32)),
        "gamma": f32(1.0 + 0.1 * rng.standard_normal(H * P, dtype=np.float32)),
        "beta": f32(0.1 * rng.standard_normal(H * P, dtype=np.float32)),
        "W_out": bf(rng.standard_normal((H * P, Dm), dtype=np.float32) * np.float32(1.0 / math.sqrt(H * P))),
    }
    return bf(u), w
