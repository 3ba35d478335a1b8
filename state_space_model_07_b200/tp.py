"""Head-sharded (tensor-parallel) mixer with a quantised all-reduce.

"5.3 Tensor Parallelism support and large-cluster training", section 4.1, partitions the Mamba-2
layer over Tp devices, each holding H / Tp heads:
  1. input projection split by columns: every device computes its own heads' x, dt and its own
     groups' B, C from the whole input u (section 3.3: B, C and dt come from u by their own linear
     maps, in parallel) -- no communication;
  2. the scan of the device's heads (the library's tcgen05 scan) -- no communication;
  3. a group norm whose groups divide among the devices (G a multiple of Tp) -- no communication;
  4. output projection split by rows: each device's partial product, summed over the devices by
     the layer's one all-reduce.
"Scaling State-Space Models on Multiple GPUs with Tensor Parallelism" (abstract) lowers the cost of
that all-reduce by quantising it.  Here it is a reduce-scatter and an all-gather on int8 codes with
one float32 scale per 64 columns (library kernels ssd_quant_chunks, ssd_dequant_sum_quant,
ssd_dequant_chunks; the exchanges by torch.distributed all-to-all and all-gather, NCCL between
GPUs): each rank moves 2 (Tp - 1) / Tp of the codes, about half the bytes of a bf16 ring all-reduce.

The projections are plain GEMMs (cuBLAS through torch.mm, bf16 in, fp32 accumulation); the scan,
the group norm and the quantisation steps are the library's kernels.  The compute steps sit behind
``TPOps`` and the exchanges behind a communicator (``TorchDistTPComm``), so that the same code runs
on gloo ranks on the CPU with other steps; ``run_local_tp`` runs Tp ranks one after another on one
device, doing their exchanges by copies.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib, ops

QBLOCK = 64
EPS = 1e-5


def _stream(dev):
    return ops._stream(None, dev)


def group_norm(x, gamma, beta, ngroups, *, eps=EPS, out=None):
    """Group norm of each row of x (rows, C): ngroups groups of consecutive channels, mean and
    biased variance in fp32, then gamma, beta (float32, (C,))."""
    ops._need(x, "x", None, 2)
    dev = x.device
    ops._need(gamma, "gamma", torch.float32, 1, dev)
    ops._need(beta, "beta", torch.float32, 1, dev)
    if x.dtype not in ops._DT:
        raise ValueError(f"x dtype {x.dtype} not supported")
    out = torch.empty_like(x) if out is None else out
    rows, C = x.shape
    with torch.cuda.device(dev):
        rc = _lib.lib().ssd_group_norm(rows, C, ngroups, ops._DT[x.dtype], ops._p(x), ops._p(gamma), ops._p(beta),
                                       ctypes.c_float(eps), ops._p(out), _stream(dev))
    _lib.check(rc)
    return out


def quant_chunks(x, ranks):
    """float32 (T, D) -> codes (ranks, T, D / ranks) int8 and scales (ranks, T, D / ranks / 64)."""
    ops._need(x, "x", torch.float32, 2)
    T, D = x.shape
    dev = x.device
    q = torch.empty((ranks, T, D // ranks), dtype=torch.int8, device=dev)
    s = torch.empty((ranks, T, D // ranks // QBLOCK), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        rc = _lib.lib().ssd_quant_chunks(T, D, ranks, ops._p(x), ops._p(q), ops._p(s), _stream(dev))
    _lib.check(rc)
    return q, s


def dequant_sum_quant(q, s):
    """Codes (ranks, T, Dc) and scales from every rank -> codes (T, Dc) and scales of their sum."""
    ops._need(q, "q", torch.int8, 3)
    ops._need(s, "scale", torch.float32, 3, q.device)
    ranks, T, Dc = q.shape
    qo = torch.empty((T, Dc), dtype=torch.int8, device=q.device)
    so = torch.empty((T, Dc // QBLOCK), dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        rc = _lib.lib().ssd_dequant_sum_quant(T, Dc, ranks, ops._p(q), ops._p(s), ops._p(qo), ops._p(so),
                                              _stream(q.device))
    _lib.check(rc)
    return qo, so


def dequant_chunks(q, s, dtype=torch.bfloat16):
    """Gathered codes (ranks, T, Dc) and scales -> (T, ranks Dc) of dtype."""
    ops._need(q, "q", torch.int8, 3)
    ops._need(s, "scale", torch.float32, 3, q.device)
    ranks, T, Dc = q.shape
    out = torch.empty((T, ranks * Dc), dtype=dtype, device=q.device)
    with torch.cuda.device(q.device):
        rc = _lib.lib().ssd_dequant_chunks(T, ranks * Dc, ranks, ops._DT[dtype], ops._p(q), ops._p(s), ops._p(out),
                                           _stream(q.device))
    _lib.check(rc)
    return out


def shard(w: dict, rank: int, ranks: int) -> dict:
    """Rank `rank`'s weights: its H / ranks heads (columns of W_x, W_dt; rows of W_out; their
    dt_bias, A, D, gamma, beta) and G / ranks groups (columns of W_B, W_C), contiguous."""
    H = w["A"].shape[0]
    P = w["W_x"].shape[1] // H
    GN = w["W_B"].shape[1]
    if H % ranks or GN % ranks:
        raise ValueError("heads and groups must divide among the ranks")
    Hr = H // ranks
    h0, h1 = rank * Hr, (rank + 1) * Hr
    g0, g1 = rank * GN // ranks, (rank + 1) * GN // ranks
    c = lambda t: t.contiguous()
    return {"W_x": c(w["W_x"][:, h0 * P:h1 * P]), "W_B": c(w["W_B"][:, g0:g1]), "W_C": c(w["W_C"][:, g0:g1]),
            "W_dt": c(w["W_dt"][:, h0:h1]), "dt_bias": c(w["dt_bias"][h0:h1]), "A": c(w["A"][h0:h1]),
            "D": c(w["D"][h0:h1]), "gamma": c(w["gamma"][h0 * P:h1 * P]), "beta": c(w["beta"][h0 * P:h1 * P]),
            "W_out": c(w["W_out"][h0 * P:h1 * P, :])}


class TPOps:
    """The compute steps of one rank: cuBLAS projections, the library's scan, group norm and
    quantisation kernels."""

    def local_output(self, u, s, *, ngroups, dstate, headdim, chunk):
        b, L, Dm = u.shape
        u2 = u.reshape(b * L, Dm)
        Hr = s["A"].shape[0]
        x = torch.mm(u2, s["W_x"]).view(b, L, Hr, headdim)
        B = torch.mm(u2, s["W_B"]).view(b, L, -1, dstate)
        C = torch.mm(u2, s["W_C"]).view(b, L, -1, dstate)
        dt = torch.mm(u2, s["W_dt"]).view(b, L, Hr)
        y, _ = ops.chunk_scan_fwd(x, dt, s["A"], B, C, dt_bias=s["dt_bias"], D=s["D"], chunk=chunk,
                                  want_final=False)
        return group_norm(y.view(b * L, Hr * headdim), s["gamma"], s["beta"], ngroups)

    def out_proj(self, n, s):
        return torch.mm(n, s["W_out"], out_dtype=torch.float32)

    quant_chunks = staticmethod(quant_chunks)
    dequant_sum_quant = staticmethod(dequant_sum_quant)

    def dequant_chunks(self, q, s, dtype):
        return dequant_chunks(q, s, dtype)


class TorchDistTPComm:
    """The exchanges over torch.distributed (NCCL between GPUs, gloo on the CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_to_all(self, q, s):
        """q (ranks, T, Dc), s (ranks, T, nb): slice j goes to rank j; returns what every rank sent
        here, stacked in rank order."""
        qr, sr = torch.empty_like(q), torch.empty_like(s)
        self.dist.all_to_all_single(qr, q.contiguous(), group=self.group)
        self.dist.all_to_all_single(sr, s.contiguous(), group=self.group)
        return qr, sr

    def all_gather(self, q, s):
        """q (T, Dc), s (T, nb) of every rank, stacked in rank order: (ranks, T, Dc), (ranks, T, nb)."""
        qa = torch.empty((self.world * q.shape[0],) + tuple(q.shape[1:]), dtype=q.dtype, device=q.device)
        sa = torch.empty((self.world * s.shape[0],) + tuple(s.shape[1:]), dtype=s.dtype, device=s.device)
        self.dist.all_gather_into_tensor(qa, q.contiguous(), group=self.group)
        self.dist.all_gather_into_tensor(sa, s.contiguous(), group=self.group)
        return qa.view((self.world,) + tuple(q.shape)), sa.view((self.world,) + tuple(s.shape))

    def all_reduce(self, x):
        self.dist.all_reduce(x, group=self.group)
        return x


class SingleRankComm:
    """The exchanges of a one-rank layer (Tp = 1): every collective is the identity."""
    rank, world = 0, 1

    def all_to_all(self, q, s):
        return q, s

    def all_gather(self, q, s):
        return q.unsqueeze(0), s.unsqueeze(0)

    def all_reduce(self, x):
        return x


def quant_allreduce(z, comm, ops_: Optional[TPOps] = None, dtype=torch.bfloat16):
    """Sum over the ranks of z (T, D) float32 through int8 codes: reduce-scatter, then all-gather."""
    o = ops_ or TPOps()
    q, s = o.quant_chunks(z, comm.world)
    qr, sr = comm.all_to_all(q, s)
    qs, ss = o.dequant_sum_quant(qr, sr)
    qa, sa = comm.all_gather(qs, ss)
    return o.dequant_chunks(qa, sa, dtype)


def mixer_fwd(u, s, comm, *, ngroups, dstate, headdim, chunk=256, quantized=True, ops_: Optional[TPOps] = None):
    """This rank's part of the layer: u (b, L, d_model) bf16, the rank's weights `s` (``shard``),
    ngroups = the layer's groups (G / Tp of them here).  Returns the layer output (b L, d_model):
    bf16 through the quantised all-reduce, or float32 through an exact one (float32 too with one
    rank, which has nothing to reduce)."""
    o = ops_ or TPOps()
    n = o.local_output(u, s, ngroups=ngroups // comm.world, dstate=dstate, headdim=headdim, chunk=chunk)
    z = o.out_proj(n, s)
    if comm.world == 1:
        return z          # one rank: its partial is the output, there is nothing to reduce
    return quant_allreduce(z, comm, o) if quantized else comm.all_reduce(z)


def run_local_tp(u, w, ranks, *, ngroups, dstate, headdim, chunk=256, quantized=True, ops_: Optional[TPOps] = None):
    """All ranks of a Tp-way layer on one device, one after another, with the exchanges done by
    copies (every exchange is a full barrier, so running each phase for all ranks in turn is a
    valid schedule).  Returns the layer output as every rank would hold it (rank 0's copy)."""
    o = ops_ or TPOps()
    shards = [shard(w, r, ranks) for r in range(ranks)]
    zs = [o.out_proj(o.local_output(u, sh, ngroups=ngroups // ranks, dstate=dstate, headdim=headdim, chunk=chunk), sh)
          for sh in shards]
    if not quantized:
        return torch.stack(zs).sum(0)
    qs = [o.quant_chunks(z, ranks) for z in zs]
    red = [o.dequant_sum_quant(torch.stack([qs[r][0][j] for r in range(ranks)]),
                               torch.stack([qs[r][1][j] for r in range(ranks)])) for j in range(ranks)]
    return o.dequant_chunks(torch.stack([q for q, _ in red]), torch.stack([s for _, s in red]), torch.bfloat16)
