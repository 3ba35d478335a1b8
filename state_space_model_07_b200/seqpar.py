"""Sequence parallelism: one long sequence split over ranks, the state passed along a ring.

"5.3 Tensor Parallelism support and large-cluster training", section 4.2, splits a long
sequence over devices and hands the N x P state of each device's last chunk to the next device
by point-to-point send / receive.  Rank r holds tokens [r Ls, (r + 1) Ls) of every batch row:

1. it scans its slice, rank 0 from the real initial state and the others from zero, which
   gives y (final on rank 0) and the slice's own final state F_r;
2. it forms the slice's total log-decay D_r = sum softplus(dt + dt_bias) A (a library kernel);
3. the ring: rank r >= 1 receives the state entering its slice h_in from rank r - 1, and every
   rank but the last sends h_out = exp(D_r) h_in + F_r (rank 0: h_out = F_0) to rank r + 1
   (the chain step is a library kernel too);
4. every rank r >= 1 adds to its y the part that comes from h_in (the state-to-output term
   exp(cs_t) C_t^T h_in, one library call), or, where that call does not take the inputs'
   dtype and shape, scans its slice again from h_in; the last rank's h_out is the
   sequence's final state.

Only the entering states cross between ranks (b H N P float32 per boundary).  The compute
steps go through the library (``SeqParOps``); the exchange goes through a communicator with
``send_next`` / ``recv_prev``: ``TorchDistComm`` (torch.distributed point-to-point, NCCL
between GPUs) or ``LocalRing``, which runs the ranks one after another in one process (the ring
only ever waits on the rank before, so that order is a valid schedule).
"""
from __future__ import annotations

import ctypes
from typing import Callable, Optional

import torch

from . import _lib, ops


def segment_logdecay(dt, A, *, dt_bias=None, out=None, stream=None):
    """Total log-decay of each batch row's slice: (b, H) float32."""
    ops._need(dt, "dt", None, 3)
    dev = dt.device
    if dt.dtype not in ops._DT:
        raise ValueError(f"dt dtype {dt.dtype} not supported")
    ops._need(A, "A", torch.float32, 1, dev)
    ops._need(dt_bias, "dt_bias", torch.float32, 1, dev)
    b, L, H = dt.shape
    if out is None:
        out = torch.empty((b, H), dtype=torch.float32, device=dev)
    else:
        ops._need(out, "out", torch.float32, 2, dev)
    dims = ops.SsdDims(b, L, H, 16, 16, 1, 0, ops._DT[dt.dtype])
    with torch.cuda.device(dev):
        rc = _lib.lib().ssd_segment_logdecay(ctypes.byref(dims), ops._p(dt), ops._p(dt_bias), ops._p(A),
                                             ops._p(out), ops._stream(stream, dev))
    _lib.check(rc)
    return out


def state_chain(h_in, logdecay, F, *, out=None, stream=None):
    """exp(logdecay) h_in + F per (batch, head): (b, H, N, P) float32."""
    ops._need(h_in, "h_in", torch.float32, 4)
    dev = h_in.device
    ops._need(F, "F", torch.float32, 4, dev)
    ops._need(logdecay, "logdecay", torch.float32, 2, dev)
    b, H, N, P = h_in.shape
    if out is None:
        out = torch.empty_like(h_in)
    else:
        ops._need(out, "out", torch.float32, 4, dev)
    dims = ops.SsdDims(b, 1, H, P, N, 1, 0, _lib.SSD_F32)
    with torch.cuda.device(dev):
        rc = _lib.lib().ssd_state_chain(ctypes.byref(dims), ops._p(h_in), ops._p(logdecay), ops._p(F),
                                        ops._p(out), ops._stream(stream, dev))
    _lib.check(rc)
    return out


def state_to_output(dt, A, C, h_in, y, *, dt_bias=None, stream=None):
    """Adds to y (b, L, H, P), in place, the output of the state h_in (b, H, N, P) entering each
    row at its start: y_t += exp(sum_{i <= t} softplus(dt_i + dt_bias) A) C_t^T h_in.  bf16 dt, C
    and y, P = 64, N = 128 (the library's tensor-core path).  Returns y."""
    ops._need(dt, "dt", torch.bfloat16, 3)
    dev = dt.device
    ops._need(C, "C", torch.bfloat16, 4, dev)
    ops._need(y, "y", torch.bfloat16, 4, dev)
    ops._need(h_in, "h_in", torch.float32, 4, dev)
    ops._need(A, "A", torch.float32, 1, dev)
    ops._need(dt_bias, "dt_bias", torch.float32, 1, dev)
    b, L, H, P = y.shape
    G, N = C.shape[2], C.shape[3]
    if dt.shape != (b, L, H) or C.shape[:2] != (b, L) or h_in.shape != (b, H, N, P):
        raise ValueError("shapes of dt, C, h_in and y disagree")
    dims = ops.SsdDims(b, L, H, P, N, G, 0, _lib.SSD_BF16)
    with torch.cuda.device(dev):
        rc = _lib.lib().ssd_state_to_output(ctypes.byref(dims), ops._p(dt), ops._p(dt_bias), ops._p(A),
                                            ops._p(C), ops._p(h_in), ops._p(y), ops._stream(stream, dev))
    _lib.check(rc)
    return y


def state_to_output_supported(x, B) -> bool:
    """True when state_to_output takes inputs of this dtype and shape."""
    return x.dtype == torch.bfloat16 and x.shape[-1] == 64 and B.shape[-1] == 128


class SeqParOps:
    """The compute steps of one rank: the library's kernels."""

    def scan(self, x, dt, A, B, C, *, dt_bias, D, init_state, chunk, y=None):
        return ops.chunk_scan_fwd(x, dt, A, B, C, dt_bias=dt_bias, D=D, init_state=init_state, chunk=chunk, y=y)

    def logdecay(self, dt, A, *, dt_bias):
        return segment_logdecay(dt, A, dt_bias=dt_bias)

    def chain(self, h_in, logdecay, F):
        return state_chain(h_in, logdecay, F)

    def empty_state(self, like_F):
        return torch.empty_like(like_F)

    def add_state(self, x, dt, A, B, C, *, dt_bias, h_in, y):
        """y += the output of h_in entering the slice; False when the library has no such call
        for these inputs (the ring then scans the slice again from h_in)."""
        if not state_to_output_supported(x, B):
            return False
        state_to_output(dt, A, C, h_in, y, dt_bias=dt_bias)
        return True


class TorchDistComm:
    """Ring neighbours over torch.distributed point-to-point (NCCL between GPUs, gloo on CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def send_next(self, t):
        self.dist.send(t.contiguous(), dst=self._global(self.rank + 1), group=self.group)

    def recv_prev(self, t):
        self.dist.recv(t, src=self._global(self.rank - 1), group=self.group)
        return t

    def _global(self, r):
        return r if self.group is None else self.dist.get_global_rank(self.group, r)


def chunk_scan_fwd_seqpar(x, dt, A, B, C, *, comm, dt_bias=None, D=None, init_state=None, chunk=256,
                          ops_: Optional[SeqParOps] = None):
    """This rank's part of one scan split over the ranks of `comm` along the sequence.

    x (b, Ls, H, P), dt (b, Ls, H), B, C (b, Ls, G, N) are this rank's slice of every batch row;
    init_state (b, H, N, P) is read on rank 0 only.  Returns (y of the slice, the state leaving
    the slice): on the last rank the latter is the sequence's final state."""
    o = ops_ or SeqParOps()
    rank, world = comm.rank, comm.world
    y, F = o.scan(x, dt, A, B, C, dt_bias=dt_bias, D=D, init_state=init_state if rank == 0 else None,
                  chunk=chunk)
    if world == 1:
        return y, F
    logd = o.logdecay(dt, A, dt_bias=dt_bias)
    h_in = None
    if rank > 0:
        h_in = comm.recv_prev(o.empty_state(F))
        h_out = o.chain(h_in, logd, F)
    else:
        h_out = F
    if rank < world - 1:
        comm.send_next(h_out)
    if rank > 0 and not o.add_state(x, dt, A, B, C, dt_bias=dt_bias, h_in=h_in, y=y):
        y, h_out = o.scan(x, dt, A, B, C, dt_bias=dt_bias, D=D, init_state=h_in, chunk=chunk, y=y)
    return y, h_out


class LocalRing:
    """All ranks of the ring in one process, run one after another: rank r's send is held
    until rank r + 1 receives it."""

    def __init__(self, world: int):
        self.world = world
        self.rank = 0
        self._box = {}

    def send_next(self, t):
        self._box[self.rank + 1] = t

    def recv_prev(self, t):
        t.copy_(self._box.pop(self.rank))
        return t


def run_local_ring(slices: list, fn: Callable[..., tuple], **kw):
    """Runs `fn(*slice, comm=ring, **kw)` for every rank's slice in rank order on one device;
    returns the per-rank results."""
    ring = LocalRing(len(slices))
    out = []
    for r, sl in enumerate(slices):
        ring.rank = r
        out.append(fn(*sl, comm=ring, **kw))
    return out
