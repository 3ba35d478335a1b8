"""Sequence parallelism across ranks, checked at the algorithm level on CPU.

"5.3 Tensor Parallelism support and large-cluster training", section 4.2, splits a long
sequence across GPUs and hands the N x P state from one GPU to the next by point-to-point
send / receive.  Here world-size 2 and 3 gloo ranks each own a contiguous slice of the tokens
and exchange real tensors:
  1. every rank scans its slice (rank 0 from the real initial state, the others from zero),
     giving its local final state F_r, and sums its slice's log-decay D_r;
  2. a ring: rank r >= 1 receives the state entering its slice from rank r - 1, and every rank
     but the last sends h_out = exp(D_r) h_in + F_r (rank 0: h_out = F_0) to rank r + 1;
  3. every rank r >= 1 adds to its y the output of h_in entering its slice (here the oracle scan
     of a zero input from h_in, which by linearity is that term), and the last rank's h_out is
     the sequence's final state.
The ranks run the library's own ring code (state_space_model_07_b200.seqpar: its send / receive
order over torch.distributed and its use of the scan, decay and chain steps) with those steps
supplied in fp64 on the CPU (the scan by the oracle), so the stitched y and final state must
equal one oracle scan of the whole sequence to rounding.  The GPU kernels of the steps are
checked in tests/test_seqpar_gpu.py.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    from state_space_model_07_b200 import inputs
    w = inputs.scaled(inputs.WORKLOADS["long_context"], batch=2, seqlen=301, nheads=4, headdim=8, dstate=16,
                      ngroups=2)
    d = inputs.make_inputs(w, "cpu")
    return {k: (None if d[k] is None else d[k].double().numpy()) for k in
            ("x", "dt", "dt_bias", "A", "B", "C", "D", "init_state")}


def _softplus(z):
    return np.where(z > 0, z + np.log1p(np.exp(-np.abs(z))), np.log1p(np.exp(np.minimum(z, 0))))


def _oracle_ops():
    """The compute steps in fp64 on the CPU (the scan by the oracle), so that the library's ring
    code (chunk_scan_fwd_seqpar, TorchDistComm) runs unchanged on gloo ranks without a GPU."""
    import torch
    import oracle
    from state_space_model_07_b200.seqpar import SeqParOps

    class OracleOps(SeqParOps):
        def scan(self, x, dt, A, B, C, *, dt_bias, D, init_state, chunk, y=None):
            h0 = None if init_state is None else init_state.numpy()
            yy, F = oracle.ssd_scan(x.numpy(), dt.numpy(), A.numpy(), B.numpy(), C.numpy(), dt_bias=dt_bias.numpy(),
                                    D=D.numpy(), init_state=h0, nthreads=1)
            return torch.from_numpy(yy), torch.from_numpy(np.ascontiguousarray(F))

        def logdecay(self, dt, A, *, dt_bias):
            return torch.from_numpy(np.sum(_softplus(dt.numpy() + dt_bias.numpy()) * A.numpy(), axis=1))

        def chain(self, h_in, logdecay, F):
            return torch.exp(logdecay)[:, :, None, None] * h_in + F

        def add_state(self, x, dt, A, B, C, *, dt_bias, h_in, y):
            # the output of h_in alone: the scan of a zero input entered by h_in (D x = 0)
            yy, _ = oracle.ssd_scan(np.zeros_like(x.numpy()), dt.numpy(), A.numpy(), B.numpy(), C.numpy(),
                                    dt_bias=dt_bias.numpy(), D=None, init_state=h_in.numpy(), nthreads=1)
            y.add_(torch.from_numpy(yy))
            return True

    return OracleOps()


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    from state_space_model_07_b200.seqpar import TorchDistComm, chunk_scan_fwd_seqpar
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        a = {k: (None if v is None else torch.from_numpy(v)) for k, v in _inputs().items()}
        L = a["x"].shape[1]
        bounds = np.linspace(0, L, world + 1).astype(int)
        sl = slice(bounds[rank], bounds[rank + 1])
        part = {k: a[k][:, sl].contiguous() for k in ("x", "dt", "B", "C")}
        y, F = chunk_scan_fwd_seqpar(part["x"], part["dt"], a["A"], part["B"], part["C"], comm=TorchDistComm(),
                                     dt_bias=a["dt_bias"], D=a["D"], init_state=a["init_state"], chunk=64,
                                     ops_=_oracle_ops())
        out[rank] = (y.numpy(), F.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_parallel_ring_reproduces_the_whole_scan(world):
    import oracle
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    a = _inputs()
    yr, fr = oracle.ssd_scan(a["x"], a["dt"], a["A"], a["B"], a["C"], dt_bias=a["dt_bias"], D=a["D"],
                             init_state=a["init_state"])
    y = np.concatenate([res[r][0] for r in range(world)], axis=1)
    assert np.max(np.abs(y - yr) / (1 + np.abs(yr))) < 1e-12
    assert np.max(np.abs(res[world - 1][1] - fr) / (1 + np.abs(fr))) < 1e-12
