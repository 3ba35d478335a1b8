"""Sequence parallelism across ranks, checked at the algorithm level on CPU.

"5.3 Tensor Parallelism support and large-cluster training", section 4.2, splits a long
sequence across GPUs and hands the N x P state from one GPU to the next by point-to-point
send / receive.  Here world-size 2 and 3 gloo ranks each own a contiguous slice of the tokens
and exchange real tensors:
  1. every rank scans its slice (rank 0 from the real initial state, the others from zero),
     giving its local final state F_r, and sums its slice's log-decay D_r;
  2. a ring: rank r >= 1 receives the state entering its slice from rank r - 1, and every rank
     but the last sends h_out = exp(D_r) h_in + F_r (rank 0: h_out = F_0) to rank r + 1;
  3. every rank r >= 1 rescans its slice from h_in (the rerun form pinned in
     tests/test_tile_model.py), and the last rank's final state is the sequence's.
The stitched y and final state equal one oracle scan of the whole sequence.  The per-slice scans
are the fp64 oracle: this checks the distributed algorithm and its message order, not GPU code.
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


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        a = _inputs()
        L = a["x"].shape[1]
        bounds = np.linspace(0, L, world + 1).astype(int)
        sl = slice(bounds[rank], bounds[rank + 1])
        part = {k: a[k][:, sl] for k in ("x", "dt", "B", "C")}
        scan = lambda h0: oracle.ssd_scan(part["x"], part["dt"], a["A"], part["B"], part["C"],
                                          dt_bias=a["dt_bias"], D=a["D"], init_state=h0, nthreads=1)
        # 1. local scan (rank 0 from the real initial state) and the slice's log-decay
        y, F = scan(a["init_state"] if rank == 0 else None)
        D = np.sum(_softplus(part["dt"] + a["dt_bias"]) * a["A"], axis=1)          # (b, H)
        # 2. the ring of entering states
        h_in = None
        if rank > 0:
            buf = torch.empty(F.shape, dtype=torch.float64)
            dist.recv(buf, src=rank - 1)
            h_in = buf.numpy()
        if rank < world - 1:
            h_out = F if rank == 0 else np.exp(D)[:, :, None, None] * h_in + F
            dist.send(torch.from_numpy(np.ascontiguousarray(h_out)), dst=rank + 1)
        # 3. rescan from the entering state
        if rank > 0:
            y, F = scan(h_in)
        out[rank] = (y, F)
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
