"""The scan entry point that allocates nothing (ssd_chunk_scan_fwd_noalloc).

It exists for callers that cannot let the library allocate device memory (a
serving engine whose pool already owns almost all of HBM, or code that must
not allocate after start-up).  It keeps its scratch in a fixed 32 MiB device
array inside the library, so these tests check that (1) through the C ABI it
matches the fp64 oracle element by element within the parity tolerance, and
agrees with the allocating ssd_chunk_scan_fwd within the same tolerance, on two
different calls in a row (the second call must not be disturbed by what the
first left in the shared scratch), and (2) a call whose scratch would not fit
is refused before anything runs.

The file name makes pytest collect it last.
"""
import ctypes

import pytest
import torch

import state_space_model_07_b200 as ssd
from state_space_model_07_b200 import _lib, inputs
from tests.helpers import TOL, assert_close, oracle_scan, to_cpu

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def noalloc_scan(d, chunk):
    x = d["x"]
    b, L, H, P = x.shape
    G, N = d["B"].shape[2], d["B"].shape[3]
    S = d["nseqs"]
    y = torch.empty_like(x)
    fs = torch.empty((S, H, N, P), dtype=torch.float32, device=x.device)
    dims = _lib.SsdDims(b, L, H, P, N, G, S if d["seq_idx"] is not None else 0,
                        _lib.SSD_BF16 if x.dtype == torch.bfloat16 else _lib.SSD_F32)
    rc = _lib.lib().ssd_chunk_scan_fwd_noalloc(
        ctypes.byref(dims), _p(x), _p(d["dt"]), _p(d["dt_bias"]), _p(d["A"]), _p(d["B"]), _p(d["C"]),
        _p(d["D"]), _p(d["init_state"]), _p(d["seq_idx"]), int(chunk), _p(y), _p(fs),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return rc, y, fs


def allocating_scan(d, chunk):
    return ssd.chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_bias=d["dt_bias"], D=d["D"],
                              init_state=d["init_state"], seq_idx=d["seq_idx"], nseqs=d["nseqs"],
                              chunk=chunk)


def test_noalloc_matches_allocating_scan_on_two_calls_in_a_row():
    w1 = inputs.scaled(inputs.WORKLOADS["packed_varlen"], nheads=8, dstate=128)
    d1 = inputs.make_inputs(w1, "cuda", lengths=[300, 17, 129, 128, 600, 1])
    w2 = inputs.Workload("noalloc2", 2, 333, 4, 32, 64, 2, 64, "f32", seed=77, init_state=True)
    d2 = inputs.make_inputs(w2, "cuda")
    refs = [allocating_scan(d1, w1.chunk), allocating_scan(d2, w2.chunk)]
    outs = []
    for d, w in ((d1, w1), (d2, w2)):
        rc, y, fs = noalloc_scan(d, w.chunk)
        assert rc == 0, _lib.lib().ssd_last_error().decode()
        outs.append((y, fs))
    torch.cuda.synchronize()
    for (y, fs), (ya, fa), d in zip(outs, refs, (d1, d2)):
        tol = TOL[d["x"].dtype]
        yo, fo = oracle_scan(to_cpu(d))
        assert_close(y, yo, tol, "no-alloc y vs oracle")
        assert_close(fs, fo, tol, "no-alloc final_state vs oracle")
        assert_close(y, ya.double().cpu().numpy(), tol, "no-alloc y vs allocating scan")
        assert_close(fs, fa.double().cpu().numpy(), tol, "no-alloc final_state vs allocating scan")


def test_noalloc_refuses_calls_beyond_its_scratch():
    # 512 chunks x 8 heads x 32 KiB states = 128 MiB of scratch > 32 MiB.
    w = inputs.Workload("big", 1, 65536, 8, 64, 128, 1, 128, "bf16", seed=3, init_state=False)
    d = inputs.make_inputs(w, "cuda")
    rc, _, _ = noalloc_scan(d, w.chunk)
    assert rc == 5  # SSD_ERR_UNSUPPORTED
    assert "32 MiB" in _lib.lib().ssd_last_error().decode()
