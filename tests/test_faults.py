"""Failure detection on the GPU without a fault.

Every mbarrier wait in the library's kernels is bounded: when it runs out it records a timeout
in a device status word and the kernel returns, so a lost arrival can never hang the GPU.
ssd_selftest_bounded_wait runs that wait on a barrier nothing ever arrives at, with a short
limit.  These tests check that the wait gives up in about the time asked for, that the host
reports SSD_ERR_TIMEOUT, and that the CUDA context stays usable: a scan right after it still
matches the oracle.  Nothing here faults, traps or hangs.
"""
import ctypes
import time

import pytest
import torch

import state_space_model_07_b200 as ssd
from state_space_model_07_b200 import _lib, inputs
from tests.helpers import TOL, assert_close, oracle_scan, to_cpu

pytestmark = pytest.mark.gpu


def _selftest(limit):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    t0 = time.perf_counter()
    rc = _lib.lib().ssd_selftest_bounded_wait(limit, stream)
    return rc, time.perf_counter() - t0, _lib.lib().ssd_last_error().decode()


def test_bounded_wait_gives_up_and_reports_timeout():
    torch.cuda.synchronize()
    _selftest(2_000_000)                      # first call: module load, pool creation
    rc, secs, msg = _selftest(2_000_000)      # ~1 ms of SM clock
    assert rc == 7, (rc, msg)                 # SSD_ERR_TIMEOUT
    assert "gave up" in msg
    assert secs < 1.0
    rc, secs, _ = _selftest(400_000_000)      # ~0.2 s
    assert rc == 7 and 0.05 < secs < 5.0


def test_context_stays_usable_after_a_timeout():
    assert _selftest(2_000_000)[0] == 7
    w = inputs.scaled(inputs.WORKLOADS["mamba2_2.7b_layer"], batch=1, seqlen=300, nheads=4, init_state=True)
    d = inputs.make_inputs(w, "cuda")
    y, fs = ssd.chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_bias=d["dt_bias"], D=d["D"],
                               init_state=d["init_state"], chunk=w.chunk)
    torch.cuda.synchronize()
    yr, fr = oracle_scan(to_cpu(d))
    assert_close(y, yr, TOL[torch.bfloat16], "y after a timeout")
    assert_close(fs, fr, TOL[torch.bfloat16], "final_state after a timeout")
