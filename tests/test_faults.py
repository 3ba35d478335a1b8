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


# --- every output element is written -------------------------------------------------------

CANARY_CASES = [
    ("tensor-core, ragged", dict(name="mamba2_2.7b_layer", batch=2, seqlen=333, nheads=4), None),
    ("tensor-core, packed", dict(name="packed_varlen", nheads=4, dstate=128), [300, 17, 129, 128, 1]),
    ("tensor-core, d_state 256, packed", dict(name="packed_varlen", nheads=4), [200, 1, 130]),
    ("CUDA cores, fp32", dict(name="tiny_fp32", seqlen=77), None),
]


@pytest.mark.parametrize("what,kw,lens", CANARY_CASES, ids=[c[0] for c in CANARY_CASES])
def test_every_output_element_is_written(what, kw, lens):
    """y and final_state start as NaN: after the call none may be left (inputs are finite)."""
    kw = dict(kw)
    w = inputs.scaled(inputs.WORKLOADS[kw.pop("name")], **kw)
    d = inputs.make_inputs(w, "cuda", lengths=lens)
    y = torch.full_like(d["x"], float("nan"))
    S = d["nseqs"]
    fs = torch.full((S, w.nheads, w.dstate, w.headdim), float("nan"), device="cuda")
    ssd.chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_bias=d["dt_bias"], D=d["D"],
                       init_state=d["init_state"], seq_idx=d["seq_idx"], nseqs=S, chunk=w.chunk, y=y,
                       final_state=fs)
    torch.cuda.synchronize()
    assert not torch.isnan(y).any(), what
    assert not torch.isnan(fs).any(), what


# --- a broken seq_idx is reported in debug mode -------------------------------------------------

_BROKEN_SEQ_IDX = r"""
import sys, torch
sys.path.insert(0, {root!r})
import state_space_model_07_b200 as ssd
from state_space_model_07_b200 import inputs
w = inputs.scaled(inputs.WORKLOADS["packed_varlen"], nheads=4, dstate=128)
d = inputs.make_inputs(w, "cuda", lengths=[100, 50, 30])
si = d["seq_idx"].clone()
si[0, 100:] += 1          # 0 -> 2 at token 100 (a step of +2), and it ends at 3 > nseqs - 1
try:
    ssd.chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_bias=d["dt_bias"], D=d["D"],
                       init_state=d["init_state"], seq_idx=si, nseqs=3, chunk=w.chunk)
    torch.cuda.synchronize()
    print("status 0")
except ssd.SsdError as e:
    print("status", e.code)
# the context is still usable: a valid call right after
y, fs = ssd.chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_bias=d["dt_bias"], D=d["D"],
                           init_state=d["init_state"], seq_idx=d["seq_idx"], nseqs=3, chunk=w.chunk)
torch.cuda.synchronize()
print("after ok", bool(torch.isfinite(y).all()))
"""


def test_broken_seq_idx_is_reported_in_debug_mode():
    """With SSD_DEBUG_CHECK=1 every call synchronises and reads the device status word: a
    seq_idx that breaks its contract comes back as SSD_ERR_SEQIDX (8), never as an
    out-of-bounds access, and the next valid call works."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SSD_DEBUG_CHECK="1")
    out = subprocess.run([sys.executable, "-c", _BROKEN_SEQ_IDX.format(root=root)], env=env,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    assert "status 8" in out.stdout, out.stdout
    assert "after ok True" in out.stdout, out.stdout


# --- the tensor-core path's fp16 operand range -----------------------------------------------

_RANGE = r"""
import sys, torch
sys.path.insert(0, {root!r})
import state_space_model_07_b200 as ssd
from state_space_model_07_b200 import inputs
w = inputs.scaled(inputs.WORKLOADS["mamba2_2.7b_layer"], batch=1, seqlen=300, nheads=4)
d = inputs.make_inputs(w, "cuda")
def run(dd):
    try:
        y, fs = ssd.chunk_scan_fwd(dd["x"], dd["dt"], dd["A"], dd["B"], dd["C"], dt_bias=dd["dt_bias"],
                                   D=dd["D"], chunk=w.chunk)
        torch.cuda.synchronize()
        return "0 finite" if bool(torch.isfinite(y).all() and torch.isfinite(fs).all()) else "0 nonfinite"
    except ssd.SsdError as e:
        return str(e.code)
over = dict(d, x=d["x"].clone())
over["x"][0, 5, 1, 3] = 1e5                      # finite in bf16, beyond fp16
big = dict(d, B=d["B"] * 1000, C=d["C"] * 1000)  # every input in range; the score matrix is not
nan = dict(d, x=d["x"].clone())
nan["x"][0, 5, 1, 3] = float("nan")
print("plain", run(d))
print("x over", run(over))
print("scores over", run(big))
print("nan input", run(nan))
"""


@pytest.mark.parametrize("debug", [True, False])
def test_fp16_operand_range_of_the_tensor_core_path(debug):
    """The tensor-core path's operands are fp16.  With SSD_DEBUG_CHECK=1 an input beyond 65504
    and a non-finite result from finite inputs (B and C 1000x larger than N(0, 1): the score
    matrix passes 65504) come back as SSD_ERR_RANGE (9); a NaN input is the caller's and is not
    a range error.  Without the debug check the same calls return non-finite values, as the
    header states."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SSD_DEBUG_CHECK="1" if debug else "0")
    out = subprocess.run([sys.executable, "-c", _RANGE.format(root=root)], env=env,
                         capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = out.stdout.splitlines()
    assert "plain 0 finite" in lines, out.stdout
    if debug:
        assert "x over 9" in lines and "scores over 9" in lines, out.stdout
        assert "nan input 0 nonfinite" in lines, out.stdout
    else:
        assert "x over 0 nonfinite" in lines and "scores over 0 nonfinite" in lines, out.stdout
        assert "nan input 0 nonfinite" in lines, out.stdout
