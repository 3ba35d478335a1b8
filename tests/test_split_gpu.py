"""The segment split of the tensor-core scan.

Rows with few heads (and the rows of a partial last wave of CTAs) are cut into K segments; one
launch of the scan takes the whole rows and every segment (segment 0 from the row's initial
state, the others from zero), and k_state_out adds to each later segment the output of the
state entering it, chained from the segments' final states and total decays (the state passing
of "5.3 Tensor Parallelism support and large-cluster training", section 4.2, at segment
granularity).  SSD_TC_SPLIT="K" splits every row into K segments, "K,R" only the last R rows; it
is read once per process, so each case runs in a subprocess.  Results must match the fp64
oracle, with one scan launch and one state-to-output launch."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

_CASE = r"""
import sys, torch
sys.path.insert(0, {root!r})
import state_space_model_07_b200 as ssd
from state_space_model_07_b200 import inputs, _lib
from tests.helpers import oracle_scan, to_cpu, assert_close
w = inputs.scaled(inputs.WORKLOADS["long_context"], batch={b}, seqlen={L}, nheads={H}, ngroups=2)
d = inputs.make_inputs(w, "cuda")
_lib.profile_read(reset=True)
y, fs = ssd.chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_bias=d["dt_bias"], D=d["D"],
                           init_state=d["init_state"], chunk=w.chunk)
torch.cuda.synchronize()
prof = _lib.profile_read(reset=True)
print("tc launches", prof.get("tc_scan", (0,))[0], "state_out launches", prof.get("state_out", (0,))[0])
yr, fr = oracle_scan(to_cpu(d))
assert_close(y, yr, 1e-2, "y"); assert_close(fs, fr, 1e-2, "final_state")
print("parity ok")
"""


@pytest.mark.parametrize("split,b,L,H", [("2", 1, 3000, 16), ("3", 1, 3000, 16), ("4", 2, 2100, 16),
                                         ("3", 1, 1000, 16), ("3,1", 3, 2100, 8), ("4,2", 3, 1337, 8),
                                         ("2,1", 2, 4096, 80)])
def test_forced_split_matches_the_oracle(split, b, L, H):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SSD_TC_SPLIT=split)
    out = subprocess.run([sys.executable, "-c", _CASE.format(root=root, b=b, L=L, H=H)], env=env,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    assert "parity ok" in out.stdout
    assert "tc launches 1 state_out launches 1" in out.stdout, out.stdout
