"""The two-pass long-sequence split of the tensor-core scan.

A sequence with few heads is cut into K segments; pass 1 scans segments 0 .. K-2 (the first from
the real initial state, the others from zero), a small kernel chains their final states across the
segments (the chunk-state passing of "5.3 Tensor Parallelism support and large-cluster training",
section 4.2, at segment granularity) and pass 2 rescans segments 1 .. K-1 from the chained states.
SSD_TC_SPLIT=K forces K segments; it is read once per process, so each case runs in a subprocess.
Results must match the fp64 oracle and the scan kernel must have run twice."""
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
w = inputs.scaled(inputs.WORKLOADS["long_context"], batch={b}, seqlen={L}, nheads=16, ngroups=2)
d = inputs.make_inputs(w, "cuda")
_lib.profile_read(reset=True)
y, fs = ssd.chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_bias=d["dt_bias"], D=d["D"],
                           init_state=d["init_state"], chunk=w.chunk)
torch.cuda.synchronize()
print("tc launches", _lib.profile_read(reset=True).get("tc_scan", (0,))[0])
yr, fr = oracle_scan(to_cpu(d))
assert_close(y, yr, 1e-2, "y"); assert_close(fs, fr, 1e-2, "final_state")
print("parity ok")
"""


@pytest.mark.parametrize("K,b,L", [(2, 1, 3000), (3, 1, 3000), (4, 2, 2100), (3, 1, 1000)])
def test_forced_split_matches_the_oracle(K, b, L):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SSD_TC_SPLIT=str(K))
    out = subprocess.run([sys.executable, "-c", _CASE.format(root=root, b=b, L=L)], env=env,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    assert "parity ok" in out.stdout
    assert "tc launches 2" in out.stdout, out.stdout
