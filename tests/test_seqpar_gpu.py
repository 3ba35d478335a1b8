"""Sequence-parallel state passing on the GPU: the library's two steps and the ring over ranks.

"5.3 Tensor Parallelism support and large-cluster training", section 4.2: a sequence split
over devices, the state handed from each device to the next.  Checked here:
* ssd_segment_logdecay against the fp64 sum of softplus(dt + dt_bias) A written out in numpy;
* ssd_state_chain against exp(D) h_in + F in fp64;
* ssd_state_to_output: a scan from zero plus the output of h_in equals the oracle's scan from h_in;
* chunk_scan_fwd_seqpar with 1 to 4 ranks emulated in order on one GPU (LocalRing), slices
  tile-aligned or ragged, batch 2, with an initial state: the stitched y and the last rank's
  final state equal one oracle scan of the whole sequence within 1e-2 (1 + |ref|).
"""
import numpy as np
import pytest
import torch

import state_space_model_07_b200 as ssd
from state_space_model_07_b200 import inputs, seqpar
from tests.helpers import TOL, assert_close, oracle_scan, to_cpu

pytestmark = pytest.mark.gpu


def _softplus(z):
    return np.where(z > 0, z + np.log1p(np.exp(-np.abs(z))), np.log1p(np.exp(np.minimum(z, 0))))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_segment_logdecay_matches_the_sum_of_log_decays(dtype):
    w = inputs.scaled(inputs.WORKLOADS["long_context"], batch=3, seqlen=1111, nheads=8, ngroups=2, dtype=dtype)
    d = inputs.make_inputs(w, "cuda")
    got = seqpar.segment_logdecay(d["dt"], d["A"], dt_bias=d["dt_bias"])
    torch.cuda.synchronize()
    dt = d["dt"].double().cpu().numpy()
    ref = np.sum(_softplus(dt + d["dt_bias"].double().cpu().numpy()), axis=1) * d["A"].double().cpu().numpy()
    assert_close(got, ref, 1e-5, "log-decay")


def test_state_chain_matches_its_formula():
    g = torch.Generator().manual_seed(3)
    h_in, F = (torch.randn((2, 4, 64, 16), generator=g) for _ in range(2))
    ld = -torch.rand((2, 4), generator=g) * 5
    got = seqpar.state_chain(h_in.cuda(), ld.cuda(), F.cuda())
    torch.cuda.synchronize()
    ref = np.exp(ld.double().numpy())[:, :, None, None] * h_in.double().numpy() + F.double().numpy()
    assert_close(got, ref, 1e-6, "chain")
    # in place over F
    Fg = F.cuda()
    seqpar.state_chain(h_in.cuda(), ld.cuda(), Fg, out=Fg)
    torch.cuda.synchronize()
    assert_close(Fg, ref, 1e-6, "chain in place")


@pytest.mark.parametrize("world,bounds", [(1, None), (2, None), (3, None), (4, [0, 256, 700, 1411, 2000]),
                                          (3, [0, 1, 900, 2000])])
def test_ring_over_ranks_reproduces_the_whole_scan(world, bounds):
    w = inputs.scaled(inputs.WORKLOADS["long_context"], batch=2, seqlen=2000, nheads=8, ngroups=2)
    d = inputs.make_inputs(w, "cuda")
    L = w.seqlen
    if bounds is None:
        bounds = [int(v) for v in np.linspace(0, L, world + 1)]
    slices = [tuple(d[k][:, bounds[r]:bounds[r + 1]].contiguous() for k in ("x", "dt")) + (d["A"],) +
              tuple(d[k][:, bounds[r]:bounds[r + 1]].contiguous() for k in ("B", "C"))
              for r in range(world)]
    res = seqpar.run_local_ring(slices, seqpar.chunk_scan_fwd_seqpar, dt_bias=d["dt_bias"], D=d["D"],
                                init_state=d["init_state"], chunk=w.chunk)
    torch.cuda.synchronize()
    y = torch.cat([r[0] for r in res], 1)
    yr, fr = oracle_scan(to_cpu(d))
    tol = TOL[torch.bfloat16]
    assert_close(y, yr, tol, "stitched y")
    assert_close(res[-1][1], fr, tol, "final state")


@pytest.mark.parametrize("b,L,H,G", [(2, 1000, 8, 2), (1, 129, 4, 1), (3, 300, 8, 8), (1, 5000, 16, 2)])
def test_state_to_output_adds_the_entering_state(b, L, H, G):
    """A scan from a zero state plus ssd_state_to_output(h_in) equals the scan from h_in (the
    oracle's); rows whose length is not a multiple of 128 exercise the partial last tile."""
    w = inputs.scaled(inputs.WORKLOADS["long_context"], batch=b, seqlen=L, nheads=H, ngroups=G)
    d = inputs.make_inputs(w, "cuda")
    y, _ = ssd.chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_bias=d["dt_bias"], D=d["D"],
                              chunk=w.chunk)
    out = seqpar.state_to_output(d["dt"], d["A"], d["C"], d["init_state"], y, dt_bias=d["dt_bias"])
    torch.cuda.synchronize()
    assert out is y
    yr, _ = oracle_scan(to_cpu(d))
    assert_close(y, yr, TOL[torch.bfloat16], "y")
