"""GPU parity of the scan's backward (ssd_chunk_scan_bwd) against the fp64 gradient oracle.

The oracle (oracle/ssd_oracle_bwd.c) is the adjoint reverse sweep, pinned in
tests/test_oracle_bwd.py by finite differences of the forward oracle, automatic
differentiation of a separately written forward, closed forms and planted mistakes.  Here the
CUDA kernel's gradients of J = sum(dy * y) + sum(dfinal * final_state) are compared with it
element by element on the same inputs: every gradient (x, dt, dt_bias, A, B, C, D, initial
state) within tol (1 + |ref|), tol 1e-4 for fp32 inputs and 1e-2 for bf16 inputs (whose dx,
ddt, dB, dC are rounded to bf16 once); the per-head sums over many tokens (dt_bias, A, D) are
compared relative to the largest term of their kind.
"""
import numpy as np
import pytest
import torch

import oracle
import state_space_model_07_b200 as ssd
from state_space_model_07_b200 import inputs
from tests.helpers import TOL, assert_close, head_slice, to_cpu

pytestmark = pytest.mark.gpu
W = inputs.WORKLOADS


def _upstream(d, w, seed):
    g = torch.Generator().manual_seed(seed)
    b, L, H, P = d["x"].shape
    S = d["nseqs"]
    dy = torch.randn((b, L, H, P), generator=g).to(d["x"].dtype).to(d["x"].device)
    dfinal = torch.randn((S, H, w.dstate, P), generator=g).float().to(d["x"].device)
    return dy, dfinal


def _check(d, w, chunk=None, seed=0, with_dfinal=True):
    dy, dfinal = _upstream(d, w, seed)
    if not with_dfinal:
        dfinal = None
    got = ssd.chunk_scan_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dy, dt_bias=d["dt_bias"], D=d["D"],
                             init_state=d["init_state"], seq_idx=d["seq_idx"], nseqs=d["nseqs"],
                             chunk=chunk or w.chunk, dfinal=dfinal)
    torch.cuda.synchronize()
    c = to_cpu(d)
    ref = oracle.ssd_scan_bwd(c["x"], c["dt"], c["A"], c["B"], c["C"], dy.cpu(), dt_bias=c["dt_bias"], D=c["D"],
                              init_state=c["init_state"], seq_idx=c["seq_idx"], nseqs=c["nseqs"],
                              dfinal=None if dfinal is None else dfinal.cpu())
    tol = TOL[d["x"].dtype]
    for k in ("x", "dt", "B", "C", "init_state"):
        assert_close(got[k], ref[k], tol, f"d{k}")
    for k in ("dt_bias", "A", "D"):
        r = np.asarray(ref[k])
        scale = 1.0 + np.max(np.abs(r))
        err = float(np.max(np.abs(got[k].double().cpu().numpy() - r))) / scale
        assert err <= tol, f"d{k}: max |d| / (1 + max |ref|) = {err:.3e} > {tol:.1e}"
    return got, ref


@pytest.mark.parametrize("case", [
    # (dtype, b, L, H, P, N, G, chunk)
    ("f32", 1, 70, 2, 16, 16, 1, 16),
    ("f32", 2, 200, 4, 32, 64, 2, 64),
    ("f32", 1, 300, 2, 64, 128, 1, 256),
    ("bf16", 2, 333, 4, 64, 128, 2, 256),
    ("bf16", 1, 129, 6, 32, 32, 3, 128),
    ("bf16", 1, 64, 2, 128, 64, 1, 64),
], ids=lambda c: "-".join(map(str, c)))
def test_backward_matches_the_gradient_oracle(case):
    dt, b, L, H, P, N, G, Q = case
    w = inputs.Workload("bwd", b, L, H, P, N, G, Q, dt, seed=200 + L, init_state=True)
    _check(inputs.make_inputs(w, "cuda"), w)


def test_backward_of_the_bench_shaped_layer_at_oracle_size():
    w = inputs.scaled(W["mamba2_2.7b_layer"], batch=2, seqlen=260, nheads=4)
    _check(inputs.make_inputs(w, "cuda"), w, seed=3)


@pytest.mark.parametrize("nheads,dstate", [(4, 64), (8, 128)])
def test_backward_packed_sequences_and_no_dfinal(nheads, dstate):
    """Packed sequences (chunks restart at every sequence start).  With 8 heads in 4 groups the
    bf16 gradient blocks split each group's two heads over two blocks (few blocks for 148 SMs),
    so the summed dB, dC partials are covered for packed input too."""
    w = inputs.scaled(W["packed_varlen"], nheads=nheads, dstate=dstate)
    lens = [100, 1, 64, 65, 30]
    d = inputs.make_inputs(w, "cuda", lengths=lens)
    _check(d, w, seed=5)
    _check(d, w, seed=6, with_dfinal=False)


def test_backward_empty_sequence_passes_dfinal_through():
    w = inputs.Workload("bwd0", 2, 0, 2, 16, 16, 1, 16, "f32", seed=1, init_state=True)
    d = inputs.make_inputs(w, "cuda")
    dy, dfinal = _upstream(d, w, 1)
    got = ssd.chunk_scan_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dy, dt_bias=d["dt_bias"], D=d["D"],
                             init_state=d["init_state"], chunk=16, dfinal=dfinal)
    torch.cuda.synchronize()
    assert torch.equal(got["init_state"], dfinal)
    for k in ("dt_bias", "A", "D"):
        assert torch.count_nonzero(got[k]) == 0


def test_backward_refuses_unsupported_shapes_before_launching():
    w = inputs.Workload("bwdbig", 1, 32, 2, 256, 64, 1, 16, "f32", seed=1, init_state=False)
    d = inputs.make_inputs(w, "cuda")
    dy = torch.zeros_like(d["x"])
    with pytest.raises(ssd.SsdError) as e:
        ssd.chunk_scan_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dy, chunk=16)
    assert e.value.code == 5


def test_backward_full_size_sampled_heads():
    """The bench-shaped layer at full size (b8 L4096 H80 P64 N128, one group), in the launch
    configuration the benchmark times.  Each head's recurrence is independent, so the oracle
    recomputes sampled heads whole (all rows and tokens): their dx, ddt, d init_state and the
    per-head sums dt_bias, A, D.  dB and dC sum all 80 heads and are checked as finite."""
    w = W["mamba2_2.7b_layer"]
    d = inputs.make_inputs(w, "cuda")
    dy, dfinal = _upstream(d, w, 11)
    got = ssd.chunk_scan_bwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dy, dt_bias=d["dt_bias"], D=d["D"],
                             init_state=d["init_state"], chunk=w.chunk, dfinal=dfinal)
    torch.cuda.synchronize()
    for k, v in got.items():
        assert torch.isfinite(v.float()).all(), f"d{k} has non-finite entries"
    tol = TOL[d["x"].dtype]
    sums = {k: [] for k in ("dt_bias", "A", "D")}
    heads = (0, 41, 79)
    for h in heads:
        hd = to_cpu(head_slice(d, h, w.nheads, w.ngroups))
        ref = oracle.ssd_scan_bwd(hd["x"], hd["dt"], hd["A"], hd["B"], hd["C"], dy[:, :, h:h + 1].cpu(),
                                  dt_bias=hd["dt_bias"], D=hd["D"], init_state=hd["init_state"],
                                  dfinal=dfinal[:, h:h + 1].cpu())
        assert_close(got["x"][:, :, h:h + 1], ref["x"], tol, f"dx head {h}")
        assert_close(got["dt"][:, :, h:h + 1], ref["dt"], tol, f"ddt head {h}")
        assert_close(got["init_state"][:, h:h + 1], ref["init_state"], tol, f"dinit head {h}")
        for k in sums:
            sums[k].append(float(ref[k][0]))
    # sums over 32 768 tokens, relative to the largest of their kind (as in _check)
    for k, refs in sums.items():
        scale = 1.0 + max(abs(r) for r in refs)
        err = max(abs(float(got[k][h]) - r) for h, r in zip(heads, refs)) / scale
        assert err <= tol, f"d{k}: max |d| / (1 + max |ref|) = {err:.3e} > {tol:.1e}"
