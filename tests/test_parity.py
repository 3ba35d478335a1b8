"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Bounds (elementwise, y and final_state): |gpu - ref| <= 1e-2 (1 + |ref|) for
bf16 inputs with fp32 state/accumulation, 1e-4 (1 + |ref|) for fp32 inputs.
"""
import numpy as np
import pytest
import torch

import state_space_model_07_b200 as ssd
from state_space_model_07_b200 import inputs
from tests.helpers import TOL, assert_close, head_slice, oracle_scan, to_cpu

pytestmark = pytest.mark.gpu
W = inputs.WORKLOADS


def gpu_scan(d, chunk=None, **kw):
    return ssd.chunk_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], dt_bias=d["dt_bias"], D=d["D"],
                              init_state=d["init_state"], seq_idx=d["seq_idx"], nseqs=d["nseqs"],
                              chunk=chunk or d["chunk"], **kw)


def check(d, chunk=None, what=""):
    y, fs = gpu_scan(d, chunk)
    torch.cuda.synchronize()
    yr, fr = oracle_scan(to_cpu(d))
    tol = TOL[d["x"].dtype]
    assert_close(y, yr, tol, f"{what} y")
    assert_close(fs, fr, tol, f"{what} final_state")
    return y, fs


# --- the five workloads at oracle size (same distributions, fewer tokens/heads) -----------

SMALL = {
    "tiny_fp32": W["tiny_fp32"],
    "mamba2_layer_small": inputs.scaled(W["mamba2_2.7b_layer"], batch=2, seqlen=700, nheads=8),
    "long_context_small": inputs.scaled(W["long_context"], seqlen=3000, nheads=16, ngroups=2),
    "prefill_small": inputs.scaled(W["prefill_decode"], batch=4, seqlen=520, nheads=8),
    "packed_small": inputs.scaled(W["packed_varlen"], nheads=8),
}
PACKED_LENS = [300, 17, 129, 128, 600, 1, 255, 256]


@pytest.mark.parametrize("name", sorted(SMALL))
def test_workload_small(name):
    w = SMALL[name]
    d = inputs.make_inputs(w, "cuda", lengths=PACKED_LENS if w.packed_nseqs else None)
    check(d, what=name)


# --- shape sweep -------------------------------------------------------------------------

SWEEP = [
    # (dtype, b, L, H, P, N, G, Q)
    ("f32", 1, 100, 2, 16, 16, 1, 16),
    ("f32", 2, 300, 4, 32, 64, 2, 64),
    ("f32", 1, 513, 2, 64, 128, 1, 128),
    ("f32", 1, 260, 2, 128, 256, 2, 256),
    ("bf16", 1, 129, 4, 16, 16, 4, 16),
    ("bf16", 2, 257, 4, 32, 64, 1, 32),
    ("bf16", 1, 1000, 4, 64, 128, 2, 128),
    ("bf16", 1, 513, 2, 64, 256, 1, 256),
    ("bf16", 3, 400, 6, 128, 64, 3, 256),
    ("bf16", 1, 384, 2, 256, 128, 1, 128),
    ("bf16", 1, 300, 2, 64, 128, 1, 64),
]


@pytest.mark.parametrize("case", SWEEP, ids=lambda c: "-".join(map(str, c)))
def test_shape_sweep(case):
    dt, b, L, H, P, N, G, Q = case
    w = inputs.Workload("sweep", b, L, H, P, N, G, Q, dt, seed=100 + SWEEP.index(case), init_state=True)
    check(inputs.make_inputs(w, "cuda"), what=str(case))


# --- edge cases ----------------------------------------------------------------------------

def test_single_token_and_empty():
    w = inputs.scaled(W["mamba2_2.7b_layer"], batch=2, seqlen=1, nheads=4, init_state=True)
    check(inputs.make_inputs(w, "cuda"), what="L=1")
    d = inputs.make_inputs(inputs.scaled(w, seqlen=0), "cuda")
    y, fs = gpu_scan(d)
    torch.cuda.synchronize()
    assert y.numel() == 0
    assert torch.equal(fs, d["init_state"])


@pytest.mark.parametrize("lens", [[1], [5, 1, 1, 3], [128, 128, 1], [127, 129, 256, 2]])
def test_packed_edge_lengths(lens):
    """Sequences shorter than a chunk, of length 1, ending exactly on chunk edges."""
    w = inputs.scaled(W["packed_varlen"], nheads=4, dstate=128)
    check(inputs.make_inputs(w, "cuda", lengths=lens), what=str(lens))


def test_chunk_size_does_not_change_result():
    w = inputs.scaled(W["mamba2_2.7b_layer"], batch=1, seqlen=1000, nheads=4)
    d = inputs.make_inputs(w, "cuda")
    outs = [gpu_scan(d, q) for q in (16, 64, 128, 256)]
    torch.cuda.synchronize()
    ref = outs[-1][0].double().cpu().numpy()
    for y, _ in outs[:-1]:
        assert_close(y, ref, 2e-2, "chunk independence")


def test_in_place_continuation_aliasing():
    """init_state == final_state: prefill in two calls through one buffer."""
    w = inputs.scaled(W["prefill_decode"], batch=2, seqlen=600, nheads=4, init_state=True)
    d = inputs.make_inputs(w, "cuda")
    y_full, fs_full = gpu_scan(d)
    st = d["init_state"].clone()
    cut = 333
    parts = []
    for sl in (slice(0, cut), slice(cut, None)):
        dd = dict(d, x=d["x"][:, sl].contiguous(), dt=d["dt"][:, sl].contiguous(),
                  B=d["B"][:, sl].contiguous(), C=d["C"][:, sl].contiguous(), init_state=st)
        y, _ = gpu_scan(dd, final_state=st)
        parts.append(y)
    torch.cuda.synchronize()
    yr, fr = oracle_scan(to_cpu(d))
    assert_close(torch.cat(parts, 1), yr, 1e-2, "split y")
    assert_close(st, fr, 1e-2, "split final_state")


def test_runs_on_a_side_stream():
    w = inputs.scaled(W["mamba2_2.7b_layer"], batch=1, seqlen=300, nheads=4)
    d = inputs.make_inputs(w, "cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y, fs = gpu_scan(d)
    s.synchronize()
    yr, fr = oracle_scan(to_cpu(d))
    assert_close(y, yr, 1e-2, "side stream y")


# --- bit-exact properties ------------------------------------------------------------------

def test_causality_bitwise():
    w = inputs.scaled(W["mamba2_2.7b_layer"], batch=1, seqlen=700, nheads=4)
    d = inputs.make_inputs(w, "cuda")
    y1, _ = gpu_scan(d)
    d2 = dict(d, x=d["x"].clone(), B=d["B"].clone(), C=d["C"].clone(), dt=d["dt"].clone())
    t = 400
    d2["x"][:, t:] = torch.randn_like(d2["x"][:, t:])
    d2["B"][:, t:] *= -1
    d2["dt"][:, t:] += 1
    y2, _ = gpu_scan(d2)
    torch.cuda.synchronize()
    assert torch.equal(y1[:, :t], y2[:, :t])
    assert not torch.equal(y1[:, t:], y2[:, t:])


@pytest.mark.parametrize("poison", ["finite", "x", "B", "C", "dt"])
@pytest.mark.parametrize("dstate", [128, 256])
def test_packed_isolation_bitwise(dstate, poison):
    """Changing one sequence's inputs leaves every other sequence unchanged, bit
    for bit, even when the changed values are not finite.

    Sequence 3 starts inside the last, partial 128-token tile of sequence 2
    (lengths 300 + 17 + 129 = 446), so the tensor-core kernels load its first
    rows of x, dt, B and C as part of sequence 2's tile and must mask all of
    them; `poison` names the input that gets inf / NaN there."""
    w = inputs.scaled(W["packed_varlen"], nheads=8, dstate=dstate)
    lens = [300, 17, 129, 128, 600, 1]
    d = inputs.make_inputs(w, "cuda", lengths=lens)
    y1, f1 = gpu_scan(d)
    k = 3
    t0, t1 = sum(lens[:k]), sum(lens[:k + 1])
    d2 = dict(d, x=d["x"].clone(), B=d["B"].clone(), C=d["C"].clone(), dt=d["dt"].clone(),
              init_state=d["init_state"].clone())
    d2["x"][:, t0:t1] = torch.randn_like(d2["x"][:, t0:t1]) * 7
    d2["B"][:, t0:t1] = torch.randn_like(d2["B"][:, t0:t1])
    d2["C"][:, t0:t1] = torch.randn_like(d2["C"][:, t0:t1])
    d2["dt"][:, t0:t1] = 30.0
    d2["init_state"][k] = 5.0
    if poison == "x":
        d2["x"][:, t0:t1] = float("nan")
    elif poison == "B":
        d2["B"][:, t0:t1] = float("inf")
    elif poison == "C":
        d2["C"][:, t0:t1] = float("inf")
    elif poison == "dt":
        d2["dt"][:, t0:t1] = float("inf")
    y2, f2 = gpu_scan(d2)
    torch.cuda.synchronize()
    assert torch.equal(y1[:, :t0], y2[:, :t0]) and torch.equal(y1[:, t1:], y2[:, t1:])
    others = [s for s in range(len(lens)) if s != k]
    assert torch.equal(f1[others], f2[others])
    assert not torch.equal(f1[k], f2[k])


def test_final_state_is_taken_at_each_sequence_end():
    """final_state[s] equals the state after s's last token: continuing a
    sequence from it with one more token matches the oracle on the longer run."""
    w = inputs.scaled(W["packed_varlen"], nheads=4, dstate=64)
    lens = [129, 1, 256, 70]
    d = inputs.make_inputs(w, "cuda", lengths=lens)
    _, fs = gpu_scan(d)
    torch.cuda.synchronize()
    _, fr = oracle_scan(to_cpu(d))
    assert_close(fs, fr, 1e-2, "per-sequence final_state")


# --- decode state update --------------------------------------------------------------------

@pytest.mark.parametrize("dtype,b,H,P,N,G", [("bf16", 64, 64, 64, 128, 1), ("bf16", 8, 80, 64, 128, 1),
                                              ("f32", 3, 4, 16, 16, 2),
                                              ("bf16", 2, 8, 128, 256, 4), ("f32", 5, 6, 256, 64, 3),
                                              ("bf16", 1, 3, 48, 80, 1)])
def test_state_update_matches_oracle(dtype, b, H, P, N, G):
    import oracle
    w = inputs.Workload("dec", b, 1, H, P, N, G, 16, dtype, seed=5, init_state=True)
    d = inputs.make_inputs(w, "cuda")
    st = (0.5 * torch.randn(b, H, N, P, device="cuda")).contiguous()
    dec = inputs.make_decode_inputs(w, 0, b, "cuda")
    st_ref, y_ref = oracle.state_update(st.cpu(), dec["x"].cpu(), dec["dt"].cpu(), d["A"].cpu(),
                                        dec["B"].cpu(), dec["C"].cpu(), dt_bias=d["dt_bias"].cpu(),
                                        D=d["D"].cpu())
    y = ssd.state_update(st, dec["x"], dec["dt"], d["A"], dec["B"], dec["C"], D=d["D"], dt_bias=d["dt_bias"])
    torch.cuda.synchronize()
    tol = TOL[w.torch_dtype]
    assert_close(y, y_ref, tol, "decode y")
    assert_close(st, st_ref, tol, "decode state")


def test_prefill_then_decode_equals_longer_scan():
    """Small prefill + decode: the state cache carries the scan exactly."""
    w = inputs.scaled(W["prefill_decode"], batch=3, seqlen=300, nheads=4, decode_steps=20)
    d = inputs.make_inputs(w, "cuda")
    _, st = gpu_scan(d)
    steps = [inputs.make_decode_inputs(w, k, w.batch, "cuda") for k in range(w.decode_steps)]
    ys = [ssd.state_update(st, s["x"], s["dt"], d["A"], s["B"], s["C"], D=d["D"], dt_bias=d["dt_bias"])
          for s in steps]
    torch.cuda.synchronize()
    long = dict(d)
    for k in ("x", "dt", "B", "C"):
        long[k] = torch.cat([d[k]] + [s[k][:, None] for s in steps], 1)
    yr, fr = oracle_scan(to_cpu(long))
    assert_close(torch.stack(ys, 1), yr[:, w.seqlen:], 1e-2, "decode outputs")
    assert_close(st, fr, 1e-2, "decode final state")


@pytest.mark.parametrize("dstate", [128, 256])
def test_tensor_core_path_runs_for_bf16_p64(dstate):
    """bf16, P = 64, N = 128 or 256, chunk 128/256 calls launch the tcgen05
    kernel (and fp32 calls the CUDA-core kernels): no silent fallback between
    the two."""
    from state_space_model_07_b200 import _lib
    w = inputs.scaled(W["mamba2_2.7b_layer"], batch=1, seqlen=300, nheads=2, dstate=dstate)
    d = inputs.make_inputs(w, "cuda")
    _lib.profile_read(reset=True)
    gpu_scan(d)
    torch.cuda.synchronize()
    launched = _lib.profile_read(reset=True)
    assert launched.get("tc_scan", (0,))[0] == 1 and "simt_chunk_out" not in launched
    d32 = inputs.make_inputs(inputs.scaled(w, dtype="f32"), "cuda")
    gpu_scan(d32)
    torch.cuda.synchronize()
    launched = _lib.profile_read(reset=True)
    assert launched.get("simt_chunk_out", (0,))[0] == 1 and "tc_scan" not in launched
