"""Pins for the fp64 oracle: each test ties it to something other than itself.

Sources: '5.3 Tensor Parallelism support and large-cluster training'
(recurrence, section 2.1; A_t = a_t I and Y = M X, section 3.1; block
decomposition and N x P state, section 3.2; packed sequences with reset,
section 4.3) and 'Scaling State-Space Models on Multiple GPUs with Tensor
Parallelism' (abstract: state cache across prefill and decode).
"""
import json
import math
import os
import re
import shutil
import subprocess

import numpy as np
import pytest

import oracle
from state_space_model_07_b200 import inputs
from tests import ssd_blocks_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "scalar_recurrence.json")


def rand_problem(rng, b=1, L=37, H=4, P=8, N=6, G=2, with_init=True, with_D=True):
    x = rng.standard_normal((b, L, H, P))
    dt = rng.standard_normal((b, L, H))
    A = -np.exp(rng.uniform(0, math.log(16), H))
    B = rng.standard_normal((b, L, G, N))
    C = rng.standard_normal((b, L, G, N))
    bias = rng.uniform(math.log(1e-3), math.log(1e-1), H)
    D = rng.standard_normal(H) if with_D else None
    h0 = 0.1 * rng.standard_normal((b, H, N, P)) if with_init else None
    return dict(x=x, dt=dt, A=A, B=B, C=C, dt_bias=bias, D=D, init_state=h0)


def run(p, **kw):
    return oracle.ssd_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], dt_bias=p["dt_bias"], D=p["D"],
                           init_state=p["init_state"], **kw)


# --- softplus: closed forms ------------------------------------------------------------

def test_softplus_closed_forms():
    assert oracle.softplus(0.0) == pytest.approx(math.log(2.0), rel=1e-15)
    assert oracle.softplus(math.log(math.e - 1.0)) == pytest.approx(1.0, rel=1e-15)
    assert oracle.softplus(40.0) == pytest.approx(40.0, rel=1e-15)
    assert oracle.softplus(-40.0) == pytest.approx(math.exp(-40.0), rel=1e-12)
    assert oracle.softplus(800.0) == 800.0          # no overflow
    assert oracle.softplus(-800.0) == 0.0


# --- hand-derived worked examples -------------------------------------------------------

@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_golden_worked_examples(case):
    L, N, P = case["L"], case["N"], case["P"]
    x = np.array(case["x"]).reshape(1, L, 1, P)
    B = np.array(case["B"]).reshape(1, L, 1, N)
    C = np.array(case["C"]).reshape(1, L, 1, N)
    dt = np.full((1, L, 1), math.log(math.e - 1.0))
    init = None if case["init_state"] is None else np.array(case["init_state"]).reshape(1, 1, N, P)
    y, fs = oracle.ssd_scan(x, dt, np.array([case["A"]]), B, C, dt_bias=np.array([case["dt_bias"]]),
                            D=np.array([case["D"]]), init_state=init)
    np.testing.assert_allclose(y.reshape(L, P), np.array(case["y"]), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(fs.reshape(N, P), np.array(case["final_state"]), rtol=1e-12, atol=1e-12)


# --- closed forms ----------------------------------------------------------------------

def test_single_token_closed_form():
    """L = 1: y = D x + d (C.B) x + C^T exp(dA) h0, final = exp(dA) h0 + d B x^T."""
    rng = np.random.default_rng(11)
    p = rand_problem(rng, b=2, L=1, H=3, P=5, N=7, G=1)
    y, fs = run(p)
    for b in range(2):
        for h in range(3):
            d = ref.softplus(p["dt"][b, 0, h] + p["dt_bias"][h])
            Bv, Cv, xv, h0 = p["B"][b, 0, 0], p["C"][b, 0, 0], p["x"][b, 0, h], p["init_state"][b, h]
            want_y = p["D"][h] * xv + d * np.dot(Cv, Bv) * xv + math.exp(d * p["A"][h]) * (Cv @ h0)
            want_h = math.exp(d * p["A"][h]) * h0 + d * np.outer(Bv, xv)
            np.testing.assert_allclose(y[b, 0, h], want_y, rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(fs[b, h], want_h, rtol=1e-12, atol=1e-13)


def test_no_decay_is_cumulative_sum():
    """A = 0: h_t = sum_{i<=t} d_i B_i x_i^T, a plain cumulative sum."""
    rng = np.random.default_rng(12)
    p = rand_problem(rng, b=1, L=50, H=2, P=3, N=4, G=1, with_init=False)
    p["A"] = np.zeros(2)
    y, fs = run(p)
    for h in range(2):
        d = ref.softplus(p["dt"][0, :, h] + p["dt_bias"][h])
        outer = d[:, None, None] * p["B"][0, :, 0, :, None] * p["x"][0, :, h, None, :]  # (L, N, P)
        hs = np.cumsum(outer, axis=0)
        want = np.einsum("tn,tnp->tp", p["C"][0, :, 0], hs) + p["D"][h] * p["x"][0, :, h]
        np.testing.assert_allclose(y[0, :, h], want, rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(fs[0, h], hs[-1], rtol=1e-11, atol=1e-11)


def test_constant_input_geometric_series():
    """N = P = 1, constant d, B = C = x = 1: h_t = d (1 - r^t) / (1 - r), r = exp(dA)."""
    L = 200
    x = np.ones((1, L, 1, 1)); B = np.ones((1, L, 1, 1)); C = np.ones((1, L, 1, 1))
    dt = np.full((1, L, 1), 0.3)
    A = np.array([-0.7])
    y, fs = oracle.ssd_scan(x, dt, A, B, C)
    d = math.log1p(math.exp(0.3))
    r = math.exp(d * A[0])
    t = np.arange(1, L + 1)
    want = d * (1 - r ** t) / (1 - r)
    np.testing.assert_allclose(y[0, :, 0, 0], want, rtol=1e-12)
    assert fs[0, 0, 0, 0] == pytest.approx(want[-1], rel=1e-12)


# --- other formulations of the same map -------------------------------------------------

def test_matches_bruteforce_semiseparable_matrix():
    rng = np.random.default_rng(13)
    p = rand_problem(rng, b=2, L=48, H=4, P=5, N=6, G=2)
    y, fs = run(p)
    y2, fs2 = ref.semiseparable_matrix_form(**p)
    np.testing.assert_allclose(y, y2, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(fs, fs2, rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("Q", [4, 16, 64])
def test_matches_block_decomposition(Q):
    rng = np.random.default_rng(14)
    p = rand_problem(rng, b=2, L=100, H=4, P=8, N=6, G=2)   # ragged last chunk for every Q
    y, fs = run(p)
    y2, fs2 = ref.block_decomposition_form(Q=Q, **p)
    np.testing.assert_allclose(y, y2, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(fs, fs2, rtol=1e-10, atol=1e-11)


# --- invariants ---------------------------------------------------------------------------

def test_state_cache_split_continuation():
    """Prefill on the first part, continue from the cached final state."""
    rng = np.random.default_rng(15)
    p = rand_problem(rng, b=2, L=90, H=2, P=4, N=5, G=1)
    y, fs = run(p)
    L1 = 33
    p1 = dict(p, x=p["x"][:, :L1], dt=p["dt"][:, :L1], B=p["B"][:, :L1], C=p["C"][:, :L1])
    ya, fa = run(p1)
    p2 = dict(p, x=p["x"][:, L1:], dt=p["dt"][:, L1:], B=p["B"][:, L1:], C=p["C"][:, L1:], init_state=fa)
    yb, fb = run(p2)
    np.testing.assert_allclose(np.concatenate([ya, yb], axis=1), y, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(fb, fs, rtol=1e-13, atol=1e-14)


def test_decode_step_equals_one_token_scan():
    rng = np.random.default_rng(16)
    b, H, P, N, G = 3, 4, 6, 5, 2
    st = rng.standard_normal((b, H, N, P))
    x = rng.standard_normal((b, H, P)); dt = rng.standard_normal((b, H))
    B = rng.standard_normal((b, G, N)); C = rng.standard_normal((b, G, N))
    A = -np.exp(rng.uniform(0, 2, H)); bias = rng.uniform(-3, -1, H); D = rng.standard_normal(H)
    st2, y = oracle.state_update(st, x, dt, A, B, C, dt_bias=bias, D=D)
    ys, fs = oracle.ssd_scan(x[:, None], dt[:, None], A, B[:, None], C[:, None], dt_bias=bias, D=D,
                             init_state=st)
    np.testing.assert_array_equal(y, ys[:, 0])
    np.testing.assert_array_equal(st2, fs)


def test_prefill_then_decode_equals_long_scan():
    rng = np.random.default_rng(17)
    p = rand_problem(rng, b=2, L=40, H=2, P=4, N=3, G=1, with_init=False)
    y, fs = run(p)
    L1 = 30
    p1 = dict(p, x=p["x"][:, :L1], dt=p["dt"][:, :L1], B=p["B"][:, :L1], C=p["C"][:, :L1])
    _, st = run(p1)
    for t in range(L1, 40):
        st, yt = oracle.state_update(st, p["x"][:, t], p["dt"][:, t], p["A"], p["B"][:, t], p["C"][:, t],
                                     dt_bias=p["dt_bias"], D=p["D"])
        np.testing.assert_allclose(yt, y[:, t], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(st, fs, rtol=1e-13, atol=1e-14)


def test_packed_equals_separate_runs():
    """Packing with a reset at every sequence start = independent runs."""
    rng = np.random.default_rng(18)
    lens = [5, 1, 17, 9, 30]
    H, P, N, G = 4, 3, 5, 2
    parts = [rand_problem(rng, b=1, L=n, H=H, P=P, N=N, G=G) for n in lens]
    same = ("A", "dt_bias", "D")
    for k in same:
        for q in parts[1:]:
            q[k] = parts[0][k]
    cat = {k: np.concatenate([q[k] for q in parts], axis=1) for k in ("x", "dt", "B", "C")}
    init = np.concatenate([q["init_state"] for q in parts], axis=0)
    seq_idx = np.repeat(np.arange(len(lens)), lens)[None]
    y, fs = oracle.ssd_scan(cat["x"], cat["dt"], parts[0]["A"], cat["B"], cat["C"],
                            dt_bias=parts[0]["dt_bias"], D=parts[0]["D"], init_state=init,
                            seq_idx=seq_idx, nseqs=len(lens))
    off = 0
    for s, q in enumerate(parts):
        ys, fss = run(q)
        np.testing.assert_array_equal(y[:, off:off + lens[s]], ys)
        np.testing.assert_array_equal(fs[s], fss[0])
        off += lens[s]


def test_groups_map_to_contiguous_head_blocks():
    """G < H: head h reads group h // (H/G); equal to G = H with B, C repeated."""
    rng = np.random.default_rng(19)
    p = rand_problem(rng, b=1, L=25, H=6, P=3, N=4, G=3)
    y, fs = run(p)
    rep = dict(p, B=np.repeat(p["B"], 2, axis=2), C=np.repeat(p["C"], 2, axis=2))
    y2, fs2 = run(rep)
    np.testing.assert_array_equal(y, y2)
    np.testing.assert_array_equal(fs, fs2)
    # head 3 alone, with group 1's B and C
    one = dict(x=p["x"][:, :, 3:4], dt=p["dt"][:, :, 3:4], A=p["A"][3:4], B=p["B"][:, :, 1:2],
               C=p["C"][:, :, 1:2], dt_bias=p["dt_bias"][3:4], D=p["D"][3:4],
               init_state=p["init_state"][:, 3:4])
    y3, _ = run(one)
    np.testing.assert_array_equal(y3[:, :, 0], y[:, :, 3])


def test_causality():
    rng = np.random.default_rng(20)
    p = rand_problem(rng, b=1, L=40, H=2, P=3, N=4, G=1)
    y, _ = run(p)
    q = dict(p, x=p["x"].copy(), B=p["B"].copy())
    q["x"][:, 25] += 3.0
    q["B"][:, 25] -= 1.0
    y2, _ = run(q)
    np.testing.assert_array_equal(y[:, :25], y2[:, :25])
    assert np.abs(y[:, 25:] - y2[:, 25:]).max() > 1e-3


def test_linearity_in_x():
    rng = np.random.default_rng(21)
    p = rand_problem(rng, b=1, L=30, H=2, P=3, N=4, G=1, with_init=False)
    x2 = rng.standard_normal(p["x"].shape)
    y1, _ = run(p)
    y2, _ = run(dict(p, x=x2))
    y3, _ = run(dict(p, x=2.0 * p["x"] - 0.5 * x2))
    np.testing.assert_allclose(y3, 2.0 * y1 - 0.5 * y2, rtol=1e-11, atol=1e-11)


def test_rejects_invalid_seq_idx():
    rng = np.random.default_rng(22)
    p = rand_problem(rng, b=1, L=6, H=2, P=2, N=2, G=1, with_init=False)
    for bad in ([0, 0, 2, 2, 3, 3], [1, 1, 1, 2, 2, 2], [0, 1, 0, 1, 1, 1]):
        with pytest.raises(ValueError):
            oracle.ssd_scan(p["x"], p["dt"], p["A"], p["B"], p["C"], seq_idx=np.array([bad]), nseqs=4)


def test_seeded_workload_inputs_are_reproducible():
    w = inputs.scaled(inputs.WORKLOADS["packed_varlen"], nheads=4, dstate=16)
    a = inputs.make_inputs(w, lengths=[3, 5])
    b = inputs.make_inputs(w, lengths=[3, 5])
    for k in ("x", "dt", "B", "C", "A", "D", "dt_bias", "init_state", "seq_idx"):
        assert (a[k] == b[k]).all()
    assert a["seq_idx"].tolist() == [[0, 0, 0, 1, 1, 1, 1, 1]]
    lens = inputs.packed_lengths(np.random.default_rng(4), 16)
    assert lens.min() >= 512 and lens.max() <= 8192


# --- planted mistakes: each one must fail at least one pin ------------------------------

MUTANTS = {
    "drop_D": ("yt[p] = Dh * xt[p];", "yt[p] = 0.0 * xt[p];"),
    "input_inside_decay": ("hn[p] = decay * hn[p] + dB * xt[p];", "hn[p] = decay * (hn[p] + dB * xt[p]);"),
    "wrong_sign_A": ("const double decay = exp(d * Ah);", "const double decay = exp(-d * Ah);"),
    "swap_B_C": ("const double *Ct = j->C + (tok * G + g) * N;", "const double *Ct = j->B + (tok * G + g) * N;"),
    "group_modulo": ("const int64_t g = h / heads_per_group;", "const int64_t g = h % G;"),
    "ignore_init": ("memcpy(state, j->init_state + (s * H + h) * N * P, sizeof(double) * N * P);",
                    "memset(state, 0, sizeof(double) * N * P);"),
    "no_softplus": ("const double d = oracle_softplus(j->dt[tok * H + h] + bias);",
                    "const double d = j->dt[tok * H + h] + bias;"),
    "dt_bias_sign": ("const double d = oracle_softplus(j->dt[tok * H + h] + bias);",
                     "const double d = oracle_softplus(j->dt[tok * H + h] - bias);"),
    "B_without_d": ("const double dB = d * Bt[n];", "const double dB = Bt[n];"),
    "A_per_group": ("const double Ah = j->A[h];", "const double Ah = j->A[g];"),
    "D_per_group": ("const double Dh = j->D ? j->D[h] : 0.0;", "const double Dh = j->D ? j->D[g] : 0.0;"),
    # y read from h_{t-1}: the output loop runs before the state update
    "output_before_update": (
        """        /* h_t = exp(d A) h_{t-1} + d B_t x_t^T */
        for (int64_t n = 0; n < N; ++n) {
            const double dB = d * Bt[n];
            double *hn = state + n * P;
            for (int64_t p = 0; p < P; ++p) hn[p] = decay * hn[p] + dB * xt[p];
        }
        /* y_t = C_t^T h_t + D x_t */
        for (int64_t p = 0; p < P; ++p) yt[p] = Dh * xt[p];
        for (int64_t n = 0; n < N; ++n) {
            const double c = Ct[n];
            const double *hn = state + n * P;
            for (int64_t p = 0; p < P; ++p) yt[p] += c * hn[p];
        }
""",
        """        for (int64_t p = 0; p < P; ++p) yt[p] = Dh * xt[p];
        for (int64_t n = 0; n < N; ++n) {
            const double c = Ct[n];
            const double *hn = state + n * P;
            for (int64_t p = 0; p < P; ++p) yt[p] += c * hn[p];
        }
        for (int64_t n = 0; n < N; ++n) {
            const double dB = d * Bt[n];
            double *hn = state + n * P;
            for (int64_t p = 0; p < P; ++p) hn[p] = decay * hn[p] + dB * xt[p];
        }
"""),
    "decode_B_without_d": ("st[n * P + p] = decay * st[n * P + p] + d * Bt[n] * xt[p];",
                           "st[n * P + p] = decay * st[n * P + p] + Bt[n] * xt[p];"),
}


def _build_mutant(tmp_path, name):
    src = open(oracle._SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    mut = tmp_path / f"m_{name}.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / f"m_{name}.so"
    subprocess.run(["gcc", "-O1", "-fPIC", "-shared", "-pthread", str(mut), "-o", str(so), "-lm"], check=True)
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, monkeypatch, name):
    """Swaps the oracle for a copy with one mistake and re-runs the pins."""
    so = _build_mutant(tmp_path, name)
    import ctypes
    lib = ctypes.CDLL(so)
    real = oracle._load()
    lib.oracle_softplus.restype = real.oracle_softplus.restype
    lib.oracle_softplus.argtypes = real.oracle_softplus.argtypes
    lib.oracle_ssd_scan.restype = ctypes.c_int
    lib.oracle_ssd_scan.argtypes = real.oracle_ssd_scan.argtypes
    lib.oracle_state_update.restype = ctypes.c_int
    lib.oracle_state_update.argtypes = real.oracle_state_update.argtypes
    monkeypatch.setattr(oracle, "_lib", lib)
    pins = [test_single_token_closed_form, test_constant_input_geometric_series,
            test_matches_bruteforce_semiseparable_matrix, test_no_decay_is_cumulative_sum,
            lambda: test_matches_block_decomposition(16), test_state_cache_split_continuation,
            test_groups_map_to_contiguous_head_blocks, test_decode_step_equals_one_token_scan]
    pins += [lambda c=c: test_golden_worked_examples(c) for c in json.load(open(GOLDEN))["cases"]]
    failures = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failures += 1
    assert failures > 0, f"mutant {name} passed every pin"
