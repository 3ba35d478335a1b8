"""Pins of the fp64 gradient oracle (oracle/ssd_oracle_bwd.c) against things other than itself.

The oracle is the hand-derived adjoint of the recurrence (a reverse sweep).  It is checked
against:
* central finite differences of the pinned forward oracle, along random directions and on single
  elements of every input;
* automatic differentiation (torch, float64) of a separately written forward: the materialised
  semiseparable form y = M x + (decayed initial-state term), a quadratic algorithm unlike the
  oracle's token loop;
* closed forms (the D gradient, zero upstream gradients, an empty sequence);
* packing (the packed gradient equals the per-sequence gradients);
* planted mistakes, each of which fails at least one of these pins.
"""
import subprocess

import numpy as np
import pytest
import torch

import oracle
from state_space_model_07_b200 import inputs

KEYS = ("x", "dt", "dt_bias", "A", "B", "C", "D", "init_state")


def _case(b=2, L=9, H=4, P=3, N=5, G=2, seed=11, init=True):
    w = inputs.Workload("bwd", b, L, H, P, N, G, 16, "f32", seed=seed, init_state=init)
    d = inputs.make_inputs(w, "cpu")
    args = {k: (None if d[k] is None else d[k].double().numpy()) for k in KEYS}
    rng = np.random.default_rng(seed + 1)
    dy = rng.standard_normal((b, L, H, P))
    dfinal = rng.standard_normal((b, H, N, P))
    return args, dy, dfinal


def _J(args, dy, dfinal):
    y, fs = oracle.ssd_scan(args["x"], args["dt"], args["A"], args["B"], args["C"], dt_bias=args["dt_bias"],
                            D=args["D"], init_state=args["init_state"])
    return float(np.sum(dy * y) + np.sum(dfinal * fs))


def _grads(args, dy, dfinal, **kw):
    return oracle.ssd_scan_bwd(args["x"], args["dt"], args["A"], args["B"], args["C"], dy, dt_bias=args["dt_bias"],
                               D=args["D"], init_state=args["init_state"], dfinal=dfinal, **kw)


def _fd_check(args, dy, dfinal, g, eps=1e-6, rtol=1e-6):
    rng = np.random.default_rng(3)
    for k in KEYS:
        v = rng.standard_normal(args[k].shape)
        plus = dict(args, **{k: args[k] + eps * v})
        minus = dict(args, **{k: args[k] - eps * v})
        fd = (_J(plus, dy, dfinal) - _J(minus, dy, dfinal)) / (2 * eps)
        an = float(np.sum(g[k] * v))
        assert abs(fd - an) <= rtol * (1 + abs(an)), (k, fd, an)


def test_matches_finite_differences_along_random_directions():
    args, dy, dfinal = _case()
    _fd_check(args, dy, dfinal, _grads(args, dy, dfinal))


def test_matches_finite_differences_elementwise():
    args, dy, dfinal = _case(b=1, L=6, H=2, P=2, N=3, G=1, seed=5)
    g = _grads(args, dy, dfinal)
    eps = 1e-6
    rng = np.random.default_rng(9)
    for k in KEYS:
        flat = args[k].reshape(-1)
        for idx in rng.choice(flat.size, size=min(4, flat.size), replace=False):
            e = np.zeros_like(flat)
            e[idx] = eps
            plus = dict(args, **{k: (flat + e).reshape(args[k].shape)})
            minus = dict(args, **{k: (flat - e).reshape(args[k].shape)})
            fd = (_J(plus, dy, dfinal) - _J(minus, dy, dfinal)) / (2 * eps)
            an = g[k].reshape(-1)[idx]
            assert abs(fd - an) <= 1e-6 * (1 + abs(an)), (k, idx, fd, an)


def _semiseparable_forward(x, dt, dt_bias, A, B, C, D, h0):
    """y and final state of the recurrence written as the materialised semiseparable matrix
    (quadratic in L), differentiable by torch: y_j = sum_{i<=j} (C_j . B_i) d_i
    exp(sum_{k=i+1..j} d_k A) x_i + exp(sum_{k<=j} d_k A) C_j^T h0 + D x_j."""
    b, L, H, P = x.shape
    G = B.shape[2]
    hg = torch.arange(H) // (H // G)
    Bh, Ch = B[:, :, hg, :], C[:, :, hg, :]                       # (b, L, H, N)
    d = torch.nn.functional.softplus(dt + dt_bias)                # (b, L, H)
    a = d * A                                                      # log-decay per token
    cum = torch.cumsum(a, dim=1)                                   # sum_{k<=j}
    seg = cum[:, :, None, :] - cum[:, None, :, :]                  # (b, j, i, H): sum_{k=i+1..j}
    causal = torch.tril(torch.ones(L, L, dtype=torch.bool))[None, :, :, None]
    decay = torch.where(causal, torch.exp(torch.where(causal, seg, torch.zeros_like(seg))), torch.zeros_like(seg))
    CB = torch.einsum("bjhn,bihn->bjih", Ch, Bh)
    M = CB * decay * d[:, None, :, :]                              # (b, j, i, H)
    y = torch.einsum("bjih,bihp->bjhp", M, x)
    y = y + torch.einsum("bjhn,bhnp->bjhp", Ch * torch.exp(cum)[..., None], h0) + D[None, None, :, None] * x
    tot = cum[:, -1:, :]                                           # (b, 1, H)
    w = torch.exp(tot - cum) * d                                   # weight of token i in the final state
    fs = torch.einsum("bih,bihn,bihp->bhnp", w, Bh, x) + torch.exp(tot[:, 0])[..., None, None] * h0
    return y, fs


def test_matches_autograd_of_the_semiseparable_form():
    args, dy, dfinal = _case(seed=21)
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True) for k, v in args.items()}
    y, fs = _semiseparable_forward(t["x"], t["dt"], t["dt_bias"], t["A"], t["B"], t["C"], t["D"], t["init_state"])
    # the two forwards agree: the comparison below is of gradients of one function
    yr, fr = oracle.ssd_scan(args["x"], args["dt"], args["A"], args["B"], args["C"], dt_bias=args["dt_bias"],
                             D=args["D"], init_state=args["init_state"])
    assert np.max(np.abs(y.detach().numpy() - yr)) < 1e-12 and np.max(np.abs(fs.detach().numpy() - fr)) < 1e-12
    J = (y * torch.tensor(dy)).sum() + (fs * torch.tensor(dfinal)).sum()
    J.backward()
    g = _grads(args, dy, dfinal)
    for k in KEYS:
        ref = t[k].grad.numpy()
        assert np.max(np.abs(g[k] - ref) / (1 + np.abs(ref))) < 1e-10, k


def test_closed_forms():
    args, dy, dfinal = _case(seed=31)
    g = _grads(args, dy, dfinal)
    # y_t = ... + D x_t: dJ/dD_h = sum over batch, time and p of dy * x
    assert np.allclose(g["D"], np.einsum("blhp,blhp->h", dy, args["x"]), rtol=1e-12, atol=1e-12)
    # no upstream gradient, no gradient anywhere
    z = _grads(args, np.zeros_like(dy), np.zeros_like(dfinal))
    assert all(np.all(z[k] == 0) for k in KEYS)
    # an empty sequence passes dfinal straight to the initial state
    e = oracle.ssd_scan_bwd(args["x"][:, :0], args["dt"][:, :0], args["A"], args["B"][:, :0], args["C"][:, :0],
                            dy[:, :0], dt_bias=args["dt_bias"], D=args["D"], init_state=args["init_state"],
                            dfinal=dfinal)
    assert np.array_equal(e["init_state"], dfinal)


def test_packed_equals_separate_sequences():
    w = inputs.scaled(inputs.WORKLOADS["packed_varlen"], nheads=4, ngroups=2, headdim=3, dstate=4, dtype="f32")
    lens = [5, 1, 7]
    d = inputs.make_inputs(w, "cpu", lengths=lens)
    a = {k: (None if d[k] is None else d[k].double().numpy()) for k in KEYS}
    rng = np.random.default_rng(7)
    dy = rng.standard_normal(a["x"].shape)
    dfinal = rng.standard_normal(a["init_state"].shape)
    packed = oracle.ssd_scan_bwd(a["x"], a["dt"], a["A"], a["B"], a["C"], dy, dt_bias=a["dt_bias"], D=a["D"],
                                 init_state=a["init_state"], seq_idx=d["seq_idx"], nseqs=len(lens), dfinal=dfinal)
    t0 = 0
    shared = {k: np.zeros_like(packed[k]) for k in ("dt_bias", "A", "D")}
    for s, n in enumerate(lens):
        sl = slice(t0, t0 + n)
        one = oracle.ssd_scan_bwd(a["x"][:, sl], a["dt"][:, sl], a["A"], a["B"][:, sl], a["C"][:, sl], dy[:, sl],
                                  dt_bias=a["dt_bias"], D=a["D"], init_state=a["init_state"][s:s + 1],
                                  dfinal=dfinal[s:s + 1])
        for k in ("x", "dt", "B", "C"):
            assert np.allclose(packed[k][:, sl], one[k], rtol=1e-12, atol=1e-14), (k, s)
        assert np.allclose(packed["init_state"][s], one["init_state"][0], rtol=1e-12, atol=1e-14)
        for k in shared:
            shared[k] += one[k]
        t0 += n
    for k in shared:
        assert np.allclose(packed[k], shared[k], rtol=1e-12, atol=1e-14), k


@pytest.mark.parametrize("grouped", [False, True])
@pytest.mark.parametrize("Q", [1, 4, 16, 64])
def test_chunked_backward_matches_the_oracle(Q, grouped):
    """The chunked backward (per chunk: quadratic terms, state terms, decay gradients by a reverse
    cumulative sum; reverse state passing between chunks) equals the token-by-token gradient
    oracle, with a ragged last chunk, groups, an initial state and dfinal.  `grouped` is the form
    the tensor-core gradient kernel takes: K^T C and K B once per (chunk, group) from K summed over
    the group's heads, Y from the dy h_prev^T product."""
    from tests.ssd_blocks_bwd_ref import chunked_bwd
    args, dy, dfinal = _case(b=2, L=23, H=4, P=3, N=5, G=2, seed=17)
    g = _grads(args, dy, dfinal)
    c = chunked_bwd(args["x"], args["dt"], args["A"], args["B"], args["C"], dy, dt_bias=args["dt_bias"],
                    D=args["D"], init_state=args["init_state"], dfinal=dfinal, Q=Q, grouped=grouped)
    for k in KEYS:
        assert np.max(np.abs(c[k] - g[k]) / (1 + np.abs(g[k]))) < 1e-12, (Q, k)


# --- planted mistakes ----------------------------------------------------------------------------

MUTANTS = {
    "no_sigmoid": ("const double dz = dd * sigmoid(z);", "const double dz = dd;"),
    "no_carry_decay": ("for (int64_t e = 0; e < N * P; ++e) g[e] *= a;", "for (int64_t e = 0; e < N * P; ++e) g[e] *= 1.0;"),
    "da_from_h_t": ("da += g[n * P + p] * prev[n * P + p];", "da += g[n * P + p] * cur[n * P + p];"),
    "dC_from_h_prev": ("for (int64_t p = 0; p < P; ++p) acc += cur[n * P + p] * dyt[p];",
                       "for (int64_t p = 0; p < P; ++p) acc += prev[n * P + p] * dyt[p];"),
    "dx_without_D": ("dxt[p] += Dh * dyt[p];", "dxt[p] += 0.0 * dyt[p];"),
    "dB_without_d": ("dBt[n] += d * gx;", "dBt[n] += gx;"),
    "dA_without_d": ("dA[h] += da * a * d;", "dA[h] += da * a;"),
    "group_modulo": ("const int64_t grp = h / (H / G);", "const int64_t grp = h % G;"),
    "dfinal_ignored": ("if (dfinal) memcpy(g, dfinal + (s * H + h) * N * P, sizeof(double) * N * P);",
                       "if (0) memcpy(g, dfinal + (s * H + h) * N * P, sizeof(double) * N * P);"),
}


@pytest.mark.parametrize("Q", [64, 128])
def test_grouped_chunked_backward_over_several_long_chunks(Q):
    """The grouped form at the chunk lengths a tensor-core backward takes (64 and 128 tokens), over
    several chunks with a ragged last one, equals the gradient oracle."""
    from tests.ssd_blocks_bwd_ref import chunked_bwd
    args, dy, dfinal = _case(b=1, L=300, H=4, P=3, N=5, G=2, seed=23)
    g = _grads(args, dy, dfinal)
    c = chunked_bwd(args["x"], args["dt"], args["A"], args["B"], args["C"], dy, dt_bias=args["dt_bias"],
                    D=args["D"], init_state=args["init_state"], dfinal=dfinal, Q=Q, grouped=True)
    for k in KEYS:
        assert np.max(np.abs(c[k] - g[k]) / (1 + np.abs(g[k]))) < 1e-12, (Q, k)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, monkeypatch, name):
    import ctypes
    src = open(oracle._SRC_BWD).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    mut = tmp_path / "m_bwd.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "m.so"
    subprocess.run(["gcc", "-O1", "-fPIC", "-shared", "-pthread", oracle._SRC, str(mut), "-o", str(so), "-lm"],
                   check=True)
    lib = ctypes.CDLL(str(so))
    real = oracle._load()
    for fn in ("oracle_softplus", "oracle_ssd_scan", "oracle_state_update", "oracle_ssd_scan_bwd"):
        getattr(lib, fn).restype = getattr(real, fn).restype
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
    monkeypatch.setattr(oracle, "_lib", lib)
    failures = 0
    for pin in (test_matches_finite_differences_along_random_directions,
                test_matches_autograd_of_the_semiseparable_form, test_closed_forms,
                test_packed_equals_separate_sequences):
        try:
            pin()
        except AssertionError:
            failures += 1
    assert failures > 0, f"mutant {name} passed every pin"


def test_backward_operand_precision():
    """Design input for a tensor-core backward: with the operands of every matrix product of the
    chunked backward rounded to fp16 (fp32 accumulation, 128-token chunks), every gradient stays
    within 1e-2 (1 + |ref|) of the oracle on the long-context distributions (seeded: <= 0.005);
    with bf16 operands x, B and the initial-state gradients miss it (0.03).  The grouped form (K
    summed over a group's heads before K^T C and K B, fp16 operands there too) stays within it as
    well.  The pages give no tolerance for gradients; the forward's form is used as a yardstick."""
    from tests.ssd_blocks_bwd_ref import chunked_bwd
    w = inputs.scaled(inputs.WORKLOADS["long_context"], seqlen=640, nheads=4, ngroups=2)
    d = inputs.make_inputs(w, "cpu")
    a = {k: (None if d[k] is None else d[k].double().numpy()) for k in KEYS}
    dy = torch.from_numpy(np.random.default_rng(5).standard_normal(a["x"].shape).astype(np.float32))
    dy = dy.to(torch.bfloat16).double().numpy()
    dfinal = np.zeros_like(a["init_state"])
    g = oracle.ssd_scan_bwd(a["x"], a["dt"], a["A"], a["B"], a["C"], dy, dt_bias=a["dt_bias"], D=a["D"],
                            init_state=a["init_state"], dfinal=dfinal)
    err = {}
    for ops in ("f16", "bf16"):
        c = chunked_bwd(a["x"], a["dt"], a["A"], a["B"], a["C"], dy, dt_bias=a["dt_bias"], D=a["D"],
                        init_state=a["init_state"], dfinal=dfinal, Q=128, operands=ops)
        err[ops] = {k: float(np.max(np.abs(c[k] - g[k]) / (1 + np.abs(g[k])))) for k in KEYS}
    assert max(err["f16"].values()) < 1e-2
    c = chunked_bwd(a["x"], a["dt"], a["A"], a["B"], a["C"], dy, dt_bias=a["dt_bias"], D=a["D"],
                    init_state=a["init_state"], dfinal=dfinal, Q=128, operands="f16", grouped=True)
    assert max(float(np.max(np.abs(c[k] - g[k]) / (1 + np.abs(g[k])))) for k in KEYS) < 1e-2
    assert err["bf16"]["x"] > 1e-2 and err["bf16"]["B"] > 1e-2 and err["bf16"]["init_state"] > 1e-2
