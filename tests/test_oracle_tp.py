"""Pins of the head-sharded mixer's oracle (oracle/tp_mixer.py), on the CPU.

"5.3 Tensor Parallelism support and large-cluster training", section 4.1: the layer split over Tp
devices by heads must equal the layer on one device, because the input projection is split by
columns (each device's heads and groups only), the scan and the group norm are local to heads and
groups, and the output projection is split by rows (the output is the sum of the partials).  The
quantised all-reduce ("Scaling State-Space Models on Multiple GPUs with Tensor Parallelism",
abstract) is pinned by hand-worked codes and by the error bound its scheme implies.
"""
import os

import numpy as np
import pytest
import torch

from oracle import tp_mixer as tpm
from state_space_model_07_b200 import inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def _small(**over):
    cfg = inputs.MIXERS["mixer_small"]
    return inputs.make_mixer(inputs.dataclasses.replace(cfg, **over) if over else cfg, "cpu"), cfg


def test_group_norm_is_torchs_group_norm():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((7, 48)) * 3 + 1
    g, b = rng.standard_normal(48), rng.standard_normal(48)
    ref = torch.nn.functional.group_norm(torch.from_numpy(x), 4, torch.from_numpy(g), torch.from_numpy(b), eps=1e-5)
    assert np.allclose(tpm.group_norm(x, g, b, 4), ref.numpy(), rtol=0, atol=1e-12)


def test_group_norm_statistics():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 60)) * 2 + 3
    n = tpm.group_norm(x, np.ones(60), np.zeros(60), 3, eps=0.25).reshape(5, 3, 20)
    assert np.allclose(n.mean(axis=2), 0, atol=1e-12)
    var = x.reshape(5, 3, 20).var(axis=2)
    assert np.allclose((n ** 2).mean(axis=2), var / (var + 0.25), atol=1e-12)


def test_group_norm_unbiased_variance_is_caught():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((3, 32))
    g = x.reshape(3, 2, 16)
    wrong = ((g - g.mean(2, keepdims=True)) / np.sqrt(g.var(2, ddof=1, keepdims=True) + 1e-5)).reshape(3, 32)
    ref = torch.nn.functional.group_norm(torch.from_numpy(x), 2, eps=1e-5).numpy()
    assert not np.allclose(wrong, ref, atol=1e-6)
    assert np.allclose(tpm.group_norm(x, np.ones(32), np.zeros(32), 2), ref, atol=1e-12)


def _golden():
    rows, scales = [], {}
    for line in open(os.path.join(HERE, "golden", "quant_block.txt")):
        line = line.split("#")[0].split()
        if not line:
            continue
        if line[0] == "scale":
            scales[int(line[1])] = float(line[2])
        else:
            rows.append((int(line[0]), int(line[1]), float(line[2]), int(line[3])))
    return rows, scales


def test_quantize_matches_the_hand_worked_codes():
    rows, scales = _golden()
    x = np.zeros((1, 3 * 64), dtype=np.float32)
    for blk, col, v, _ in rows:
        x[0, blk * 64 + col] = v
    codes, sc = tpm.quantize(x)
    for blk, col, _, want in rows:
        assert codes[0, blk * 64 + col] == want, (blk, col)
    for blk, want in scales.items():
        assert abs(sc[0, blk] - want) <= 1e-8
    assert codes[0, 64 + 1:128].tolist() == [0] * 63


def test_quantize_error_is_within_half_a_step():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((16, 256)) * np.exp(rng.uniform(-8, 8, (16, 1)))).astype(np.float32)
    codes, sc = tpm.quantize(x)
    err = np.abs(tpm.dequantize(codes, sc).astype(np.float64) - x)
    step = np.repeat(sc.astype(np.float64), 64, axis=1)
    assert np.all(err <= step * 0.5 * (1 + 1e-5) + 1e-30)
    assert np.abs(codes).max() == 127


def test_floor_instead_of_rint_is_caught():
    rows, _ = _golden()
    x = np.zeros((1, 64), dtype=np.float32)
    for blk, col, v, _ in rows:
        if blk == 0:
            x[0, col] = v
    floored = np.floor(x).astype(np.int64)
    want = np.array([r[3] for r in rows if r[0] == 0])
    cols = [r[1] for r in rows if r[0] == 0]
    assert np.any(floored[0, cols] != want)
    assert np.all(tpm.quantize(x)[0][0, cols] == want)


@pytest.mark.parametrize("ranks", [1, 2, 4])
def test_quant_allreduce_is_within_its_bound(ranks):
    rng = np.random.default_rng(10 + ranks)
    parts = [(rng.standard_normal((9, 512)) * rng.uniform(0.1, 10)).astype(np.float32) for _ in range(ranks)]
    got = tpm.quant_allreduce(parts).astype(np.float64)
    exact = np.sum([p.astype(np.float64) for p in parts], axis=0)
    bound = tpm.quant_allreduce_bound(parts)
    assert np.all(np.abs(got - exact) <= bound)
    # a reduce that loses a rank is far outside it
    if ranks > 1:
        lost = tpm.quant_allreduce(parts[:-1] + [np.zeros_like(parts[-1])]).astype(np.float64)
        assert np.any(np.abs(lost - exact) > bound)


def test_quant_allreduce_of_one_rank_quantises_twice():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((4, 128)).astype(np.float32)
    once = tpm.dequantize(*tpm.quantize(x))
    assert np.array_equal(tpm.quant_allreduce([x]), tpm.dequantize(*tpm.quantize(once)))


@pytest.mark.parametrize("ranks", [2, 4])
def test_sharded_layer_equals_the_whole_layer(ranks):
    (u, w), cfg = _small()
    whole = tpm.mixer(u, w, cfg.ngroups, cfg.dstate, cfg.headdim)
    parts = [tpm.partial_output(u, w, r, ranks, cfg.ngroups, cfg.dstate, cfg.headdim) for r in range(ranks)]
    assert np.max(np.abs(np.sum(parts, axis=0) - whole)) <= 1e-9 * (1 + np.max(np.abs(whole)))
    # each rank's local output is the matching slice of the whole layer's normalised output
    s = tpm.shard_weights(w, 1, ranks)
    full = tpm.local_output(u, tpm.shard_weights(w, 0, 1), cfg.ngroups, cfg.dstate, cfg.headdim)
    Hr = cfg.nheads // ranks
    loc = tpm.local_output(u, s, cfg.ngroups // ranks, cfg.dstate, cfg.headdim)
    assert np.allclose(loc, full[:, Hr * cfg.headdim:2 * Hr * cfg.headdim], atol=1e-10)


def test_norm_groups_that_straddle_ranks_would_not_be_local():
    """With fewer groups than ranks a group's statistics span two devices: the per-rank norm then
    differs from the whole layer's (why the groups must be a multiple of the TP degree)."""
    (u, w), cfg = _small()
    whole = tpm.local_output(u, tpm.shard_weights(w, 0, 1), 1, cfg.dstate, cfg.headdim)
    Hr = cfg.nheads // 2
    half = tpm.local_output(u, tpm.shard_weights(w, 0, 2), 1, cfg.dstate, cfg.headdim)
    assert not np.allclose(half, whole[:, :Hr * cfg.headdim], atol=1e-6)


def test_bf16_hand_offs_round_only_between_steps():
    """With bf16 hand-offs the layer's output moves by the roundings' size, not more; for a zero
    input (y = 0, so the norm's output is beta) the only rounding left is that of beta."""
    (u, w), cfg = _small()
    a = tpm.mixer(u, w, cfg.ngroups, cfg.dstate, cfg.headdim)
    b = tpm.mixer(u, w, cfg.ngroups, cfg.dstate, cfg.headdim, bf16_between_steps=True)
    rel = np.abs(a - b) / (1 + np.abs(a))
    assert 1e-5 < rel.max() < 0.1
    z = u * 0
    beta = w["beta"].double().numpy()
    W_out = w["W_out"].double().numpy()
    assert np.allclose(tpm.mixer(z, w, cfg.ngroups, cfg.dstate, cfg.headdim), beta @ W_out, rtol=0, atol=1e-12)
    beta16 = torch.from_numpy(beta).to(torch.bfloat16).double().numpy()
    assert np.allclose(tpm.mixer(z, w, cfg.ngroups, cfg.dstate, cfg.headdim, bf16_between_steps=True),
                       beta16 @ W_out, rtol=0, atol=1e-12)
