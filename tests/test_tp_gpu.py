"""The head-sharded mixer's library kernels and the emulated Tp-way layer against the oracle.

"5.3 Tensor Parallelism support and large-cluster training", section 4.1 (heads split over Tp
devices; group norm local; one all-reduce of the output projection's partials) and "Scaling
State-Space Models on Multiple GPUs with Tensor Parallelism", abstract (quantised all-reduce):
* ssd_group_norm against the oracle's group norm (fp32 and bf16);
* the quantisation kernels code for code against the oracle's quantiser (the codes are decided in
  float32 on both sides, the products and sums rounded separately);
* Tp = 1, 2, 4 ranks run in turn on one GPU (run_local_tp): with an exact all-reduce within the
  bf16 bound of the fp64 layer (whose tensors are rounded to bf16 where the layer hands them from
  one step to the next in bf16), with the quantised one within that plus the scheme's own bound.
"""
import numpy as np
import pytest
import torch

from oracle import tp_mixer as tpm
from state_space_model_07_b200 import inputs, tp

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,rows,C,ng", [(torch.float32, 37, 640, 4), (torch.bfloat16, 300, 512, 4),
                                             (torch.bfloat16, 5, 2048, 1), (torch.float32, 1, 64, 64)])
def test_group_norm_matches_the_oracle(dtype, rows, C, ng):
    rng = np.random.default_rng(rows + C)
    x = torch.from_numpy((rng.standard_normal((rows, C)) * 3 + 1).astype(np.float32)).to(dtype).cuda()
    g = torch.from_numpy(rng.standard_normal(C).astype(np.float32)).cuda()
    b = torch.from_numpy(rng.standard_normal(C).astype(np.float32)).cuda()
    out = tp.group_norm(x, g, b, ng)
    ref = tpm.group_norm(x, g, b, ng)
    tol = 1e-4 if dtype == torch.float32 else 1e-2
    assert np.max(np.abs(out.float().cpu().numpy() - ref) / (1 + np.abs(ref))) <= tol


def _partials(ranks, T=33, D=None, seed=0):
    rng = np.random.default_rng(seed)
    D = D or 64 * ranks * 3
    parts = []
    for _ in range(ranks):
        p = rng.standard_normal((T, D)) * np.exp(rng.uniform(-6, 6, (T, 1)))
        p[3, :64] = 0.0                      # an all-zero block
        parts.append(p.astype(np.float32))
    return parts


@pytest.mark.parametrize("ranks", [1, 2, 3, 4])
def test_quantisation_kernels_match_the_oracle_code_for_code(ranks):
    parts = _partials(ranks, seed=ranks)
    T, D = parts[0].shape
    Dc, nbc = D // ranks, D // ranks // 64
    qs = [tp.quant_chunks(torch.from_numpy(p).cuda(), ranks) for p in parts]
    for p, (q, s) in zip(parts, qs):
        codes, sc = tpm.quantize(p)
        for j in range(ranks):
            assert np.array_equal(q[j].cpu().numpy(), codes[:, j * Dc:(j + 1) * Dc])
            assert np.array_equal(s[j].cpu().numpy(), sc[:, j * nbc:(j + 1) * nbc])
    # the reduce step and the final dequantisation: the whole quantised all-reduce, bit for bit
    red = [tp.dequant_sum_quant(torch.stack([qs[r][0][j] for r in range(ranks)]),
                                torch.stack([qs[r][1][j] for r in range(ranks)])) for j in range(ranks)]
    qa, sa = torch.stack([q for q, _ in red]), torch.stack([s for _, s in red])
    got = tp.dequant_chunks(qa, sa, torch.float32).cpu().numpy()
    assert np.array_equal(got, tpm.quant_allreduce(parts))
    got16 = tp.dequant_chunks(qa, sa, torch.bfloat16).cpu()
    assert torch.equal(got16, torch.from_numpy(tpm.quant_allreduce(parts)).to(torch.bfloat16))


@pytest.mark.parametrize("ranks", [1, 2, 4])
@pytest.mark.parametrize("quantized", [False, True])
def test_sharded_layer_matches_the_oracle(ranks, quantized):
    cfg = inputs.MIXERS["mixer_small"]
    u, w = inputs.make_mixer(cfg, "cuda")
    out = tp.run_local_tp(u, w, ranks, ngroups=cfg.ngroups, dstate=cfg.dstate, headdim=cfg.headdim,
                          chunk=cfg.chunk, quantized=quantized)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    # the oracle rounds to bf16 where the layer hands a tensor from one step to the next in bf16
    ref = tpm.mixer(u, w, cfg.ngroups, cfg.dstate, cfg.headdim, bf16_between_steps=True)
    bound = 1e-2 * (1 + np.abs(ref))
    if quantized:
        parts = [tpm.partial_output(u, w, r, ranks, cfg.ngroups, cfg.dstate, cfg.headdim,
                                    bf16_between_steps=True).astype(np.float32) for r in range(ranks)]
        # plus the scheme's own bound, and the bf16 rounding of the dequantised output
        bound = bound + tpm.quant_allreduce_bound(parts) + np.abs(ref) * 2.0 ** -8
    assert np.all(np.abs(got - ref) <= bound), float(np.max(np.abs(got - ref) / bound))
