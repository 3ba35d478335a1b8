"""The head-sharded mixer's exchanges on gloo ranks (CPU): the library's mixer_fwd with its
torch.distributed communicator (all-to-all of the code chunks, all-gather of the reduced chunks),
the compute steps supplied by the fp64 / float32 oracle, must reproduce the oracle's quantised
all-reduce of the per-rank partials bit for bit ("5.3 Tensor Parallelism support and large-cluster
training", section 4.1: one all-reduce per layer; "Scaling State-Space Models on Multiple GPUs with
Tensor Parallelism", abstract: quantised).  The GPU kernels are checked in tests/test_tp_gpu.py."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_ops():
    import torch
    from oracle import tp_mixer as tpm
    from state_space_model_07_b200.tp import TPOps

    class OracleTPOps(TPOps):
        def local_output(self, u, s, *, ngroups, dstate, headdim, chunk):
            sd = {k: v.double().numpy() for k, v in s.items()}
            return torch.from_numpy(tpm.local_output(u, sd, ngroups, dstate, headdim))

        def out_proj(self, n, s):
            return torch.from_numpy((n.numpy() @ s["W_out"].double().numpy()).astype(np.float32))

        def quant_chunks(self, z, ranks):
            codes, sc = tpm.quantize(z.numpy())
            T, D = codes.shape
            q = codes.reshape(T, ranks, D // ranks).transpose(1, 0, 2).copy()
            s = sc.reshape(T, ranks, -1).transpose(1, 0, 2).copy()
            return torch.from_numpy(q), torch.from_numpy(s)

        def dequant_sum_quant(self, q, s):
            acc = np.zeros(q.shape[1:], dtype=np.float32)
            for r in range(q.shape[0]):
                acc = (acc + tpm.dequantize(q[r].numpy(), s[r].numpy())).astype(np.float32)
            codes, sc = tpm.quantize(acc)
            return torch.from_numpy(codes), torch.from_numpy(sc)

        def dequant_chunks(self, q, s, dtype):
            ranks, T, Dc = q.shape
            out = np.concatenate([tpm.dequantize(q[j].numpy(), s[j].numpy()) for j in range(ranks)], axis=1)
            return torch.from_numpy(out)

    return OracleTPOps()


def _worker(rank, world, port, out):
    import torch.distributed as dist
    from state_space_model_07_b200 import inputs
    from state_space_model_07_b200.tp import TorchDistTPComm, mixer_fwd, shard
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = inputs.MIXERS["mixer_small"]
        u, w = inputs.make_mixer(cfg, "cpu")
        z = mixer_fwd(u, shard(w, rank, world), TorchDistTPComm(), ngroups=cfg.ngroups, dstate=cfg.dstate,
                      headdim=cfg.headdim, chunk=cfg.chunk, ops_=_oracle_ops())
        out[rank] = z.numpy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_quantised_all_reduce_over_gloo_ranks(world):
    from oracle import tp_mixer as tpm
    from state_space_model_07_b200 import inputs
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    cfg = inputs.MIXERS["mixer_small"]
    u, w = inputs.make_mixer(cfg, "cpu")
    parts = [(tpm.local_output(u, tpm.shard_weights(w, r, world), cfg.ngroups // world, cfg.dstate, cfg.headdim)
              @ tpm.shard_weights(w, r, world)["W_out"]).astype(np.float32) for r in range(world)]
    want = tpm.quant_allreduce(parts)
    for r in range(world):
        assert np.array_equal(res[r], want), r
