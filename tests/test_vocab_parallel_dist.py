"""Vocabulary-parallel step over two gloo ranks on the CPU.

`vocab_parallel_forward_backward` splits the classifier by rows across ranks:
each rank computes per-token (max, sum exp, target logit) over its shard, the
ranks all-gather these 12 bytes per token, merge them into the log-sum-exp
(lse = M + log sum_r s_r exp(m_r - M)), run their shard's backward with the
merged lse and all-reduce the dE shares.  On a GPU the three per-shard steps
are the library's CUDA entry points; here they are replaced by fp64 stand-ins
built from the oracle that follow the same contract, so that the exchange
itself (gather order, stacking, merge input, the dE all-reduce) runs on two
real processes and is checked against the unsharded oracle.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
IGN = -100


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _bits(t):
    import torch
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _install_stand_ins(L):
    """Per-shard compute in fp64 on the CPU, same inputs and outputs as the
    library's forward_shard / merge_shards / backward_shard."""
    import torch
    import oracle

    def forward_shard(E, C_shard, y, v_offset, ignore_index=IGN, **_):
        z = oracle.logits(oracle.bf16_bits_to_f64(_bits(E)), oracle.bf16_bits_to_f64(_bits(C_shard)))
        m = z.max(axis=1)
        s = np.exp(z - m[:, None]).sum(axis=1)
        yl = y.numpy() - v_offset
        own = (y.numpy() != ignore_index) & (yl >= 0) & (yl < z.shape[1])
        t = np.where(own, z[np.arange(len(yl)), np.clip(yl, 0, z.shape[1] - 1)], 0.0)
        return torch.from_numpy(np.stack([m, s, t]).astype(np.float32))

    def merge_shards(stats, y, V_total, ignore_index=IGN, **_):
        st = stats.numpy().astype(np.float64)            # [R, 3, N]
        M = st[:, 0].max(axis=0)
        lse = M + np.log((st[:, 1] * np.exp(st[:, 0] - M)).sum(axis=0))
        keep = y.numpy() != ignore_index
        loss = np.where(keep, lse - st[:, 2].sum(axis=0), 0.0)
        return torch.from_numpy(loss.astype(np.float32)), torch.from_numpy(lse.astype(np.float32))

    def backward_shard(E, C_shard, y, lse, dloss, v_offset, filter_eps=0.0, ignore_index=IGN, **_):
        E64 = oracle.bf16_bits_to_f64(_bits(E))
        C64 = oracle.bf16_bits_to_f64(_bits(C_shard))
        z = oracle.logits(E64, C64)
        G = np.exp(z - lse.numpy().astype(np.float64)[:, None])
        yl = y.numpy() - v_offset
        rows = np.nonzero((y.numpy() != ignore_index) & (yl >= 0) & (yl < z.shape[1]))[0]
        G[rows, yl[rows]] -= 1.0
        G[y.numpy() == ignore_index] = 0.0
        G *= dloss.numpy().astype(np.float64)[:, None]
        return torch.from_numpy((G @ C64).astype(np.float32)), torch.from_numpy((G.T @ E64).astype(np.float32))

    L.forward_shard = forward_shard
    L.merge_shards = merge_shards
    L.backward_shard = backward_shard


def _worker(rank, world, port, bounds, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    import linear_cross_entropy_05_b200 as L
    from linear_cross_entropy_05_b200 import synth
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        _install_stand_ins(L)
        w = synth.GEMMA2_2B.with_sizes(N=96, V=bounds[-1], D=32)
        inp = synth.make_inputs(w)
        E = torch.from_numpy(inp["E"].view(np.int16)).view(torch.bfloat16)
        C = torch.from_numpy(inp["C"].view(np.int16)).view(torch.bfloat16)
        y = torch.from_numpy(inp["y"])
        y[5] = IGN
        lo, hi = bounds[rank], bounds[rank + 1]
        loss, lse, dE, dC = L.vocab_parallel_forward_backward(E, C[lo:hi].contiguous(), y, lo, w.V,
                                                              filter_eps=0.0, ignore_index=IGN)
        out[rank] = (loss.numpy(), lse.numpy(), dE.numpy(), dC.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("bounds", [[0, 130, 300], [0, 1, 300]], ids=["uneven", "one-row-shard"])
def test_two_rank_vocab_parallel_step_matches_unsharded_oracle(bounds):
    import oracle
    from linear_cross_entropy_05_b200 import synth
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), bounds, out), nprocs=world, join=True,
                       start_method="spawn")
    w = synth.GEMMA2_2B.with_sizes(N=96, V=bounds[-1], D=32)
    inp = synth.make_inputs(w)
    y = inp["y"].copy()
    y[5] = IGN
    loss, lse = oracle.forward(inp["E"], inp["C"], y, IGN)
    keep = y != IGN
    dloss = keep / keep.sum()
    dE, dC = oracle.backward(inp["E"], inp["C"], y, lse, dloss, IGN)
    for r in range(world):
        l_r, lse_r, dE_r, dC_r = out[r]
        # loss, lse and dE are the same on every rank and equal the unsharded result
        np.testing.assert_allclose(l_r, loss, rtol=0, atol=1e-5)
        np.testing.assert_allclose(lse_r, lse, rtol=0, atol=1e-5)
        np.testing.assert_allclose(dE_r, dE, rtol=1e-4, atol=1e-9)
        # each rank holds exactly its own rows of dC
        np.testing.assert_allclose(dC_r, dC[bounds[r]:bounds[r + 1]], rtol=1e-4, atol=1e-9)
    assert (out[0][2] == out[1][2]).all()   # the all-reduce leaves identical dE everywhere
