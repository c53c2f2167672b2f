"""The five LLM-head workloads at full size, in the launch configuration the
benchmark times.  The oracle checks sampled outputs it can compute one by one
(per-token loss/lse rows, dE rows of whole 128-token blocks) and, for the
Gemma-2-2B-shaped head, dC rows after its own full fp64 forward; identities
that hold at any size cover the rest."""
import numpy as np
import pytest

import oracle
from linear_cross_entropy_05_b200 import synth

from _gpu_helpers import (GRAD_REL_FILTER_ON, IGN, LOSS_ABS, gpu_backward, gpu_forward, rel_fro, to_dev)

pytestmark = pytest.mark.gpu

FULL = [synth.GEMMA2_2B, synth.LLAMA3_8B, synth.SMALL_LARGE_VOCAB] + \
       [synth.SWEEP.with_sizes(N=n, name=f"long-batch-sweep[N={n}]") for n in synth.SWEEP_NS]


def _sample_rows(N, k, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, N - 1], rng.choice(N, size=k, replace=False)]))


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_full_size_forward_backward_sampled(w):
    import torch
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    assert st["status"] == 0 and st["flags"] == 0
    rows = _sample_rows(w.N, 48, 7)
    ol, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN, rows=rows)
    assert np.abs(loss[rows] - ol).max() <= LOSS_ABS
    assert np.abs(lse[rows] - olse).max() <= LOSS_ABS
    assert np.isfinite(lse).all()

    dloss = synth.mean_dloss(inp["y"])
    dE, dC, st = gpu_backward(E, C, y, lse, dloss, w.filter_eps)
    assert st["status"] == 0 and st["flags"] == 0
    n_tiles = -(-w.N // 32) * -(-w.V // 32)   # 32 x 32 filter units
    assert st["live_tiles"] + st["dead_tiles"] + st["pruned_tiles"] == n_tiles
    # at full vocabulary size |E_i| max|C_v| < lse_i + ln(eps) for these
    # random-init heads: only label tiles are recomputed
    assert st["pruned_tiles"] > 0.8 * n_tiles

    # dE rows of two whole token blocks (the tile filter needs the block's lse)
    blocks = [0, (w.N // 128) // 2]
    lse_o = np.full(w.N, np.nan)
    for b in blocks:
        r = np.arange(b * 128, min(w.N, (b + 1) * 128))
        _, lse_o[r] = oracle.forward(inp["E"], inp["C"], inp["y"], IGN, rows=r)
    rE = np.concatenate([np.arange(b * 128, min(w.N, (b + 1) * 128)) for b in blocks])
    oE, _ = oracle.backward_sampled(inp["E"], inp["C"], inp["y"], lse_o, dloss, IGN, rE, [],
                                    filter_eps=w.filter_eps, tile=(32, 32))
    gE = dE[torch.from_numpy(rE).cuda()].cpu().numpy()
    assert rel_fro(gE, oE) <= GRAD_REL_FILTER_ON

    # <E, dE> = <C, dC> for any filtered G
    a = float((E.double() * dE.double()).sum())
    b = float((C.double() * dC.double()).sum())
    assert abs(a - b) <= 1e-2 * max(abs(a), abs(b))


def test_full_size_gemma_dC_rows_and_mean_loss():
    import torch
    w = synth.GEMMA2_2B
    inp = synth.make_inputs(w)
    E, C, y = to_dev(inp)
    loss, lse, st = gpu_forward(E, C, y)
    ol, olse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN)   # full fp64 forward
    assert np.abs(loss - ol).max() <= LOSS_ABS
    keep = inp["y"] != IGN
    assert abs(loss[keep].astype(np.float64).mean() - ol[keep].mean()) <= 1e-4 * ol[keep].mean()
    dloss = synth.mean_dloss(inp["y"])
    dE, dC, st = gpu_backward(E, C, y, lse, dloss, w.filter_eps)
    # vocabulary rows: the most frequent labels, a rare one, the last row and
    # rows of the ragged last tile region
    counts = np.bincount(inp["y"], minlength=w.V)
    rC = np.unique(np.concatenate([np.argsort(-counts)[:6], [int(np.argmax(counts == 1))], [w.V - 1, 7777]]))
    _, oC = oracle.backward_sampled(inp["E"], inp["C"], inp["y"], olse, dloss, IGN, [], rC,
                                    filter_eps=w.filter_eps, tile=(32, 32))
    gC = dC[torch.from_numpy(rC).cuda()].cpu().numpy()
    assert rel_fro(gC, oC) <= GRAD_REL_FILTER_ON
