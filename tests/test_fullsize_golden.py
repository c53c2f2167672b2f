"""The stored full-size oracle values (tests/golden/fullsize_oracle.npz,
written by tests/golden/make_fullsize_oracle.py) still match the oracle and
the input generator: a few seeded rows of a workload are recomputed here
with the oracle and compared.  Drawing a full-size workload takes 5-40 s on a
few host cores, so the default run checks three of them (the Gemma-2-2B
head, the small-model head and the smallest sweep); CCE_GOLDEN_ALL=1 checks
every one."""
import os

import numpy as np
import pytest

import oracle
from linear_cross_entropy_05_b200 import synth

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "fullsize_oracle.npz")
IGN = -100

FULL = [synth.GEMMA2_2B, synth.LLAMA3_8B, synth.SMALL_LARGE_VOCAB] + \
       [synth.SWEEP.with_sizes(N=n, name=f"long-batch-sweep[N={n}]") for n in synth.SWEEP_NS]


def test_golden_file_covers_every_full_size_workload():
    with np.load(GOLDEN) as f:
        for w in FULL:
            for k in ("loss", "lse"):
                a = f[f"{w.name}/{k}"]
                assert a.shape == (w.N,) and a.dtype == np.float64 and np.isfinite(a).all()


DEFAULT = {synth.GEMMA2_2B.name, synth.SMALL_LARGE_VOCAB.name, "long-batch-sweep[N=4096]"}


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_golden_rows_recomputed_by_the_oracle(w):
    if w.name not in DEFAULT and os.environ.get("CCE_GOLDEN_ALL") != "1":
        pytest.skip("set CCE_GOLDEN_ALL=1 to recompute rows of every full-size workload")
    inp = synth.make_inputs(w)
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, w.N - 1], rng.choice(w.N, size=6, replace=False)]))
    loss, lse = oracle.forward(inp["E"], inp["C"], inp["y"], IGN, rows=rows)
    with np.load(GOLDEN) as f:
        g_loss, g_lse = f[f"{w.name}/loss"][rows], f[f"{w.name}/lse"][rows]
    np.testing.assert_allclose(lse, g_lse, rtol=1e-12, atol=0)
    np.testing.assert_allclose(loss, g_loss, rtol=1e-10, atol=1e-12)
    # the workload's kept/ignored pattern is the one the file was made from
    assert ((inp["y"][rows] == IGN) == (g_loss == 0)).all()
