"""The seeded input generator: determinism and the stated distributions."""
import numpy as np

from linear_cross_entropy_05_b200 import synth


def test_deterministic_and_seed_sensitive():
    w = synth.TINY.with_sizes(N=64, V=512, D=32)
    a = synth.make_inputs(w)
    b = synth.make_inputs(w)
    assert (a["E"] == b["E"]).all() and (a["C"] == b["C"]).all() and (a["y"] == b["y"]).all()
    c = synth.make_inputs(w.__class__(**{**w.__dict__, "seed": w.seed + 1}))
    assert not (a["E"] == c["E"]).all()


def test_shapes_dtypes_and_std():
    w = synth.GEMMA2_2B.with_sizes(N=512, V=4096, D=256)
    inp = synth.make_inputs(w)
    assert inp["E"].shape == (512, 256) and inp["E"].dtype == np.uint16
    assert inp["C"].shape == (4096, 256) and inp["y"].dtype == np.int64
    x = (inp["C"].astype(np.uint32) << 16).view(np.float32)
    assert abs(x.std() - 0.02) < 0.0005
    assert abs(x.mean()) < 0.0005


def test_ignore_fraction_is_exact():
    w = synth.LLAMA3_8B.with_sizes(N=1000, V=2048, D=16)
    y = synth.make_inputs(w)["y"]
    assert int((y == synth.IGNORE_INDEX).sum()) == 100
    assert ((y == synth.IGNORE_INDEX) | ((y >= 0) & (y < 2048))).all()


def test_peaky_rows_scaled_before_rounding():
    w = synth.SMALL_LARGE_VOCAB.with_sizes(N=64, V=3000, D=64)
    inp = synth.make_inputs(w)
    assert inp["peaky_rows"].shape == (30,)
    x = (inp["C"].astype(np.uint32) << 16).view(np.float32)
    norms = np.linalg.norm(x, axis=1)
    peaky = np.zeros(3000, bool)
    peaky[inp["peaky_rows"]] = True
    assert norms[peaky].mean() / norms[~peaky].mean() > 7.0


def test_zipf_labels_range_and_rank_order():
    rng = np.random.Generator(np.random.PCG64(5))
    y = synth.zipf_labels(rng, 200000, 1000, 1.1)
    assert y.min() >= 0 and y.max() < 1000
    cnt = np.bincount(y, minlength=1000)
    assert cnt[0] > cnt[1] > cnt[3] > cnt[10] > cnt[100]
    # P(rank 1) / P(rank 2) = 2^s
    assert abs(cnt[0] / cnt[1] - 2 ** 1.1) < 0.1


def test_mean_dloss():
    y = np.array([3, synth.IGNORE_INDEX, 1, 0])
    d = synth.mean_dloss(y)
    assert d.dtype == np.float32 and np.allclose(d, [1 / 3, 0, 1 / 3, 1 / 3])
    assert (synth.mean_dloss(np.full(4, synth.IGNORE_INDEX)) == 0).all()
