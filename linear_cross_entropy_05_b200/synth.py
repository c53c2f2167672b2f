"""Seeded synthetic inputs for the Cut Cross-Entropy hot path.

This module only draws inputs; it holds none of the loss arithmetic.  Both the
CUDA path and the CPU oracle are fed from here, so they see identical bits.

Workloads follow the LLM classifier-head shapes the CCE abstract talks about
(Cut Cross-Entropy abstract, sentences 1-3 and 8: vocabularies that grow with
model size, a Gemma 2 (2B) example):

* embeddings E (N x D) and classifier C (V x D) drawn in fp32 from N(0, std)
  and rounded to bf16 with round-to-nearest-even; they are returned as raw
  uint16 bf16 bit patterns so that no consumer re-rounds them;
* labels y (N, int64) drawn uniformly or from a truncated Zipf law over the
  vocabulary (P(rank k) proportional to k^-s, k = 1..V, label id = k - 1);
* optionally a fixed fraction of tokens replaced by ignore_index, chosen by a
  seeded shuffle, and a fixed fraction of C rows scaled before rounding
  (a "peaky" softmax).

Draw order inside one workload: E, C, the scaled C-row subset, labels, the
ignored positions.  Every draw comes from numpy's PCG64 seeded per workload.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

IGNORE_INDEX = -100


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    D: int
    V: int
    std: float            # standard deviation of the N(0, std) draws for E and C
    labels: str           # "uniform" or "zipf"
    zipf_s: float = 1.1
    ignore_frac: float = 0.0
    peaky_frac: float = 0.0   # fraction of C rows scaled by peaky_scale
    peaky_scale: float = 1.0
    filter_eps: float = 0.0   # gradient filter threshold used with this workload (<= 0: off)
    seed: int = 0

    def with_sizes(self, N: Optional[int] = None, V: Optional[int] = None,
                   D: Optional[int] = None, name: Optional[str] = None) -> "Workload":
        """Same distributions at other sizes (used for parity tests that the
        oracle finishes in seconds)."""
        return dataclasses.replace(
            self, N=self.N if N is None else N, V=self.V if V is None else V,
            D=self.D if D is None else D,
            name=name or f"{self.name}[N={N or self.N},D={D or self.D},V={V or self.V}]")


EPS_BF16_FILTER = 2.0 ** -12

# The five LLM-head workloads.
TINY = Workload("tiny", N=256, D=256, V=4096, std=1.0 / 16.0, labels="uniform",
                filter_eps=0.0, seed=20260000)
GEMMA2_2B = Workload("gemma2-2b-head", N=8192, D=2304, V=256000, std=0.02, labels="zipf",
                     zipf_s=1.1, filter_eps=EPS_BF16_FILTER, seed=20260001)
LLAMA3_8B = Workload("llama3-8b-head", N=16384, D=4096, V=128256, std=0.02, labels="zipf",
                     zipf_s=1.1, ignore_frac=0.10, filter_eps=EPS_BF16_FILTER, seed=20260002)
SMALL_LARGE_VOCAB = Workload("small-model-large-vocab", N=32768, D=896, V=151936, std=0.02,
                             labels="zipf", zipf_s=1.2, peaky_frac=0.01, peaky_scale=8.0,
                             filter_eps=EPS_BF16_FILTER, seed=20260003)
SWEEP = Workload("long-batch-sweep", N=16384, D=2048, V=262144, std=0.02, labels="uniform",
                 filter_eps=EPS_BF16_FILTER, seed=20260004)
SWEEP_NS = (4096, 16384, 65536)

WORKLOADS = {w.name: w for w in (TINY, GEMMA2_2B, LLAMA3_8B, SMALL_LARGE_VOCAB, SWEEP)}


def round_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit pattern, round to nearest, ties to even (inputs are finite)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def _normal_bf16(rng: np.random.Generator, rows: int, cols: int, std: float,
                 chunk_rows: int = 8192) -> np.ndarray:
    out = np.empty((rows, cols), dtype=np.uint16)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = rng.standard_normal((r1 - r0, cols), dtype=np.float32)
        x *= np.float32(std)
        out[r0:r1] = round_to_bf16_bits(x)
    return out


def zipf_labels(rng: np.random.Generator, n: int, V: int, s: float) -> np.ndarray:
    """Truncated Zipf over ranks 1..V by inverse CDF; rank k maps to id k-1."""
    w = np.arange(1, V + 1, dtype=np.float64) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(n)
    ids = np.searchsorted(cdf, u, side="right")
    return np.minimum(ids, V - 1).astype(np.int64)


def make_inputs(w: Workload) -> dict:
    """Draw E, C (bf16 bits), y (int64) for workload w."""
    rng = np.random.Generator(np.random.PCG64(w.seed))
    E = _normal_bf16(rng, w.N, w.D, w.std)
    if w.peaky_frac > 0.0:
        # C is drawn in fp32 first so the chosen rows can be scaled before rounding.
        C = np.empty((w.V, w.D), dtype=np.uint16)
        Cf = rng.standard_normal((w.V, w.D), dtype=np.float32)
        Cf *= np.float32(w.std)
        n_peaky = int(np.floor(w.peaky_frac * w.V))
        peaky = rng.permutation(w.V)[:n_peaky]
        Cf[peaky] *= np.float32(w.peaky_scale)
        C[:] = round_to_bf16_bits(Cf)
        del Cf
    else:
        C = _normal_bf16(rng, w.V, w.D, w.std)
        peaky = np.zeros(0, dtype=np.int64)
    if w.labels == "uniform":
        y = rng.integers(0, w.V, size=w.N, dtype=np.int64)
    elif w.labels == "zipf":
        y = zipf_labels(rng, w.N, w.V, w.zipf_s)
    else:
        raise ValueError(f"unknown label law {w.labels!r}")
    n_ign = int(np.floor(w.ignore_frac * w.N))
    if n_ign:
        y[rng.permutation(w.N)[:n_ign]] = IGNORE_INDEX
    return {"E": E, "C": C, "y": y, "peaky_rows": np.sort(peaky), "workload": w}


def mean_dloss(y: np.ndarray, ignore_index: int = IGNORE_INDEX) -> np.ndarray:
    """Upstream gradient of a mean reduction over non-ignored tokens (fp32).

    This is the caller's reduction, not part of the per-token loss: each kept
    token gets 1/#kept, ignored tokens get 0.  All tokens ignored gives zeros.
    """
    keep = y != ignore_index
    n = int(keep.sum())
    out = np.zeros(y.shape[0], dtype=np.float32)
    if n:
        out[keep] = np.float32(1.0 / n)
    return out


def random_dloss(seed: int, n: int) -> np.ndarray:
    """Seeded per-token upstream gradients in [0.5, 1.5) (fp32), so that a
    dropped or misplaced dLoss factor shows up in parity checks."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return (0.5 + rng.random(n)).astype(np.float32)
