"""Writes fullsize_oracle.npz: the fp64 oracle's per-token loss and lse for
every full-size LLM-head workload.

    python tests/golden/make_fullsize_oracle.py [--threads T]

The full fp64 forward of these workloads (2 N D V flops plus N V
exponentials each, ~130 TFLOP in all) takes tens of minutes on a few host
cores, too long to repeat inside every GPU test run.  This script runs it
once and stores the result; the full-size parity tests read it, so they can
hold every token's loss, the mean loss and the gradient rows (which need the
lse of every token) to the oracle at full size.

Only two modules are used: the seeded input generator and the oracle.  The
rows of each workload are split into contiguous chunks that the oracle
evaluates in worker threads (numpy releases the GIL in its matrix products and
exponentials; each worker's BLAS runs single-threaded); the oracle's
arithmetic per row does not depend on the chunking.

Stored per workload (key = workload name): `<name>/loss`, `<name>/lse`
(float64, N each).  tests/test_fullsize_golden.py recomputes sampled rows
with the oracle and checks them against the file.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from linear_cross_entropy_05_b200 import synth  # noqa: E402

OUT = os.path.join(HERE, "fullsize_oracle.npz")
IGN = synth.IGNORE_INDEX


def full_workloads():
    """The full-size workloads whose per-token outputs are stored."""
    return [synth.GEMMA2_2B, synth.LLAMA3_8B, synth.SMALL_LARGE_VOCAB] + \
        [synth.SWEEP.with_sizes(N=n, name=f"long-batch-sweep[N={n}]") for n in synth.SWEEP_NS]


def oracle_forward_rows(inp, r0, r1, C64):
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1, user_api="blas"):
        E64 = oracle.bf16_bits_to_f64(inp["E"][r0:r1])
        return oracle.forward_f64(E64, C64, inp["y"][r0:r1], IGN)


def run(threads: int, only=None):
    data = {}
    if os.path.exists(OUT):
        with np.load(OUT) as f:
            data = {k: f[k] for k in f.files}
    for w in full_workloads():
        if only and w.name not in only:
            continue
        if f"{w.name}/lse" in data:
            print(f"{w.name}: stored already", flush=True)
            continue
        t0 = time.time()
        inp = synth.make_inputs(w)
        C64 = oracle.bf16_bits_to_f64(inp["C"])
        chunk = max(64, -(-w.N // (8 * threads)))
        bounds = [(r0, min(w.N, r0 + chunk)) for r0 in range(0, w.N, chunk)]
        loss = np.empty(w.N, dtype=np.float64)
        lse = np.empty(w.N, dtype=np.float64)
        with cf.ThreadPoolExecutor(threads) as ex:
            futs = {ex.submit(oracle_forward_rows, inp, r0, r1, C64): (r0, r1) for r0, r1 in bounds}
            for fu in cf.as_completed(futs):
                r0, r1 = futs[fu]
                loss[r0:r1], lse[r0:r1] = fu.result()
        data[f"{w.name}/loss"] = loss
        data[f"{w.name}/lse"] = lse
        np.savez(OUT, **data)
        print(f"{w.name}: N={w.N} D={w.D} V={w.V} in {time.time() - t0:.0f} s", flush=True)


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--threads", type=int, default=os.cpu_count())
    ap.add_argument("--only", nargs="*", default=None)
    a = ap.parse_args()
    run(a.threads, a.only)
