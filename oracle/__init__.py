"""fp64 CPU oracle for the Cut Cross-Entropy (CCE) hot path.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check of the graft
entry point and the CPU-baseline leg of the benchmark may import this module.
The product path (the CUDA library and its Python binding) never calls it and
shares no code with it.

What it computes (Cut Cross-Entropy abstract, sentences 4-5: the cross-entropy
loss is the log-sum-exp over all logits minus the logit of the correct token;
CCE reaches exactly that value without storing the logits, so the oracle is the
plain definition):

    z[i, v]   = sum_d E[i, d] * C[v, d]                       (logits)
    lse[i]    = max_v z[i, v] + log sum_v exp(z[i, v] - max_v z[i, v])
    loss[i]   = lse[i] - z[i, y[i]]        (0 where y[i] == ignore_index)
    P[i, v]   = exp(z[i, v] - lse[i])                           (softmax)
    G[i, v]   = dloss[i] * (P[i, v] - [v == y[i]])    (0 for ignored rows)
    dE        = G @ C,    dC = G^T @ E

The backward recomputation and the gradient filter follow the abstract's
sentence 9 (skip the elements of the gradient computation whose contribution
is below numerical precision).  The filter is written for any tile of the
gradient: a (Bn x Bv) tile of G, anchored at (0, 0), is dropped iff every
entry has |P - onehot| < eps; ignored rows and out-of-range rows/columns
count as zero; eps <= 0 disables it.  The default tile is (1, 1): every
element is kept or dropped on its own, which is the reading the library
computes.  Larger tiles (32 x 32 is one unit of the library's work
skipping) give the unit liveness the library counts.

Everything is float64 on the bf16-rounded inputs decoded exactly.  The only
blocking is over token rows (to bound memory); each row block materialises its
full logit row, so the log-sum-exp is the textbook max-shifted form.
A matrix product from numpy's BLAS is the one library primitive used.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(closed forms, invariants, finite differences, a library cross-entropy and
autograd, brute-force tile liveness and a hand-worked example).
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "bf16_bits_to_f64", "logits", "forward", "forward_f64", "mean_loss",
    "softmax_grad_f64", "backward", "backward_f64", "backward_sampled",
    "tile_live_map", "tile_live_map_f64",
]


# ---------------------------------------------------------------------------
# input decoding
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode raw bf16 bit patterns (uint16) exactly: bf16 is the top half of
    an fp32, so widening the bits by 16 zero bits gives the fp32 value, which
    fp64 holds exactly."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def _rows_per_block(V: int, budget_elems: int = 1 << 23) -> int:
    return max(1, budget_elems // max(1, V))


# ---------------------------------------------------------------------------
# forward: loss and LSE
# ---------------------------------------------------------------------------

def logits(E64: np.ndarray, C64: np.ndarray) -> np.ndarray:
    """z = E C^T, the full logit block for the given rows (fp64)."""
    return E64 @ C64.T


def _lse_of_rows(z: np.ndarray) -> np.ndarray:
    m = z.max(axis=1)
    return m + np.log(np.exp(z - m[:, None]).sum(axis=1))


def forward_f64(E64: np.ndarray, C64: np.ndarray, y: np.ndarray, ignore_index: int,
                rows: Optional[Sequence[int]] = None):
    """Per-token (loss, lse) in fp64 for fp64 inputs.

    rows: optional subset of token indices (sampled checks); the outputs then
    follow that order.  Labels outside [0, V) that are not ignore_index give
    NaN loss (the label is invalid), lse is still defined.
    """
    V = C64.shape[0]
    idx = np.arange(E64.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    loss = np.zeros(idx.shape[0], dtype=np.float64)
    lse = np.zeros(idx.shape[0], dtype=np.float64)
    rb = _rows_per_block(V)
    for r0 in range(0, idx.shape[0], rb):
        sel = idx[r0:r0 + rb]
        z = logits(E64[sel], C64)
        l = _lse_of_rows(z)
        lse[r0:r0 + rb] = l
        yy = y[sel]
        for k in range(sel.shape[0]):
            t = int(yy[k])
            if t == ignore_index:
                loss[r0 + k] = 0.0
            elif 0 <= t < V:
                loss[r0 + k] = l[k] - z[k, t]
            else:
                loss[r0 + k] = math.nan
    return loss, lse


def forward(E_bits: np.ndarray, C_bits: np.ndarray, y: np.ndarray, ignore_index: int,
            rows: Optional[Sequence[int]] = None):
    """forward_f64 on bf16 bit-pattern inputs."""
    return forward_f64(bf16_bits_to_f64(E_bits) if rows is None
                       else bf16_bits_to_f64(E_bits[np.asarray(rows)]),
                       bf16_bits_to_f64(C_bits), y if rows is None else y[np.asarray(rows)],
                       ignore_index)


def mean_loss(loss: np.ndarray, y: np.ndarray, ignore_index: int) -> float:
    """Mean over non-ignored tokens; NaN when every token is ignored."""
    keep = y != ignore_index
    n = int(keep.sum())
    return float(loss[keep].sum() / n) if n else math.nan


# ---------------------------------------------------------------------------
# backward
# ---------------------------------------------------------------------------

def softmax_grad_f64(z: np.ndarray, lse: np.ndarray, y: np.ndarray, dloss: np.ndarray,
                     ignore_index: int):
    """Return (P, onehot-difference D = P - onehot, G = dloss * D) for a block
    of full logit rows; ignored rows give D = G = 0."""
    P = np.exp(z - lse[:, None])
    Dm = P.copy()
    for k in range(z.shape[0]):
        t = int(y[k])
        if t == ignore_index:
            Dm[k, :] = 0.0
        else:
            Dm[k, t] -= 1.0
    G = Dm * dloss.astype(np.float64)[:, None]
    return P, Dm, G


def tile_live_map_f64(Dm_rows: np.ndarray, row0: int, Bn: int, Bv: int, eps: float):
    """Liveness of the (Bn x Bv) tiles covering a block of rows of
    D = P - onehot that starts at token row0 (row0 a multiple of Bn).
    A tile is live iff some entry has |D| >= eps."""
    assert row0 % Bn == 0
    nr, V = Dm_rows.shape
    nt_r = -(-nr // Bn)
    nt_v = -(-V // Bv)
    # pad with zeros (out-of-range rows/columns count as zero) and ask, per
    # (Bn x Bv) block, whether any entry reaches eps
    big = np.zeros((nt_r * Bn, nt_v * Bv), dtype=bool)
    big[:nr, :V] = np.abs(Dm_rows) >= eps
    return big.reshape(nt_r, Bn, nt_v, Bv).any(axis=(1, 3))


def backward_f64(E64, C64, y, lse, dloss, ignore_index: int, filter_eps: float = 0.0,
                 tile=(1, 1), return_live: bool = False):
    """Full dE (N x D) and dC (V x D) in fp64 from the given per-token lse.

    With filter_eps > 0 the tiles of G that are not live (see module doc) are
    dropped before the two products.  return_live adds the tile live map.
    """
    N, D = E64.shape
    V = C64.shape[0]
    Bn, Bv = tile
    dE = np.zeros((N, D), dtype=np.float64)
    dC = np.zeros((V, D), dtype=np.float64)
    rb = max(Bn, (_rows_per_block(V) // Bn) * Bn)
    lives = []
    for r0 in range(0, N, rb):
        r1 = min(N, r0 + rb)
        z = logits(E64[r0:r1], C64)
        _, Dm, G = softmax_grad_f64(z, lse[r0:r1], y[r0:r1], dloss[r0:r1], ignore_index)
        if filter_eps > 0.0 or return_live:
            live = tile_live_map_f64(Dm, r0, Bn, Bv, filter_eps if filter_eps > 0 else 0.0)
            lives.append(live)
            if filter_eps > 0.0:
                mask = np.repeat(np.repeat(live, Bn, axis=0), Bv, axis=1)[:r1 - r0, :V]
                G = np.where(mask, G, 0.0)
        dE[r0:r1] = G @ C64
        dC += G.T @ E64[r0:r1]
    if return_live:
        return dE, dC, np.concatenate(lives, axis=0)
    return dE, dC


def backward(E_bits, C_bits, y, lse, dloss, ignore_index: int, filter_eps: float = 0.0,
             tile=(1, 1), return_live: bool = False):
    """backward_f64 on bf16 bit-pattern inputs (lse from the oracle's forward)."""
    return backward_f64(bf16_bits_to_f64(E_bits), bf16_bits_to_f64(C_bits), y,
                        np.asarray(lse, dtype=np.float64), np.asarray(dloss), ignore_index,
                        filter_eps, tile, return_live)


def backward_sampled(E_bits, C_bits, y, lse_all, dloss, ignore_index: int,
                     rows_dE: Sequence[int], rows_dC: Sequence[int],
                     filter_eps: float = 0.0, tile=(1, 1)):
    """Selected rows of dE and of dC without forming the full gradients.

    rows_dE: token rows i; dE[i] = sum_v G[i, v] C[v] needs only row i's lse.
    rows_dC: vocab rows v; dC[v] = sum_i G[i, v] E[i] needs every token's lse
    (lse_all, the oracle's own forward over all tokens).
    With filter_eps > 0 the tile filter is applied, which needs every entry of
    the tiles that hold the requested rows/columns; those tiles are evaluated
    in full.
    """
    E64 = bf16_bits_to_f64(E_bits)
    C64 = bf16_bits_to_f64(C_bits)
    lse_all = np.asarray(lse_all, dtype=np.float64)
    dloss = np.asarray(dloss)
    N, V = E64.shape[0], C64.shape[0]
    Bn, Bv = tile
    rows_dE = np.asarray(rows_dE, dtype=np.int64)
    rows_dC = np.asarray(rows_dC, dtype=np.int64)

    # dE rows: full logit row per token; the tile filter needs the Bn rows of
    # the token's tile block, so evaluate the whole block when filtering.
    out_dE = np.zeros((rows_dE.shape[0], E64.shape[1]), dtype=np.float64)
    if filter_eps > 0.0:
        # the token blocks holding requested rows, a few at a time (one matrix
        # product per group); each block's tile mask is its own
        blocks = sorted({int(i) // Bn for i in rows_dE})
        per = max(1, 64 // Bn)
        for g0 in range(0, len(blocks), per):
            grp = blocks[g0:g0 + per]
            spans = [(b * Bn, min(N, (b + 1) * Bn)) for b in grp]
            rows_all = np.concatenate([np.arange(b0, b1) for b0, b1 in spans])
            z = logits(E64[rows_all], C64)
            _, Dm, G = softmax_grad_f64(z, lse_all[rows_all], y[rows_all], dloss[rows_all], ignore_index)
            pos = 0
            for b0, b1 in spans:
                n = b1 - b0
                live = tile_live_map_f64(Dm[pos:pos + n], b0, Bn, Bv, filter_eps)
                mask = np.repeat(live[0], Bv)[:V]
                for k in np.nonzero((rows_dE >= b0) & (rows_dE < b1))[0]:
                    out_dE[k] = np.where(mask, G[pos + int(rows_dE[k]) - b0], 0.0) @ C64
                pos += n
    else:
        # the requested rows, a few at a time (one matrix product per group)
        for k0 in range(0, rows_dE.shape[0], 64):
            sel = rows_dE[k0:k0 + 64]
            z = logits(E64[sel], C64)
            _, _, G = softmax_grad_f64(z, lse_all[sel], y[sel], dloss[sel], ignore_index)
            out_dE[k0:k0 + sel.shape[0]] = G @ C64

    # dC rows: the column v of G over all tokens.  With filtering, the column
    # tile of v must be evaluated in full for each token block.
    out_dC = np.zeros((rows_dC.shape[0], E64.shape[1]), dtype=np.float64)
    if rows_dC.shape[0]:
        tiles = sorted({int(v) // Bv for v in rows_dC}) if filter_eps > 0.0 else None
        rb = max(Bn, (_rows_per_block(V) // Bn) * Bn)
        for r0 in range(0, N, rb):
            r1 = min(N, r0 + rb)
            if filter_eps > 0.0:
                cols = np.concatenate([np.arange(t * Bv, min(V, (t + 1) * Bv)) for t in tiles])
            else:
                cols = rows_dC
            zc = E64[r0:r1] @ C64[cols].T
            P = np.exp(zc - lse_all[r0:r1, None])
            Dm = P.copy()
            yy = y[r0:r1]
            for k in range(r1 - r0):
                t = int(yy[k])
                if t == ignore_index:
                    Dm[k, :] = 0.0
                else:
                    hit = np.nonzero(cols == t)[0]
                    if hit.size:
                        Dm[k, hit[0]] -= 1.0
            if filter_eps > 0.0 and Bn == 1 and Bv == 1:
                Dm = np.where(np.abs(Dm) >= filter_eps, Dm, 0.0)   # element by element
            elif filter_eps > 0.0:
                A = np.abs(Dm)
                pos = 0
                for t in tiles:
                    w = min(V, (t + 1) * Bv) - t * Bv
                    for a0 in range(r0, r1, Bn):
                        a1 = min(r1, a0 + Bn)
                        blk = A[a0 - r0:a1 - r0, pos:pos + w]
                        if not (blk >= filter_eps).any():
                            Dm[a0 - r0:a1 - r0, pos:pos + w] = 0.0
                    pos += w
            if filter_eps > 0.0:
                colpos = {int(c): j for j, c in enumerate(cols)}
                take = np.array([colpos[int(v)] for v in rows_dC])
                Dsel = Dm[:, take]
            else:
                Dsel = Dm
            G = Dsel * dloss[r0:r1].astype(np.float64)[:, None]
            out_dC += G.T @ E64[r0:r1]
    return out_dE, out_dC


def tile_live_map(E_bits, C_bits, y, lse, ignore_index: int, filter_eps: float,
                  tile=(32, 32)):
    """Tile live map (N/Bn x V/Bv, ceil) for bf16 inputs and the given lse."""
    E64 = bf16_bits_to_f64(E_bits)
    C64 = bf16_bits_to_f64(C_bits)
    N, V = E64.shape[0], C64.shape[0]
    Bn, Bv = tile
    rb = max(Bn, (_rows_per_block(V) // Bn) * Bn)
    lse = np.asarray(lse, dtype=np.float64)
    ones = np.ones(N, dtype=np.float32)
    out = []
    for r0 in range(0, N, rb):
        r1 = min(N, r0 + rb)
        z = logits(E64[r0:r1], C64)
        _, Dm, _ = softmax_grad_f64(z, lse[r0:r1], y[r0:r1], ones[r0:r1], ignore_index)
        out.append(tile_live_map_f64(Dm, r0, Bn, Bv, filter_eps))
    return np.concatenate(out, axis=0)
