"""Cut Cross-Entropy for B200 (sm_100a): Python binding of libcce.so.

The binding only marshals arguments; every step of the loss and its gradient
runs in the library's CUDA kernels (see include/cce.h).  The native library is
loaded on first use; a missing or unloadable library raises immediately, and
there is no CPU fallback.

Low-level entry points carry the C names and take raw device pointers
(Python ints):  cce_forward, cce_forward_noalloc, cce_backward, cce_forward_workspace_size,
cce_backward_workspace_size, cce_read_status, cce_status_string, cce_version,
cce_debug_forward_logits, cce_debug_set_wait_limit_ns, cce_debug_set_kernel_events.

Tensor helpers (torch supplies device memory and the current stream):
forward(E, C, y) -> (loss, lse), backward(E, C, y, lse, dloss, filter_eps)
-> (dE, dC), and linear_cross_entropy(E, C, y) for a mean-reduced loss with
autograd.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

from . import _native
from ._native import (CCE_BWD_ACCUMULATE, CCE_BWD_BF16_GRADS, CCE_BWD_DETERMINISTIC, CCE_BWD_PREPARED,
                      CCE_BWD_STRIPES, CCE_BWD_ROW_MAX, CCEError, cce_forward_ex, cce_backward_prepare_rows, cce_debug_stripe_schedule, cce_debug_set_reduce_prefetch,
                      cce_debug_set_stripe_params, cce_debug_set_l2_hints, cce_debug_set_forward_schedule,
                      cce_debug_set_forward_order, cce_debug_l2_halves, cce_debug_forward_plan,
                      cce_debug_set_stripe_order,
                      cce_backward, cce_backward_ex, cce_backward_prepare,
                      cce_backward_shard, cce_backward_workspace_size, cce_backward_workspace_size_ex,
                      cce_forward_shard, cce_merge_shards, cce_debug_forward_logits,
                      cce_debug_set_backward_trace, cce_debug_set_backward_variant, cce_debug_set_prefetch, cce_debug_set_forward_variant, cce_debug_set_kernel_events, cce_debug_set_wait_limit_ns,
                      cce_debug_withhold_loads, cce_forward, cce_forward_noalloc,
                      cce_forward_workspace_size, cce_read_status,
                      cce_status_string, cce_version, load_library)

IGNORE_INDEX = -100

__all__ = [
    "CCEError", "IGNORE_INDEX", "CCE_BWD_DETERMINISTIC", "CCE_BWD_BF16_GRADS", "CCE_BWD_ACCUMULATE",
    "CCE_BWD_PREPARED", "CCE_BWD_STRIPES", "cce_debug_stripe_schedule", "cce_debug_set_reduce_prefetch",
    "cce_debug_set_stripe_params", "cce_debug_set_l2_hints", "cce_debug_set_forward_schedule",
    "cce_debug_set_forward_order", "cce_debug_l2_halves", "cce_debug_forward_plan",
    "cce_debug_set_stripe_order",
    "cce_backward_prepare",
    "backward_prepare", "cce_forward",
    "cce_forward_noalloc", "cce_backward", "cce_backward_ex", "cce_backward_workspace_size_ex",
    "cce_forward_shard", "cce_merge_shards", "cce_backward_shard", "forward_shard", "merge_shards",
    "backward_shard", "vocab_parallel_forward_backward", "cce_forward_workspace_size",
    "cce_backward_workspace_size", "cce_read_status", "cce_status_string", "cce_version",
    "cce_debug_forward_logits", "cce_debug_set_wait_limit_ns", "cce_debug_set_kernel_events", "cce_debug_withhold_loads", "cce_debug_set_forward_variant",
    "cce_debug_set_backward_variant", "cce_debug_set_backward_trace", "cce_debug_set_prefetch",
    "load_library",
    "forward", "backward", "read_status", "linear_cross_entropy", "Workspace",
    "CCE_BWD_ROW_MAX", "cce_forward_ex", "cce_backward_prepare_rows",
]


def _torch():
    import torch
    return torch


def _check_inputs(E, C, y):
    torch = _torch()
    if E.dtype != torch.bfloat16 or C.dtype != torch.bfloat16:
        raise TypeError("E and C must be torch.bfloat16")
    if y.dtype != torch.int64:
        raise TypeError("y must be torch.int64")
    if not (E.is_cuda and C.is_cuda and y.is_cuda):
        raise ValueError("E, C, y must be CUDA tensors")
    if not (E.is_contiguous() and C.is_contiguous() and y.is_contiguous()):
        raise ValueError("E, C, y must be contiguous")
    if E.dim() != 2 or C.dim() != 2 or E.shape[1] != C.shape[1] or y.shape != (E.shape[0],):
        raise ValueError("shapes must be E [N, D], C [V, D], y [N]")


class Workspace:
    """A caller-owned device scratch buffer (torch uint8), grown on demand."""

    def __init__(self, device=None):
        self.buf = None
        self.device = device

    def get(self, nbytes: int):
        torch = _torch()
        nbytes = max(int(nbytes), 256)
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device or "cuda")
        return self.buf


def _stream_ptr(stream) -> int:
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def forward(E, C, y, ignore_index: int = IGNORE_INDEX, workspace: Optional[Workspace] = None,
            stream=None, out=None, row_max=None) -> Tuple["object", "object"]:
    """Per-token loss and log-sum-exp (fp32 tensors of shape [N]).  row_max:
    an optional fp32 tensor [N] that receives each token's largest logit
    (cce_forward_ex), for backward(..., row_max=...)."""
    torch = _torch()
    _check_inputs(E, C, y)
    N, D = E.shape
    V = C.shape[0]
    if out is None:
        loss = torch.empty(N, dtype=torch.float32, device=E.device)
        lse = torch.empty(N, dtype=torch.float32, device=E.device)
    else:
        loss, lse = out
    ws_bytes = cce_forward_workspace_size(N, D, V)
    if ws_bytes == 0:
        raise CCEError(1, "cce_forward_workspace_size: invalid sizes or no sm_100 device")
    ws = (workspace or Workspace(E.device)).get(ws_bytes)
    if row_max is not None:
        if row_max.dtype != torch.float32 or not row_max.is_cuda or not row_max.is_contiguous() or \
                row_max.shape != (N,):
            raise ValueError("row_max must be a contiguous CUDA float32 tensor of shape [N]")
        cce_forward_ex(E.data_ptr(), C.data_ptr(), y.data_ptr(), N, D, V, ignore_index, loss.data_ptr(),
                       lse.data_ptr(), row_max.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(stream))
    else:
        cce_forward(E.data_ptr(), C.data_ptr(), y.data_ptr(), N, D, V, ignore_index, loss.data_ptr(),
                    lse.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(stream))
    return loss, lse


def backward_prepare(C, N: int, workspace: Workspace, deterministic: bool = False, bf16_grads: bool = False,
                     stream=None):
    """The classifier-only part of the backward's pre-pass (max_v |C_v|) into
    `workspace`, sized for the backward call that will use it; that call then
    passes prepared=True.  Can run on another stream while the forward runs."""
    torch = _torch()
    if C.dtype != torch.bfloat16 or not C.is_cuda or not C.is_contiguous() or C.dim() != 2:
        raise ValueError("C must be a contiguous CUDA bfloat16 tensor [V, D]")
    V, D = C.shape
    flags = (CCE_BWD_DETERMINISTIC if deterministic else 0) | (CCE_BWD_BF16_GRADS if bf16_grads else 0)
    ws = workspace.get(cce_backward_workspace_size_ex(N, D, V, flags))
    cce_backward_prepare(C.data_ptr(), N, D, V, ws.data_ptr(), ws.numel(), _stream_ptr(stream))


def backward(E, C, y, lse, dloss, filter_eps: float = 0.0, ignore_index: int = IGNORE_INDEX,
             workspace: Optional[Workspace] = None, stream=None, out=None, deterministic: bool = False,
             bf16_grads: bool = False, accumulate: bool = False, prepared: bool = False,
             stripes: Optional[bool] = None, row_max=None):
    """dE [N, D] and dC [V, D] of sum_i dloss[i] * loss[i]: fp32, or bf16 with
    bf16_grads; deterministic=True gives bitwise reproducible gradients
    (fixed-point accumulation, extra (N + V) * D * 8 bytes of workspace).
    accumulate=True adds them to the tensors given in `out` (required)
    instead of overwriting them.  prepared=True: backward_prepare already ran
    on `workspace` for this C.  stripes (default: on when filter_eps <= 0):
    the backward through softmax-gradient stripes
    (CCE_BWD_STRIPES), which needs a larger workspace (about 24 KB per
    token, at most ~400 MB); with deterministic=True it sums in a fixed
    order instead of using the int64 fixed-point accumulators.  With
    filter_eps > 0 it applies the same entry filter but skips no work: the
    faster choice only when a large share of the gradient is above the
    threshold (a peaky, non-flat softmax).  row_max: the tokens' largest
    logits from forward(..., row_max=...) on the same E and C; with the
    filter on they replace the Cauchy-Schwarz bound in the pre-pass
    (CCE_BWD_ROW_MAX), which finds more token blocks flat."""
    torch = _torch()
    _check_inputs(E, C, y)
    N, D = E.shape
    V = C.shape[0]
    for t, n in ((lse, "lse"), (dloss, "dloss")):
        if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or t.shape != (N,):
            raise ValueError(f"{n} must be a contiguous CUDA float32 tensor of shape [N]")
    flags = ((CCE_BWD_DETERMINISTIC if deterministic else 0) | (CCE_BWD_BF16_GRADS if bf16_grads else 0) |
             (CCE_BWD_ACCUMULATE if accumulate else 0) | (CCE_BWD_PREPARED if prepared else 0))
    if stripes is None:
        stripes = filter_eps <= 0
    if stripes:
        flags |= CCE_BWD_STRIPES
    use_rows = row_max is not None and filter_eps > 0 and not stripes
    if use_rows:
        if row_max.dtype != torch.float32 or not row_max.is_cuda or not row_max.is_contiguous() or \
                row_max.shape != (N,):
            raise ValueError("row_max must be a contiguous CUDA float32 tensor of shape [N]")
        flags |= CCE_BWD_ROW_MAX
    if prepared and workspace is None:
        raise ValueError("prepared=True needs the workspace that backward_prepare filled")
    if accumulate and out is None:
        raise ValueError("accumulate=True adds into existing gradients: pass them as out=(dE, dC)")
    gdt = torch.bfloat16 if bf16_grads else torch.float32
    if out is None:
        dE = torch.empty((N, D), dtype=gdt, device=E.device)
        dC = torch.empty((V, D), dtype=gdt, device=E.device)
    else:
        dE, dC = out
        if dE.dtype != gdt or dC.dtype != gdt:
            raise TypeError(f"dE and dC must be {gdt}")
    ws_bytes = cce_backward_workspace_size_ex(N, D, V, flags)
    if prepared and (workspace.buf is None or workspace.buf.numel() < ws_bytes):
        raise ValueError("prepared=True: the workspace backward_prepare filled is smaller than this call needs")
    ws = (workspace or Workspace(E.device)).get(ws_bytes)
    if use_rows:
        cce_backward_prepare_rows(row_max.data_ptr(), N, D, V, ws.data_ptr(), ws.numel(), _stream_ptr(stream))
    cce_backward_ex(E.data_ptr(), C.data_ptr(), y.data_ptr(), lse.data_ptr(), dloss.data_ptr(), N, D, V,
                    ignore_index, float(filter_eps), flags, dE.data_ptr(), dC.data_ptr(), ws.data_ptr(), ws.numel(),
                    _stream_ptr(stream))
    return dE, dC


def read_status(workspace: Workspace, stream=None, raise_on_flag: bool = False) -> dict:
    """Synchronise the stream and decode the workspace's status block."""
    st, c = cce_read_status(workspace.buf.data_ptr(), _stream_ptr(stream))
    if raise_on_flag and st != 0:
        raise CCEError(st, cce_status_string(st))
    return {"status": st, "flags": c[0], "live_tiles": c[1], "dead_tiles": c[2], "logit_tiles": c[3],
            "pruned_tiles": c[4], "flat_units": c[5]}


def linear_cross_entropy(E, C, y, ignore_index: int = IGNORE_INDEX, filter_eps: float = 2.0 ** -12):
    """Mean cross-entropy over non-ignored tokens of the logits E C^T, with
    autograd support; the N x V logits are never materialised."""
    from ._autograd import LinearCrossEntropy
    return LinearCrossEntropy.apply(E, C, y, ignore_index, filter_eps)


# ---------------------------------------------------------------------------
# vocabulary-parallel form (one classifier shard per rank)
# ---------------------------------------------------------------------------

def forward_shard(E, C_shard, y, v_offset: int, ignore_index: int = IGNORE_INDEX,
                  workspace: Optional[Workspace] = None, stream=None):
    """Per-token (max, sum exp, target logit or 0) over the shard C_shard =
    C[v_offset : v_offset + V_shard]: a float32 tensor [3, N]."""
    torch = _torch()
    _check_inputs(E, C_shard, y)
    N, D = E.shape
    V = C_shard.shape[0]
    stats = torch.empty((3, N), dtype=torch.float32, device=E.device)
    ws = (workspace or Workspace(E.device)).get(cce_forward_workspace_size(N, D, V))
    cce_forward_shard(E.data_ptr(), C_shard.data_ptr(), y.data_ptr(), N, D, V, int(v_offset), ignore_index,
                      stats.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(stream))
    return stats


def merge_shards(stats, y, V_total: int, ignore_index: int = IGNORE_INDEX, stream=None):
    """stats [R, 3, N] (all shards) -> (loss, lse), fp32 [N]."""
    torch = _torch()
    stats = stats.contiguous()
    R, three, N = stats.shape
    if three != 3 or y.shape != (N,):
        raise ValueError("stats must be [R, 3, N] and y [N]")
    loss = torch.empty(N, dtype=torch.float32, device=stats.device)
    lse = torch.empty(N, dtype=torch.float32, device=stats.device)
    cce_merge_shards(stats.data_ptr(), R, N, y.data_ptr(), int(V_total), ignore_index, loss.data_ptr(),
                     lse.data_ptr(), _stream_ptr(stream))
    return loss, lse


def backward_shard(E, C_shard, y, lse, dloss, v_offset: int, filter_eps: float = 0.0,
                   ignore_index: int = IGNORE_INDEX, workspace: Optional[Workspace] = None, stream=None):
    """(dE share, dC_shard) for one shard given the merged lse."""
    torch = _torch()
    _check_inputs(E, C_shard, y)
    N, D = E.shape
    V = C_shard.shape[0]
    dE = torch.empty((N, D), dtype=torch.float32, device=E.device)
    dC = torch.empty((V, D), dtype=torch.float32, device=E.device)
    ws = (workspace or Workspace(E.device)).get(cce_backward_workspace_size(N, D, V))
    cce_backward_shard(E.data_ptr(), C_shard.data_ptr(), y.data_ptr(), lse.data_ptr(), dloss.data_ptr(), N, D, V,
                       int(v_offset), ignore_index, float(filter_eps), dE.data_ptr(), dC.data_ptr(), ws.data_ptr(),
                       ws.numel(), _stream_ptr(stream))
    return dE, dC


def vocab_parallel_forward_backward(E, C_shard, y, v_offset: int, V_total: int, dloss=None,
                                    filter_eps: float = 2.0 ** -12, ignore_index: int = IGNORE_INDEX, group=None):
    """One vocabulary-parallel step on this rank's classifier shard.

    Collectives (torch.distributed, NCCL on GPUs): an all-gather of the
    [3, N] shard statistics (12 bytes per token per rank) and an all-reduce
    of the dE shares.  Returns (loss, lse, dE, dC_shard); loss, lse and dE
    are identical on every rank.  dloss defaults to the mean over kept
    tokens.  Without an initialised process group this is the single-shard
    case.
    """
    torch = _torch()
    import torch.distributed as dist
    stats = forward_shard(E, C_shard, y, v_offset, ignore_index)
    if dist.is_available() and dist.is_initialized():
        world = dist.get_world_size(group)
        gathered = [torch.empty_like(stats) for _ in range(world)]
        dist.all_gather(gathered, stats, group=group)
        all_stats = torch.stack(gathered)
    else:
        all_stats = stats[None]
    loss, lse = merge_shards(all_stats, y, V_total, ignore_index)
    if dloss is None:
        keep = (y != ignore_index).to(torch.float32)
        dloss = keep / keep.sum().clamp_min(1.0)
    dE, dC = backward_shard(E, C_shard, y, lse, dloss.contiguous(), v_offset, filter_eps, ignore_index)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(dE, group=group)
    return loss, lse, dE, dC
