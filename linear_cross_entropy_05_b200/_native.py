"""ctypes declarations of libcce.so (include/cce.h, include/cce_debug.h)."""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcce.so")

_lib = None
_lock = threading.Lock()

c_i64 = ctypes.c_int64
c_vp = ctypes.c_void_p
c_size = ctypes.c_size_t
c_f32 = ctypes.c_float


class CCECounters(ctypes.Structure):
    _fields_ = [("flags", ctypes.c_uint64), ("live_tiles", ctypes.c_uint64),
                ("dead_tiles", ctypes.c_uint64), ("logit_tiles", ctypes.c_uint64),
                ("pruned_tiles", ctypes.c_uint64), ("flat_units", ctypes.c_uint64)]


class CCEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{msg} (status {status})")
        self.status = status


def load_library():
    """Load libcce.so from the package directory; raise if it is missing."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m linear_cross_entropy_05_b200.build` "
                "(there is no CPU fallback)")
        lib = ctypes.CDLL(LIB_PATH)
        lib.cce_forward_workspace_size.argtypes = [c_i64, c_i64, c_i64]
        lib.cce_forward_workspace_size.restype = c_size
        lib.cce_backward_workspace_size.argtypes = [c_i64, c_i64, c_i64]
        lib.cce_backward_workspace_size.restype = c_size
        lib.cce_forward.argtypes = [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_vp, c_vp, c_vp, c_size, c_vp]
        lib.cce_forward.restype = ctypes.c_int
        lib.cce_backward.argtypes = [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_f32, c_vp, c_vp,
                                     c_vp, c_size, c_vp]
        lib.cce_backward.restype = ctypes.c_int
        lib.cce_backward_workspace_size_ex.argtypes = [c_i64, c_i64, c_i64, ctypes.c_uint]
        lib.cce_backward_workspace_size_ex.restype = c_size
        lib.cce_backward_ex.argtypes = [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_f32, ctypes.c_uint,
                                        c_vp, c_vp, c_vp, c_size, c_vp]
        lib.cce_backward_ex.restype = ctypes.c_int
        lib.cce_backward_prepare.argtypes = [c_vp, c_i64, c_i64, c_i64, c_vp, c_size, c_vp]
        lib.cce_backward_prepare.restype = ctypes.c_int
        lib.cce_backward_prepare_rows.argtypes = [c_vp, c_i64, c_i64, c_i64, c_vp, c_size, c_vp]
        lib.cce_backward_prepare_rows.restype = ctypes.c_int
        lib.cce_forward_ex.argtypes = [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_vp, c_vp, c_vp, c_vp, c_size,
                                       c_vp]
        lib.cce_forward_ex.restype = ctypes.c_int
        lib.cce_forward_shard.argtypes = [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_i64, c_vp, c_vp, c_size,
                                          c_vp]
        lib.cce_forward_shard.restype = ctypes.c_int
        lib.cce_merge_shards.argtypes = [c_vp, ctypes.c_int, c_i64, c_vp, c_i64, c_i64, c_vp, c_vp, c_vp]
        lib.cce_merge_shards.restype = ctypes.c_int
        lib.cce_backward_shard.argtypes = [c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_i64, c_f32,
                                           c_vp, c_vp, c_vp, c_size, c_vp]
        lib.cce_backward_shard.restype = ctypes.c_int
        lib.cce_read_status.argtypes = [c_vp, c_vp, ctypes.POINTER(CCECounters)]
        lib.cce_read_status.restype = ctypes.c_int
        lib.cce_status_string.argtypes = [ctypes.c_int]
        lib.cce_status_string.restype = ctypes.c_char_p
        lib.cce_version.argtypes = []
        lib.cce_version.restype = ctypes.c_int
        lib.cce_debug_forward_logits.argtypes = [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_vp, c_vp, c_vp,
                                                 c_vp, c_size, c_vp]
        lib.cce_debug_forward_logits.restype = ctypes.c_int
        lib.cce_debug_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        lib.cce_debug_set_wait_limit_ns.restype = None
        lib.cce_forward_noalloc.argtypes = [c_vp, c_vp, c_vp, c_i64, c_i64, c_i64, c_i64, c_vp, c_vp, c_vp]
        lib.cce_forward_noalloc.restype = ctypes.c_int
        lib.cce_debug_set_forward_variant.argtypes = [ctypes.c_int]
        lib.cce_debug_set_forward_variant.restype = ctypes.c_int
        lib.cce_debug_set_backward_variant.argtypes = [ctypes.c_int]
        lib.cce_debug_set_backward_variant.restype = ctypes.c_int
        lib.cce_debug_withhold_loads.argtypes = [ctypes.c_int]
        lib.cce_debug_withhold_loads.restype = None
        lib.cce_debug_set_kernel_events.argtypes = [ctypes.c_int, c_vp, c_vp]
        lib.cce_debug_set_kernel_events.restype = ctypes.c_int
        lib.cce_debug_set_prefetch.argtypes = [ctypes.c_int, ctypes.c_int]
        lib.cce_debug_set_prefetch.restype = ctypes.c_int
        lib.cce_debug_set_stripe_params.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.cce_debug_set_stripe_params.restype = ctypes.c_int
        lib.cce_debug_set_l2_hints.argtypes = [ctypes.c_int]
        lib.cce_debug_set_l2_hints.restype = ctypes.c_int
        lib.cce_debug_set_forward_schedule.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.cce_debug_set_forward_schedule.restype = ctypes.c_int
        lib.cce_debug_set_forward_order.argtypes = [ctypes.c_int]
        lib.cce_debug_set_forward_order.restype = ctypes.c_int
        lib.cce_debug_l2_halves.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.c_int]
        lib.cce_debug_l2_halves.restype = ctypes.c_int
        lib.cce_debug_forward_plan.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                               ctypes.POINTER(ctypes.c_int)]
        lib.cce_debug_forward_plan.restype = ctypes.c_int
        lib.cce_debug_set_reduce_prefetch.argtypes = [ctypes.c_int]
        lib.cce_debug_set_reduce_prefetch.restype = ctypes.c_int
        lib.cce_debug_stripe_schedule.argtypes = [ctypes.c_int] * 8 + [c_vp, c_i64]
        lib.cce_debug_stripe_schedule.restype = c_i64
        lib.cce_debug_set_stripe_order.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.cce_debug_set_stripe_order.restype = ctypes.c_int
        lib.cce_debug_set_backward_trace.argtypes = [c_vp, c_i64]
        lib.cce_debug_set_backward_trace.restype = ctypes.c_int
        _lib = lib
        return lib


def _check(st: int, what: str):
    if st != 0:
        raise CCEError(st, f"{what}: {cce_status_string(st)}")


def cce_status_string(status: int) -> str:
    return load_library().cce_status_string(int(status)).decode()


def cce_version() -> int:
    return load_library().cce_version()


def cce_forward_workspace_size(N: int, D: int, V: int) -> int:
    return int(load_library().cce_forward_workspace_size(N, D, V))


def cce_backward_workspace_size(N: int, D: int, V: int) -> int:
    return int(load_library().cce_backward_workspace_size(N, D, V))


def cce_forward(E: int, C: int, y: int, N: int, D: int, V: int, ignore_index: int, loss: int, lse: int,
                workspace: int, workspace_bytes: int, stream: int, check: bool = True) -> int:
    st = load_library().cce_forward(E, C, y, N, D, V, ignore_index, loss, lse, workspace, workspace_bytes,
                                    stream)
    if check:
        _check(st, "cce_forward")
    return st


def cce_forward_ex(E: int, C: int, y: int, N: int, D: int, V: int, ignore_index: int, loss: int, lse: int,
                   row_max: int, workspace: int, workspace_bytes: int, stream: int, check: bool = True) -> int:
    st = load_library().cce_forward_ex(E, C, y, N, D, V, ignore_index, loss, lse, row_max, workspace,
                                       workspace_bytes, stream)
    if check:
        _check(st, "cce_forward_ex")
    return st


def cce_forward_noalloc(E: int, C: int, y: int, N: int, D: int, V: int, ignore_index: int, loss: int, lse: int,
                        stream: int, check: bool = True) -> int:
    """Forward pass without a workspace, for callers that cannot allocate
    device memory; scratch is a static 8 MiB device array in the library."""
    st = load_library().cce_forward_noalloc(E, C, y, N, D, V, ignore_index, loss, lse, stream)
    if check:
        _check(st, "cce_forward_noalloc")
    return st


def cce_backward(E: int, C: int, y: int, lse: int, dloss: int, N: int, D: int, V: int, ignore_index: int,
                 filter_eps: float, dE: int, dC: int, workspace: int, workspace_bytes: int, stream: int,
                 check: bool = True) -> int:
    st = load_library().cce_backward(E, C, y, lse, dloss, N, D, V, ignore_index, filter_eps, dE, dC, workspace,
                                     workspace_bytes, stream)
    if check:
        _check(st, "cce_backward")
    return st


CCE_BWD_DETERMINISTIC = 1
CCE_BWD_BF16_GRADS = 2
CCE_BWD_ACCUMULATE = 4
CCE_BWD_PREPARED = 8
CCE_BWD_STRIPES = 16
CCE_BWD_ROW_MAX = 32


def cce_backward_prepare_rows(row_max: int, N: int, D: int, V: int, workspace: int, workspace_bytes: int,
                              stream: int, check: bool = True) -> int:
    st = load_library().cce_backward_prepare_rows(row_max, N, D, V, workspace, workspace_bytes, stream)
    if check:
        _check(st, "cce_backward_prepare_rows")
    return st


def cce_backward_prepare(C: int, N: int, D: int, V: int, workspace: int, workspace_bytes: int, stream: int,
                         check: bool = True) -> int:
    st = load_library().cce_backward_prepare(C, N, D, V, workspace, workspace_bytes, stream)
    if check:
        _check(st, "cce_backward_prepare")
    return st


def cce_backward_workspace_size_ex(N: int, D: int, V: int, flags: int) -> int:
    return int(load_library().cce_backward_workspace_size_ex(N, D, V, flags))


def cce_backward_ex(E: int, C: int, y: int, lse: int, dloss: int, N: int, D: int, V: int, ignore_index: int,
                    filter_eps: float, flags: int, dE: int, dC: int, workspace: int, workspace_bytes: int,
                    stream: int, check: bool = True) -> int:
    st = load_library().cce_backward_ex(E, C, y, lse, dloss, N, D, V, ignore_index, filter_eps, flags, dE, dC,
                                        workspace, workspace_bytes, stream)
    if check:
        _check(st, "cce_backward_ex")
    return st


def cce_forward_shard(E: int, C_shard: int, y: int, N: int, D: int, V_shard: int, v_offset: int,
                      ignore_index: int, stats: int, workspace: int, workspace_bytes: int, stream: int,
                      check: bool = True) -> int:
    st = load_library().cce_forward_shard(E, C_shard, y, N, D, V_shard, v_offset, ignore_index, stats, workspace,
                                          workspace_bytes, stream)
    if check:
        _check(st, "cce_forward_shard")
    return st


def cce_merge_shards(stats: int, R: int, N: int, y: int, V_total: int, ignore_index: int, loss: int, lse: int,
                     stream: int, check: bool = True) -> int:
    st = load_library().cce_merge_shards(stats, R, N, y, V_total, ignore_index, loss, lse, stream)
    if check:
        _check(st, "cce_merge_shards")
    return st


def cce_backward_shard(E: int, C_shard: int, y: int, lse: int, dloss: int, N: int, D: int, V_shard: int,
                       v_offset: int, ignore_index: int, filter_eps: float, dE_partial: int, dC_shard: int,
                       workspace: int, workspace_bytes: int, stream: int, check: bool = True) -> int:
    st = load_library().cce_backward_shard(E, C_shard, y, lse, dloss, N, D, V_shard, v_offset, ignore_index,
                                           filter_eps, dE_partial, dC_shard, workspace, workspace_bytes, stream)
    if check:
        _check(st, "cce_backward_shard")
    return st


def cce_read_status(workspace: int, stream: int):
    c = CCECounters()
    st = load_library().cce_read_status(workspace, stream, ctypes.byref(c))
    return st, (c.flags, c.live_tiles, c.dead_tiles, c.logit_tiles, c.pruned_tiles, c.flat_units)


def cce_debug_forward_logits(E: int, C: int, y: int, N: int, D: int, V: int, ignore_index: int, loss: int,
                             lse: int, logits: int, workspace: int, workspace_bytes: int, stream: int,
                             check: bool = True) -> int:
    st = load_library().cce_debug_forward_logits(E, C, y, N, D, V, ignore_index, loss, lse, logits, workspace,
                                                 workspace_bytes, stream)
    if check:
        _check(st, "cce_debug_forward_logits")
    return st


def cce_debug_set_wait_limit_ns(limit_ns: int) -> None:
    load_library().cce_debug_set_wait_limit_ns(int(limit_ns))


def cce_debug_set_kernel_events(kernel: int, start_event: int, stop_event: int) -> None:
    _check(load_library().cce_debug_set_kernel_events(int(kernel), start_event, stop_event),
           "cce_debug_set_kernel_events")


def cce_debug_withhold_loads(on: bool) -> None:
    load_library().cce_debug_withhold_loads(1 if on else 0)


def cce_debug_set_forward_variant(variant: int) -> None:
    """1 = CTA-pair forward kernel (default), 0 = single-CTA forward kernel."""
    _check(load_library().cce_debug_set_forward_variant(int(variant)), "cce_debug_set_forward_variant")


def cce_debug_set_backward_variant(variant: int) -> None:
    """0 = 3 stages / 1 staging buffer (default), 1 = 2 stages / 2 staging buffers,
    2 = 2 stages / eight epilogue warps, 3 = as 0 with load/store-path reductions."""
    _check(load_library().cce_debug_set_backward_variant(int(variant)), "cce_debug_set_backward_variant")


def cce_debug_set_prefetch(fwd_slices: int, bwd_slices: int) -> None:
    """L2 prefetch distances (64-wide K slices) of the forward / backward operand streams; 0 = off."""
    _check(load_library().cce_debug_set_prefetch(int(fwd_slices), int(bwd_slices)), "cce_debug_set_prefetch")


def cce_debug_set_backward_trace(trace: int, tiles_per_cta: int) -> None:
    """Per-tile globaltimer stamps of every backward launch into the device
    buffer `trace` (u64 [SMs][tiles_per_cta][4]); trace = 0 turns it off."""
    _check(load_library().cce_debug_set_backward_trace(trace or None, int(tiles_per_cta)),
           "cce_debug_set_backward_trace")


def cce_debug_stripe_schedule(n_m2: int, n_vtile: int, n_dc: int, vt_per_s: int, nbuf: int, order: int = 0,
                              group_m2: int = 4, lag: int = 2):
    """Task order of the stripe backward (host-side decode, no kernel):
    an int32 array [tasks + 1, 4] of (kind, stripe, a, b); kind -1 ends it."""
    import numpy as np
    lib = load_library()
    total = int(lib.cce_debug_stripe_schedule(n_m2, n_vtile, n_dc, vt_per_s, nbuf, order, group_m2, lag, None, 0))
    if total < 0:
        raise CCEError(1, "cce_debug_stripe_schedule: invalid sizes")
    out = np.zeros((total + 1, 4), dtype=np.int32)
    lib.cce_debug_stripe_schedule(n_m2, n_vtile, n_dc, vt_per_s, nbuf, order, group_m2, lag, out.ctypes.data,
                                  total + 1)
    return out


def cce_debug_set_stripe_order(order: int = 0, group_m2: int = 4, lag: int = 2) -> None:
    """Stripe backward task order (A/B): 0 stripe-major, 1 interleaved with
    groups of group_m2 token blocks and the dE tasks lag groups behind."""
    _check(load_library().cce_debug_set_stripe_order(int(order), int(group_m2), int(lag)),
           "cce_debug_set_stripe_order")


def cce_debug_set_reduce_prefetch(slices: int) -> None:
    """L2 prefetch distance (64-wide K slices) of the filtered backward's
    reduction targets (live dE / dC rows); 0 = off."""
    _check(load_library().cce_debug_set_reduce_prefetch(int(slices)), "cce_debug_set_reduce_prefetch")


def cce_debug_set_stripe_params(tokens_per_launch: int = 0, dE_prefetch: int = 0, vtiles_per_stripe: int = 0) -> None:
    """Stripe backward knobs (A/B): tokens per launch (multiple of 256, <= 16384;
    0 = default), the L2 prefetch of dE rows for dE-tile tasks (0/1) and the
    stripe width in 256-wide vocabulary tiles (0 = default 8, at most 32)."""
    _check(load_library().cce_debug_set_stripe_params(int(tokens_per_launch), int(dE_prefetch),
                                                      int(vtiles_per_stripe)),
           "cce_debug_set_stripe_params")


def cce_debug_set_l2_hints(on: bool) -> None:
    """L2 eviction priorities in the filtered backward (evict-first classifier
    slices, evict-last dE reductions); A/B knob, off by default."""
    _check(load_library().cce_debug_set_l2_hints(1 if on else 0), "cce_debug_set_l2_hints")


def cce_debug_set_forward_schedule(n_split: int = 0, group_m: int = 0, l2_hints: int = 0, stages: int = 0) -> None:
    """Forward schedule knobs (A/B): vocabulary splits per token block, token
    blocks per raster group (0 = chosen per shape), L2 eviction hints of the
    CTA-pair kernel (bit 0: E evict_last, bit 1: C evict_first) and its
    operand stages per CTA (0 = default 7, or 6)."""
    _check(load_library().cce_debug_set_forward_schedule(int(n_split), int(group_m), int(l2_hints), int(stages)),
           "cce_debug_set_forward_schedule")


def cce_debug_forward_plan(N: int, D: int, V: int, sms: int) -> dict:
    """The forward's launch plan for these sizes on a GPU with `sms` SMs
    (host arithmetic; no device needed)."""
    out = (ctypes.c_int * 6)()
    if load_library().cce_debug_forward_plan(int(N), int(D), int(V), int(sms), out) != 0:
        raise ValueError("cce_debug_forward_plan: invalid sizes")
    return dict(pair=bool(out[0]), n_mblk=out[1], n_vtile=out[2], n_split=out[3], group_m=out[4], grid=out[5])


def cce_debug_l2_halves(max_sms: int = 256) -> list:
    """L2 half (1 or 2; 0 unknown) of SM ids 0 .. max_sms-1 on the current
    device, as found by the two-queue forward's probe."""
    buf = (ctypes.c_int * int(max_sms))()
    n = load_library().cce_debug_l2_halves(buf, int(max_sms))
    if n < 0:
        raise RuntimeError("cce_debug_l2_halves failed")
    return list(buf[:n])


def cce_debug_set_forward_order(order: int) -> None:
    """Unit order of the CTA-pair forward (A/B): 0 round-robin, 1 one queue
    per L2 half of the GPU (same results bit for bit)."""
    _check(load_library().cce_debug_set_forward_order(int(order)), "cce_debug_set_forward_order")
