"""The C-ABI library loads and exports every symbol its headers declare;
host-side argument validation returns the documented codes without a GPU."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        with open(h) as f:
            src = f.read()
        names |= set(re.findall(r"CCE_API\s+[\w\s\*]+?\b(cce_\w+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from linear_cross_entropy_05_b200 import build, _native
    build.build()
    return _native.load_library()


def test_headers_declare_the_boundary():
    names = _declared_symbols()
    for n in ("cce_forward", "cce_backward", "cce_forward_workspace_size", "cce_backward_workspace_size",
              "cce_read_status", "cce_status_string", "cce_version"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared_symbols() if not hasattr(lib, n)]
    assert not missing, missing


def test_library_exports_nothing_else(lib):
    from linear_cross_entropy_05_b200 import _native
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _native.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert exported == set(_declared_symbols())


def test_status_strings(lib):
    from linear_cross_entropy_05_b200 import cce_status_string
    assert cce_status_string(0) == "CCE_OK"
    assert cce_status_string(3) == "CCE_ERR_WORKSPACE_TOO_SMALL"
    assert cce_status_string(7) == "CCE_ERR_BAD_LABEL"
    assert cce_status_string(99) == "CCE_ERR_UNKNOWN"


def test_version(lib):
    from linear_cross_entropy_05_b200 import cce_version
    assert cce_version() >= 100


def _cpu_only():
    try:
        import torch
        if torch.cuda.is_available():
            pytest.skip("validation-with-fake-pointers cases only run where no GPU could be touched")
    except ImportError:
        pass


def test_forward_argument_errors_are_reported_on_the_host(lib):
    _cpu_only()
    from linear_cross_entropy_05_b200 import cce_forward
    P = 1 << 20  # a non-null, 256-aligned fake address: never dereferenced by these cases
    ok = dict(E=P, C=P, y=P, N=256, D=256, V=4096, ignore_index=-100, loss=P, lse=P, workspace=P,
              workspace_bytes=1 << 20, stream=0)

    def call(**kw):
        a = dict(ok)
        a.update(kw)
        return cce_forward(a["E"], a["C"], a["y"], a["N"], a["D"], a["V"], a["ignore_index"], a["loss"], a["lse"],
                           a["workspace"], a["workspace_bytes"], a["stream"], check=False)

    assert call(E=0) == 1
    assert call(workspace=0) == 1
    assert call(N=0) == 1
    assert call(V=-5) == 1
    assert call(D=260) == 1          # D % 8 != 0
    assert call(N=1 << 40) == 1      # does not fit int32
    assert call(E=P + 8) == 2        # bf16 matrices need 16-byte alignment
    assert call(workspace=P + 64) == 2
    assert call() == 4               # valid arguments, but no sm_100 device here


def test_backward_argument_errors_are_reported_on_the_host(lib):
    _cpu_only()
    from linear_cross_entropy_05_b200 import cce_backward
    P = 1 << 20
    base = [P, P, P, P, P, 256, 256, 4096, -100, 0.0, P, P, P, 1 << 20, 0]

    def call(i=None, v=None):
        a = list(base)
        if i is not None:
            a[i] = v
        return cce_backward(*a, check=False)

    assert call(3, 0) == 1                 # lse null
    assert call(7, 0) == 1                 # V = 0
    assert call(6, 12) == 1                # D % 8
    assert call(9, float("nan")) == 1      # NaN filter threshold
    assert call(10, P + 4) == 2            # dE not 16-byte aligned
    assert call() == 4


def test_workspace_size_without_device_is_zero(lib):
    _cpu_only()
    from linear_cross_entropy_05_b200 import cce_backward_workspace_size, cce_forward_workspace_size
    assert cce_forward_workspace_size(8192, 2304, 256000) == 0
    assert cce_forward_workspace_size(0, 8, 8) == 0
    # status 256 + header 256 + one bit per vocabulary row + 2 x [N/128] i32 + N f32
    # (token norms) + N f32 (the tokens' maximum logits), each rounded to 256 bytes
    up = lambda x: (x + 255) // 256 * 256
    for N, V in ((8192, 256000), (300, 4173), (65536, 262144)):
        want = 512 + up(4 * (-(-V // 32))) + 2 * up(4 * (-(-N // 128))) + 2 * up(4 * N)
        assert cce_backward_workspace_size(N, 2304, V) == want
    assert cce_backward_workspace_size(8192, 2305, 256000) == 0


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    from linear_cross_entropy_05_b200 import _native
    monkeypatch.setattr(_native, "_lib", None)
    monkeypatch.setattr(_native, "LIB_PATH", str(tmp_path / "libcce.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        _native.load_library()


def test_backward_ex_workspace_and_flags(lib):
    _cpu_only()
    from linear_cross_entropy_05_b200 import (cce_backward_ex, cce_backward_workspace_size,
                                              cce_backward_workspace_size_ex)
    up = lambda x: (x + 255) // 256 * 256
    N, D, V = 8192, 2304, 256000
    base = cce_backward_workspace_size(N, D, V)
    assert cce_backward_workspace_size_ex(N, D, V, 0) == base
    for flags in (1, 2, 3, 5, 6, 7):   # deterministic / bf16 outputs: int64 accumulators for dE and dC
        assert cce_backward_workspace_size_ex(N, D, V, flags) == base + up(8 * N * D) + up(8 * V * D)
    assert cce_backward_workspace_size_ex(N, D, V, 4) == base   # accumulate alone: no extra workspace
    assert cce_backward_workspace_size_ex(N, D, V, 8) == base   # prepared: no extra workspace
    # stripes: counters + three bf16 stripe buffers of 8192 tokens x 4096 columns
    n_vt, n_s, n_dc = -(-V // 256), -(-V // 4096), -(-D // 256)
    # task counters (u32) and one byte per G tile of every stripe (nonzero flags)
    ctr = up(8 + 4 * (n_vt + n_s * 32 + n_s + 32 * n_dc) + n_s * 32 * 16)
    assert cce_backward_workspace_size_ex(N, D, V, 16) == base + ctr + up(3 * 8192 * 4096 * 2)
    # deterministic with stripes: fixed stripe order, no int64 accumulators
    assert cce_backward_workspace_size_ex(N, D, V, 17) == base + ctr + up(3 * 8192 * 4096 * 2)
    # bf16 outputs through stripes: fp32 dE / dC scratch, rounded once
    assert cce_backward_workspace_size_ex(N, D, V, 18) == base + up(4 * N * D) + up(4 * V * D) + ctr + \
        up(3 * 8192 * 4096 * 2)
    # token super-blocks of 16384 bound the stripe buffers whatever N
    big = cce_backward_workspace_size_ex(65536, 2048, 262144, 16) - cce_backward_workspace_size(65536, 2048, 262144)
    assert big < 3 * 16384 * 4096 * 2 + (1 << 20)
    assert cce_backward_workspace_size_ex(N, D, V, 32) == base  # row maxima: no extra workspace
    assert cce_backward_workspace_size_ex(N, D, V, 64) == 0     # unknown flag
    P = 1 << 20
    args = [P, P, P, P, P, 256, 256, 4096, -100, 0.0, 0, P, P, P, 1 << 30, 0]
    args[10] = 64
    assert cce_backward_ex(*args, check=False) == 1          # unknown flag: rejected on the host
    for flags in (3, 4, 7, 8, 15, 16, 17, 21, 32, 40):
        args[10] = flags
        assert cce_backward_ex(*args, check=False) == 4      # valid, but no device here


def test_backward_prepare_validates_on_the_host(lib):
    _cpu_only()
    from linear_cross_entropy_05_b200 import cce_backward_prepare
    P = 1 << 20
    assert cce_backward_prepare(0, 256, 256, 4096, P, 1 << 30, 0, check=False) == 1        # null C
    assert cce_backward_prepare(P, 256, 260, 4096, P, 1 << 30, 0, check=False) == 1        # D % 8 != 0
    assert cce_backward_prepare(P + 8, 256, 256, 4096, P, 1 << 30, 0, check=False) == 2    # misaligned C
    assert cce_backward_prepare(P, 256, 256, 4096, P, 1 << 30, 0, check=False) == 4        # valid, no device


def test_shard_entry_points_validate_on_the_host(lib):
    _cpu_only()
    from linear_cross_entropy_05_b200 import cce_backward_shard, cce_forward_shard, cce_merge_shards
    P = 1 << 20
    assert cce_forward_shard(P, P, P, 256, 256, 4096, 0, -100, 0, P, 1 << 20, 0, check=False) == 1   # no stats
    assert cce_forward_shard(P, P, P, 256, 256, 4096, -1, -100, P, P, 1 << 20, 0, check=False) == 1  # offset < 0
    assert cce_forward_shard(P, P, P, 256, 256, 4096, 4096, -100, P, P, 1 << 20, 0, check=False) == 4
    assert cce_merge_shards(P, 0, 256, P, 8192, -100, P, P, 0, check=False) == 1                      # R = 0
    assert cce_merge_shards(P, 2, 256, P + 4, 8192, -100, P, P, 0, check=False) == 2                  # y misaligned
    assert cce_merge_shards(P, 2, 256, P, 8192, -100, P, P, 0, check=False) == 4
    assert cce_backward_shard(P, P, P, P, P, 256, 256, 4096, -5, -100, 0.0, P, P, P, 1 << 20, 0,
                              check=False) == 1


def test_forward_order_knob_validates_on_the_host(lib):
    import ctypes
    assert lib.cce_debug_l2_halves(None, 4) == -1
    assert lib.cce_debug_l2_halves((ctypes.c_int * 4)(), 0) == -1
    assert lib.cce_debug_set_forward_order(-1) == 1
    assert lib.cce_debug_set_forward_order(2) == 1
    assert lib.cce_debug_set_forward_order(1) == 0
    assert lib.cce_debug_set_forward_order(0) == 0


def test_forward_schedule_knob_validates_on_the_host(lib):
    assert lib.cce_debug_set_forward_schedule(257, 0, 0, 0) == 1      # more than 256 splits
    assert lib.cce_debug_set_forward_schedule(0, -1, 0, 0) == 1
    assert lib.cce_debug_set_forward_schedule(0, 0, 4, 0) == 1        # hint bits beyond E and C
    assert lib.cce_debug_set_forward_schedule(0, 0, 0, 8) == 1        # 8 stages do not fit
    assert lib.cce_debug_set_forward_schedule(37, 8, 3, 7) == 0
    assert lib.cce_debug_set_forward_schedule(0, 0, 0, 0) == 0        # back to the defaults


def test_stripe_knob_validates_on_the_host(lib):
    assert lib.cce_debug_set_stripe_params(100, 0, 0) == 1          # not a multiple of 256
    assert lib.cce_debug_set_stripe_params(0, 2, 0) == 1
    assert lib.cce_debug_set_stripe_params(0, 0, 33) == 1           # wider than 32 tiles
    assert lib.cce_debug_set_stripe_params(4096, 1, 16) == 0
    assert lib.cce_debug_set_stripe_params(0, 0, 0) == 0            # back to the defaults


def test_row_max_entry_points_validate_on_the_host(lib):
    _cpu_only()
    from linear_cross_entropy_05_b200 import cce_backward_prepare_rows, cce_forward_ex
    P = 1 << 20
    assert cce_backward_prepare_rows(0, 4096, 256, 8192, P, 1 << 30, 0, check=False) == 1     # no row maxima
    assert cce_backward_prepare_rows(P + 2, 4096, 256, 8192, P, 1 << 30, 0, check=False) == 2  # misaligned
    assert cce_backward_prepare_rows(P, 4096, 255, 8192, P, 1 << 30, 0, check=False) == 1     # D % 8 != 0
    assert cce_backward_prepare_rows(P, 4096, 256, 8192, P, 16, 0, check=False) == 3          # workspace too small
    # the forward with row maxima validates like cce_forward (no device here)
    assert cce_forward_ex(P, P, P, 4096, 256, 8192, -100, P, P, P + 2, P, 1 << 30, 0, check=False) == 2
    assert cce_forward_ex(0, P, P, 4096, 256, 8192, -100, P, P, P, P, 1 << 30, 0, check=False) == 1
