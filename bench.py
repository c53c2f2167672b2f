#!/usr/bin/env python
"""Benchmark of the Cut Cross-Entropy hot path on B200.

One step = cce_forward + cce_backward (gradient filter 2^-12) over one batch
of the Gemma-2-2B-shaped classifier head: N = 8192 tokens, D = 2304,
V = 256000, bf16 E, C ~ N(0, 0.02), Zipf(1.1) labels (synthetic, seeded).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints ONE JSON line on rank 0.  Under torchrun each rank runs an independent
replica of the same problem on its own GPU (the operator runs on one GPU; there
is no data-path collective); timing is the max over ranks.

--impl reference times the fp64 CPU oracle (the plain definition of the loss
and its gradient) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CCE fwd+bwd tokens/s"
UNIT = "tokens/s"
IGN = -100
BM, BN = 128, 256      # logit tile (token block x vocabulary tile)
STRIPE_COLS = 4096     # vocabulary columns per stripe of the dense backward (the library's default)
FU = (32, 32)          # the unit of skipped work: 32 tokens x 32 vocabulary entries (the filter itself
                       # drops single entries)


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------------------
# distributed plumbing (replicas)
# ---------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend: str):
    import torch.distributed as dist
    ws, rank, _ = dist_env()
    if ws > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist if ws > 1 else None


def reduce_max(dist, x: float, device) -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(dist, x: float, device) -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def aggregate_throughput(dist, tokens_local: float, seconds_local: float, device):
    """Whole-job throughput: tokens processed by all ranks / max time over ranks."""
    tmax = reduce_max(dist, seconds_local, device)
    tok = reduce_sum(dist, tokens_local, device)
    return tok / tmax, tmax


def aggregate_shared_batch(dist, tokens: float, seconds_local: float, device):
    """Throughput of one batch processed jointly by all ranks (the
    vocabulary-parallel mode: every rank works on the same tokens, each on
    its classifier shard): tokens / max time over ranks."""
    tmax = reduce_max(dist, seconds_local, device)
    return tokens / tmax, tmax


def vocab_shard(V: int, world: int, rank: int, tile: int = 256):
    """Contiguous classifier shard [v_offset, v_offset + V_shard) of `rank`:
    whole 256-row vocabulary tiles dealt as evenly as possible (the first
    V_tiles % world ranks get one tile more), the ragged last tile with the
    last rank."""
    n_t = -(-V // tile)
    if n_t < world:
        raise ValueError(f"{V} vocabulary rows make {n_t} tiles: fewer than the {world} ranks")
    base, extra = divmod(n_t, world)
    t0 = rank * base + min(rank, extra)
    t1 = t0 + base + (1 if rank < extra else 0)
    v0, v1 = min(V, t0 * tile), min(V, t1 * tile)
    return v0, v1 - v0


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------

class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU sampled during a
    timed region: through NVML every 2 ms when the bindings import (the
    source nvidia-smi reads), else `nvidia-smi -lms 100`.  The GPU is found by
    the PCI bus id of the CUDA device when torch exposes it (the NVML index
    may differ from the CUDA index under CUDA_VISIBLE_DEVICES)."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.002

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.nvml = None
        self.lines = []
        self.samples = []   # (sm MHz, power W, reasons bitmask) from NVML

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            pr = torch.cuda.get_device_properties(self.gpu)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus.upper())
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def start(self):
        try:
            self.nvml = self._nvml_handle()
        except Exception as e:
            log("NVML unavailable, sampling with nvidia-smi:", e)
            self.nvml = None
        if self.nvml is not None:
            self.stop_flag = False
            self.thread = threading.Thread(target=self._poll_nvml, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception as e:  # nvidia-smi missing
            log("clock sampler unavailable:", e)
            self.proc = None

    def _poll_nvml(self):
        nv, h = self.nvml
        while not self.stop_flag:
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except Exception:
                pass
            time.sleep(self.PERIOD_S)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def _stop_nvml(self):
        nv, h = self.nvml
        self.stop_flag = True
        self.thread.join(timeout=2)
        try:
            smax = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        except Exception:
            smax = None
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "hw_power_brake_slowdown": nv.nvmlClocksEventReasonHwPowerBrakeSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        sm = [float(c) for c, _, _ in self.samples]
        pw = [p for _, p, _ in self.samples]
        reasons = sorted(n for n, b in bits.items() if any(r & b for _, _, r in self.samples))
        cap = [bool(r & bits["sw_power_cap"]) for _, _, r in self.samples]
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": smax,
                "sm_mhz_min": min(sm) if sm else None, "sm_mhz_p90": float(np.percentile(sm, 90)) if sm else None,
                "reasons": reasons, "samples": len(sm), "source": "nvml 2 ms",
                "power_cap_frac": float(np.mean(cap)) if cap else None,
                "power_w_max": max(pw) if pw else None}

    def stop(self):
        if self.nvml is not None:
            return self._stop_nvml()
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons, pw = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                pw.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi 100 ms",
                "power_w_max": max(pw) if pw else None}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def launches_per_step(eps: float, fixed_point: bool, row_max: bool = False, stripes: bool = False) -> int:
    """Kernels of this library launched by one forward + backward call pair:
    forward logit/LSE kernel and finalize; backward tile kernel (or the
    stripe kernel, one launch up to 16384 tokens, and nothing else); the
    norm pass (classifier and token norms) when the filter (without the
    forward's row maxima) or the fixed-point mode needs it; with the filter
    on the pre-pass (blocks, totals) and the flat-row kernel; the dloss
    maximum and two conversion passes in fixed point; and with both, the
    clearing of the dC accumulator rows that can receive a gradient."""
    n = 2 + 1
    if stripes and not fixed_point:
        return n
    if fixed_point or (eps > 0 and not row_max):
        n += 2
    if eps > 0:
        n += 3
    if fixed_point:
        n += 3
    if eps > 0 and fixed_point:
        n += 1
    return n


def scale_bf16_bits(bits, scale):
    """bf16 bit patterns times `scale`, rounded back to bf16."""
    from linear_cross_entropy_05_b200 import synth
    return synth.round_to_bf16_bits((bits.astype(np.uint32) << 16).view(np.float32) * np.float32(scale))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_hash(which: str) -> str:
    """Hash of the code of a kernel's sources and of the host code that plans
    its launches (split counts, unit orders: they change the traffic too),
    comments and blank lines removed (a comment edit does not change the
    kernel the counters came from)."""
    import re
    base = os.path.join(ROOT, "linear_cross_entropy_05_b200", "csrc")
    h = hashlib.sha256()
    for f in (f"{which}.cu", "common.cuh", "ptx.cuh", "api.cu"):
        with open(os.path.join(base, f)) as fh:
            src = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        for line in src.splitlines():
            line = line.split("//", 1)[0].rstrip()
            if line.strip():
                h.update(line.encode() + b"\n")
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel, {}).get(workload)
    if not e or e.get("source_hash") != kernel_source_hash("fwd" if kernel.startswith("fwd") else "bwd"):
        return None
    return e.get("dram_bytes_per_launch")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_step(inp, rows, eps, C64=None):
    """The oracle's forward + backward for the token rows `rows` (a whole
    number of 32-row units): loss/lse for those rows, then their full
    contribution to dE and dC (entry filter applied).  C64: the classifier
    already decoded to fp64 (resident input), else decoded here."""
    import oracle
    E64 = oracle.bf16_bits_to_f64(inp["E"][rows])
    if C64 is None:
        C64 = oracle.bf16_bits_to_f64(inp["C"])
    y = inp["y"][rows]
    loss, lse = oracle.forward_f64(E64, C64, y, IGN)
    dl = np.full(len(rows), 1.0 / max(1, len(rows)))
    dE, dC = oracle.backward_f64(E64, C64, y, lse, dl, IGN, filter_eps=eps, tile=(1, 1))
    return loss


def cpu_baseline(inp, w, rows_n: int, gpu_loss=None):
    """Time the oracle on the first rows_n tokens; if the GPU's per-token
    losses are given, also report their largest deviation from the oracle's
    on those tokens (the same oracle run, no extra work)."""
    rows = np.arange(rows_n)
    t0 = time.perf_counter()
    oloss = oracle_step(inp, rows, w.filter_eps)
    dt = time.perf_counter() - t0
    out = {"value": rows_n / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
           "sample": f"fp64 oracle forward+backward (tile filter {w.filter_eps:g}) on the first {rows_n} tokens "
                     f"of the {w.name} workload (full V={w.V}, D={w.D}); {dt:.2f} s"}
    if gpu_loss is not None:
        keep = inp["y"][rows] != IGN
        err = np.abs(np.asarray(gpu_loss[:rows_n], dtype=np.float64) - oloss)[keep]
        out["parity_loss_max_abs_err"] = float(err.max()) if err.size else 0.0
    return out


# ---------------------------------------------------------------------------
# arms
# ---------------------------------------------------------------------------

def run_reference(args, w):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    from linear_cross_entropy_05_b200 import synth
    log(f"[reference] generating {w.name} ...")
    inp = synth.make_inputs(w)
    import oracle
    # the classifier is a resident input (decoded to fp64 once, as the GPU
    # arm keeps C on the device); every step decodes its token rows
    C64 = oracle.bf16_bits_to_f64(inp["C"])
    rows_n = max(32, args.ref_rows // 32 * 32)
    # size the per-step sample so that warm-up + timed steps stay within the
    # time budget: the first warm-up step calibrates (the oracle's cost is
    # linear in the number of token rows)
    t_cal = time.perf_counter()
    oracle_step(inp, np.arange(rows_n), w.filter_eps, C64)
    t_cal = time.perf_counter() - t_cal
    total_steps = args.steps + max(0, args.warmup - 1)
    if total_steps * t_cal > args.ref_budget_s:
        rows_n = max(32, int(rows_n * args.ref_budget_s / (total_steps * t_cal)) // 32 * 32)
    rows = np.arange(rows_n)
    for _ in range(args.warmup - 1):
        oracle_step(inp, rows, w.filter_eps, C64)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(inp, rows, w.filter_eps, C64)
    dt = time.perf_counter() - t0
    value = rows_n * args.steps / dt
    sample = (f"each step: fp64 oracle forward+backward (unit filter {w.filter_eps:g}) on {rows_n} tokens of the "
              f"{w.name} workload (full V={w.V}, D={w.D}; classifier decoded to fp64 once, outside the steps)")
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, ws), "gpu_launches": 0, "device": f"host cores (rank 0 of {ws})",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


def config_of(w, world):
    return {"workload": w.name, "N": w.N, "D": w.D, "V": w.V, "labels": f"{w.labels}({w.zipf_s})",
            "input_std": w.std, "filter_eps": w.filter_eps, "global_batch": w.N * world, "seq_len": None,
            "parallelism": f"replicas{world}" if world > 1 else "single-gpu",
            "l2": "inputs larger than L2 (C alone is %.2f GB, L2 126 MB); no flush" % (w.V * w.D * 2 / 1e9)}


def run_gpu(args, w):
    import torch
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist("nccl")
    import linear_cross_entropy_05_b200 as L
    from linear_cross_entropy_05_b200 import synth

    t0 = time.perf_counter()
    inp = synth.make_inputs(w)
    log(f"[rank {rank}] generated {w.name} in {time.perf_counter() - t0:.1f} s")
    if args.e_scale:
        # stress variant (not one of the workloads): E scaled so that the
        # softmax is peaky and token blocks are no longer flat
        inp["E"] = scale_bf16_bits(inp["E"], args.e_scale)
    N, D, V = w.N, w.D, w.V
    E = torch.from_numpy(inp["E"].view(np.int16)).view(torch.bfloat16).to(dev)
    C = torch.from_numpy(inp["C"].view(np.int16)).view(torch.bfloat16).to(dev)
    y = torch.from_numpy(inp["y"]).to(dev)
    dloss = torch.from_numpy(synth.mean_dloss(inp["y"])).to(dev)
    loss = torch.empty(N, device=dev)
    lse = torch.empty(N, device=dev)
    dE = torch.empty((N, D), device=dev)
    dC = torch.empty((V, D), device=dev)
    ws_f = L.Workspace(dev)
    ws_b = L.Workspace(dev)
    eps = w.filter_eps
    stream = torch.cuda.current_stream()
    ws_b.get(L.cce_backward_workspace_size_ex(
        N, D, V, (L.CCE_BWD_DETERMINISTIC if args.deterministic else 0) |
        (L.CCE_BWD_BF16_GRADS if args.bf16_grads else 0) |
        (L.CCE_BWD_STRIPES if args.bwd_stripes else 0)))   # allocated before the side stream uses it

    gkw = dict(deterministic=args.deterministic, bf16_grads=args.bf16_grads)
    if args.bwd_stripes:
        gkw["stripes"] = True
    if args.bf16_grads:
        dE = torch.empty((N, D), device=dev, dtype=torch.bfloat16)
        dC = torch.empty((V, D), device=dev, dtype=torch.bfloat16)

    # Side stream during the (tensor-bound) forward: the classifier-only part
    # of the backward's pre-pass (cce_backward_prepare: max_v |C_v|, one read
    # of C) and, by default, the clearing of the fp32 dE/dC, into which the
    # backward then adds (CCE_BWD_ACCUMULATE; in the deterministic mode the
    # conversion pass then adds once per entry and leaves the rows of
    # unvisited vocabulary tiles alone); the bf16 outputs are written anyway.
    overlap_zero = not (args.bf16_grads or args.no_overlap_zero)
    # (the classifier bound is used only by the filter and the fixed-point modes)
    # the forward's row maxima bound the logits for the filter's pre-pass
    # (CCE_BWD_ROW_MAX); then only the fixed-point modes need max_v |C_v|
    use_rows = eps > 0 and not args.bwd_stripes and not args.no_row_max
    row_max = torch.empty(N, device=dev) if use_rows else None
    fixed_mode = args.deterministic or args.bf16_grads
    prepare = (not args.no_prepare and not args.bwd_stripes and
               (fixed_mode or (eps > 0 and not use_rows)))
    side_stream = torch.cuda.Stream(device=dev)
    side_done = torch.cuda.Event()

    def fwd_bwd(Eb, Cb, yb, dlb):
        if overlap_zero or prepare:
            with torch.cuda.stream(side_stream):
                # after the previous backward (dE/dC and the backward workspace
                # are free) and after this step's inputs have arrived
                side_stream.wait_stream(stream)
                if prepare:
                    L.backward_prepare(Cb, N, ws_b, stream=side_stream, **gkw)
                if overlap_zero:
                    dE.zero_()
                    dC.zero_()
                side_done.record(side_stream)
        L.forward(Eb, Cb, yb, IGN, workspace=ws_f, out=(loss, lse), row_max=row_max)
        if overlap_zero or prepare:
            stream.wait_event(side_done)
        L.backward(Eb, Cb, yb, lse, dlb, eps, IGN, workspace=ws_b, out=(dE, dC), accumulate=overlap_zero,
                   prepared=prepare, row_max=row_max, **gkw)

    def step():
        fwd_bwd(E, C, y, dloss)

    # warm-up (also loads the module) and status check
    for _ in range(max(3, args.warmup)):
        step()
    stf = L.read_status(ws_f)
    stb = L.read_status(ws_b)
    if stf["status"] != 0 or stb["status"] != 0:
        raise RuntimeError(f"device status not clean: fwd {stf} bwd {stb}")
    # vocabulary splits of the forward (its workspace holds N (max, sum) pairs per split)
    fwd_splits = (L.cce_forward_workspace_size(N, D, V) - 256) // (8 * N)
    live, dead, pruned = stb["live_tiles"], stb["dead_tiles"], stb["pruned_tiles"]
    flat = stb["flat_units"]            # live units formed by the flat-row kernel (no tensor-core work)
    recomputed = stb["logit_tiles"]     # 128 x 256 logit tiles the backward recomputed

    # extra global memory of one step: the library allocates nothing itself
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info(dev)
    step()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info(dev)
    lib_alloc = max(0, free0 - free1)
    extra_hbm = ws_f.buf.numel() + ws_b.buf.numel() + lib_alloc

    # ---- timed region: K steps, per-kernel events through the library hook ----
    K = args.steps
    ev = {k: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
          for k in (0, 1)}
    for k in (0, 1):               # torch creates the CUDA event on first record
        for a, b in ev[k]:
            a.record(stream)
            b.record(stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_stop = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(K):
        L.cce_debug_set_kernel_events(0, ev[0][i][0].cuda_event, ev[0][i][1].cuda_event)
        L.cce_debug_set_kernel_events(1, ev[1][i][0].cuda_event, ev[1][i][1].cuda_event)
        step()
    t_stop.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    L.cce_debug_set_kernel_events(0, 0, 0)
    L.cce_debug_set_kernel_events(1, 0, 0)
    clk = clocks.stop()
    sec_local = t_start.elapsed_time(t_stop) / 1e3
    value, sec = aggregate_throughput(dist, float(N * K), sec_local, dev)
    fwd_ms = float(np.mean([a.elapsed_time(b) for a, b in ev[0]]))
    bwd_ms = float(np.mean([a.elapsed_time(b) for a, b in ev[1]]))
    step_ms = 1e3 * sec / K

    # ---- the dense backward (filter off), outside the timed region ----
    # Every 32 x 32 unit is live: recompute of every logit tile plus both
    # full contractions, 6 N D V flops.  This is the path of a head whose
    # softmax is not sparse (a trained model); timed per launch through the
    # kernel-event hook on the same inputs.
    dense = None
    if not args.no_dense and not (args.deterministic or args.bf16_grads):
        ws_d = L.Workspace(dev)
        evd = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(3)]
        stripes = not args.dense_fused
        L.backward(E, C, y, lse, dloss, 0.0, IGN, workspace=ws_d, out=(dE, dC), stripes=stripes)   # warm-up
        for a_, b_ in evd:
            a_.record(stream)
            b_.record(stream)
        torch.cuda.synchronize()
        clocks_d = ClockSampler(local)
        clocks_d.start()
        time.sleep(0.3)
        for a_, b_ in evd:
            L.cce_debug_set_kernel_events(1, a_.cuda_event, b_.cuda_event)
            L.backward(E, C, y, lse, dloss, 0.0, IGN, workspace=ws_d, out=(dE, dC), stripes=stripes)
        torch.cuda.synchronize()
        L.cce_debug_set_kernel_events(1, 0, 0)
        clk_d = clocks_d.stop()
        std = L.read_status(ws_d)
        dense = {"path": ("softmax-gradient stripes (CCE_BWD_STRIPES)" if stripes else
                          "fused per-tile contractions with fp32 reduce-adds"),
                 "workspace_bytes": int(ws_d.buf.numel()),
                 "ms": float(np.mean([a_.elapsed_time(b_) for a_, b_ in evd])), "launches": len(evd),
                 "flop_per_launch": 6.0 * N * D * V, "status": std["status"],
                 "live_units": std["live_tiles"], "logit_tiles_recomputed": std["logit_tiles"],
                 "clocks": {"sm_mhz": clk_d["sm_mhz"], "reasons": clk_d["reasons"]}}
        del ws_d

    # ---- end to end through the public API with host buffers ----
    # Every step copies its inputs (E, C, y, dloss) from pinned host memory
    # and reads its per-token loss back.  Two device input buffers let step
    # k+1's copy (on a copy stream) overlap step k's kernels.
    E_h = torch.from_numpy(inp["E"].view(np.int16)).view(torch.bfloat16).pin_memory()
    C_h = torch.from_numpy(inp["C"].view(np.int16)).view(torch.bfloat16).pin_memory()
    y_h = torch.from_numpy(inp["y"]).pin_memory()
    dl_h = torch.from_numpy(synth.mean_dloss(inp["y"])).pin_memory()
    h2d = E_h.numel() * 2 + C_h.numel() * 2 + y_h.numel() * 8 + dl_h.numel() * 4
    d2h = N * 4
    e2e_value = e2e_resident = None
    if not args.no_e2e:
        Ke = max(3, K // 4)
        bufs = [(E, C, y, dloss)]
        bufs.append((torch.empty_like(E), torch.empty_like(C), torch.empty_like(y), torch.empty_like(dloss)))
        loss_h = [torch.empty(N, dtype=torch.float32).pin_memory() for _ in range(2)]
        copy_stream = torch.cuda.Stream(device=dev)
        copied = [torch.cuda.Event() for _ in range(2)]
        consumed = [torch.cuda.Event() for _ in range(2)]
        for b in range(2):
            consumed[b].record(stream)

        def e2e_run(steps, copy_c=True):
            for k in range(steps):
                b = k % 2
                Eb, Cb, yb, dlb = bufs[b]
                with torch.cuda.stream(copy_stream):
                    copy_stream.wait_event(consumed[b])
                    Eb.copy_(E_h, non_blocking=True)
                    if copy_c:
                        Cb.copy_(C_h, non_blocking=True)
                    yb.copy_(y_h, non_blocking=True)
                    dlb.copy_(dl_h, non_blocking=True)
                    copied[b].record(copy_stream)
                stream.wait_event(copied[b])
                fwd_bwd(Eb, Cb if copy_c else C, yb, dlb)
                loss_h[b].copy_(loss, non_blocking=True)
                consumed[b].record(stream)

        def e2e_time(copy_c):
            e2e_run(2, copy_c)
            torch.cuda.synchronize()
            if dist is not None:
                dist.barrier()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            e2e_run(Ke, copy_c)
            e1.record(stream)
            torch.cuda.synchronize()
            v, _ = aggregate_throughput(dist, float(N * Ke), e0.elapsed_time(e1) / 1e3, dev)
            if not np.isfinite(loss_h[(Ke - 1) % 2].numpy()).all():
                raise RuntimeError("end-to-end loss read back non-finite values")
            return v

        e2e_value = e2e_time(True)
        # the same with the classifier C resident on the device (a training
        # step's weights): only E, y and dloss cross the host link each step
        e2e_resident = e2e_time(False)
        del bufs

    # ---- roofline of the dominant kernel ----
    peaks, peak_src = measured_peaks()
    unit_flop = 2.0 * FU[0] * FU[1] * D    # one filter unit's products, per contraction
    flop_fwd = 2.0 * N * D * V
    # recompute of the visited logit tiles + the dE and dC products of the live
    # units the tile kernel contracted (the flat-row kernel's are not tensor work)
    flop_bwd = recomputed * 2.0 * BM * BN * D + (live - flat) * 2.0 * unit_flop
    fwd_name = "fwd_lse_pair_kernel" if args.fwd_variant == "pair" else "fwd_lse_kernel"
    dominant = "bwd_kernel" if bwd_ms >= fwd_ms else fwd_name
    dom_flop, dom_ms = (flop_bwd, bwd_ms) if dominant == "bwd_kernel" else (flop_fwd, fwd_ms)
    # The timed region is well under a second of work per launch, so the
    # kernels are held to the burst figure; the sustained one (a seconds-long
    # cuBLAS loop that settles at a lower clock under the power cap) is
    # reported beside it, with the SM clock sampled during the timed region.
    peak = float(peaks["bf16_tflops"])
    peak_sus = float(peaks.get("bf16_tflops_sustained") or peak)
    achieved = dom_flop / (dom_ms * 1e-3) / 1e12
    traffic = ncu_traffic(dominant, w.name)
    executed_flop = flop_fwd + flop_bwd
    if dense is not None:
        dense["tflops"] = dense["flop_per_launch"] / dense["ms"] / 1e9
        dense["frac_of_burst_peak"] = dense["tflops"] / peak
        dense["frac_of_sustained_peak"] = dense["tflops"] / peak_sus

    out = None
    if rank == 0:
        cpu = (cpu_baseline(inp, w, args.cpu_rows, gpu_loss=loss.cpu().numpy())
               if world == 1 and not args.no_cpu_baseline else None)
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded numpy PCG64; random-init classifier, Zipf labels)",
            "config": dict(config_of(w, world), forward_kernel=args.fwd_variant,
                           backward_accumulation=("fixed-point int64" if (args.deterministic or args.bf16_grads)
                                                  else "fp32 atomic (TMA reduce-add)"),
                           grad_dtype="bf16" if args.bf16_grads else "fp32",
                           grad_zeroing=("side stream during the forward; backward accumulates (CCE_BWD_ACCUMULATE)"
                                         if overlap_zero else "inside the backward call"),
                           classifier_norm=("cce_backward_prepare on the side stream during the forward"
                                            if prepare else
                                            "not needed (the forward's row maxima bound the logits)"
                                            if use_rows and not fixed_mode else "inside the backward call"),
                           row_max=use_rows,
                           l2_prefetch_slices=list(args.prefetch) if args.prefetch else [0, 0],
                           reduce_prefetch_slices=args.reduce_prefetch, l2_hints=bool(args.l2_hints),
                           forward_splits=fwd_splits,
                           e_scale=args.e_scale,
                           backward_path=("stripes (CCE_BWD_STRIPES)" if args.bwd_stripes else
                                          "pre-pass, flat rows, tile kernel" if eps > 0 else "stripes"),
                           forward_schedule=list(args.fwd_schedule) if args.fwd_schedule else None,
                           forward_order=("round-robin" if args.fwd_order == 0 else "one queue per L2 half")),
            "roofline": {"bound": "tensor", "kernel": dominant, "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16_tflops (burst: the timed region is under a second)",
                         "frac_sustained": achieved / peak_sus, "peak_sustained": peak_sus,
                         "sm_mhz_median": clk["sm_mhz"],
                         "flop_per_launch": dom_flop, "launch_ms": dom_ms},
            "kernels": {fwd_name: {"ms": fwd_ms, "tflops": flop_fwd / fwd_ms / 1e9,
                                   "frac_of_burst_peak": flop_fwd / fwd_ms / 1e9 / peak},
                        "bwd_kernel": {"ms": bwd_ms, "tflops": flop_bwd / bwd_ms / 1e9,
                                       "frac_of_burst_peak": flop_bwd / bwd_ms / 1e9 / peak,
                                       "live_units": live, "dead_units": dead, "pruned_units": pruned,
                                       "flat_units": flat,
                                       "logit_tiles_recomputed": recomputed},
                        "bwd_dense": dense},
            # flops the tensor cores executed in a step (forward, recomputed
            # tiles, live units' contractions) over the step time, against the
            # burst peak; pruned units are not counted
            "pct_bf16_peak_executed": executed_flop / (step_ms * 1e-3) / 1e12 / peak,
            "filter_unit": [1, 1],          # entries are kept or dropped one by one
            "skip_unit": list(FU),          # live / dead / pruned counts are of these units
            "live_unit_frac": live / max(1, live + dead + pruned),
            "extra_hbm_bytes": int(extra_hbm),
            "materialised_logits_fp32_bytes": N * V * 4,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "inputs_copied": "E, C, y, dloss every step",
                    "weights_resident": {"value": e2e_resident, "unit": UNIT,
                                         "h2d_bytes_per_step": int(h2d - C_h.numel() * 2),
                                         "inputs_copied": "E, y, dloss every step; C uploaded once"}},
            # our kernels per step (launches_per_step lists them)
            "gpu_launches": launches_per_step(eps, args.deterministic or args.bf16_grads, use_rows,
                                              args.bwd_stripes) * K,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if out is not None:
        print(json.dumps(out), flush=True)
    return 0


def run_vocab_parallel(args, w):
    """The vocabulary-parallel form on N ranks (one GPU each, NCCL): rank r
    holds the classifier shard C[v_offset : v_offset + V_r] and runs
    vocab_parallel_forward_backward on the whole batch (forward on its shard,
    all-gather of 12 bytes per token, merge, backward on its shard,
    all-reduce of the dE shares).  The batch is shared, so the throughput is
    N tokens / max time over ranks ("scaling": "strong").  No TMA multicast:
    every load of the kernels reads this GPU's own memory."""
    import torch
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist("nccl")
    import linear_cross_entropy_05_b200 as L
    from linear_cross_entropy_05_b200 import synth
    inp = synth.make_inputs(w)
    N, D, V = w.N, w.D, w.V
    v0, Vr = vocab_shard(V, world, rank)
    E = torch.from_numpy(inp["E"].view(np.int16)).view(torch.bfloat16).to(dev)
    C_sh = torch.from_numpy(inp["C"][v0:v0 + Vr].view(np.int16)).view(torch.bfloat16).to(dev)
    y = torch.from_numpy(inp["y"]).to(dev)
    dloss = torch.from_numpy(synth.mean_dloss(inp["y"])).to(dev)
    stream = torch.cuda.current_stream()

    def step():
        return L.vocab_parallel_forward_backward(E, C_sh, y, v0, V, dloss=dloss, filter_eps=w.filter_eps)

    for _ in range(max(3, args.warmup)):
        loss, lse, dE, dC = step()
    torch.cuda.synchronize()
    K = args.steps
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(K):
        loss, lse, dE, dC = step()
    t1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    value, sec = aggregate_shared_batch(dist, float(N * K), t0.elapsed_time(t1) / 1e3, dev)
    finite = bool(torch.isfinite(loss).all())
    out = None
    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": 1e3 * sec / K, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded numpy PCG64; random-init classifier, Zipf labels)",
            "config": dict(config_of(w, world), parallelism=f"vocab{world}", global_batch=N,
                           shard_rows=[vocab_shard(V, world, r)[1] for r in range(world)],
                           collectives="all-gather of [3, N] fp32 shard statistics; all-reduce of dE (N x D fp32)"),
            # per step: shard forward (logit kernel + finalize), the merge, and the
            # shard backward's kernels (as in a one-GPU step)
            "gpu_launches": (launches_per_step(w.filter_eps, False) + 1) * K,
            "clocks": clk, "loss_finite": finite, "e2e": None, "cpu_baseline": None,
        }
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if out is not None:
        print(json.dumps(out), flush=True)
    return 0


def run_trace(args, w):
    """Per-tile timeline of one backward launch (cce_debug_set_backward_trace):
    per CTA and tile, how long the epilogue waited for the recomputed logits,
    how long it took to form and publish the gradient tile, and how long the
    contraction and its drain took until the next tile.  One JSON object
    (documentation, not the contract line)."""
    import torch
    import linear_cross_entropy_05_b200 as L
    from linear_cross_entropy_05_b200 import synth
    dev = torch.device("cuda", 0)
    inp = synth.make_inputs(w)
    E = torch.from_numpy(inp["E"].view(np.int16)).view(torch.bfloat16).to(dev)
    C = torch.from_numpy(inp["C"].view(np.int16)).view(torch.bfloat16).to(dev)
    y = torch.from_numpy(inp["y"]).to(dev)
    dl = torch.from_numpy(synth.mean_dloss(inp["y"])).to(dev)
    wf, wb = L.Workspace(dev), L.Workspace(dev)
    loss, lse = L.forward(E, C, y, IGN, workspace=wf)
    dE = torch.empty((w.N, w.D), device=dev)
    dC = torch.empty((w.V, w.D), device=dev)
    for _ in range(3):
        L.backward(E, C, y, lse, dl, w.filter_eps, IGN, workspace=wb, out=(dE, dC))
    cap = 256
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    tr = torch.zeros(sms * cap * 4, dtype=torch.int64, device=dev)
    L.cce_debug_set_backward_trace(tr.data_ptr(), cap)
    try:
        L.backward(E, C, y, lse, dl, w.filter_eps, IGN, workspace=wb, out=(dE, dC))
        torch.cuda.synchronize()
    finally:
        L.cce_debug_set_backward_trace(0, 1)
    st = L.read_status(wb)
    t = tr.view(sms, cap, 4).cpu().numpy().astype(np.int64)
    t0 = t[:, 0, 0][t[:, 0, 0] > 0].min()
    S, G, Cc, ntiles, ends = [], [], [], [], []
    for b in range(sms):
        k = 0
        while k < cap - 1 and t[b, k, 1] > 0:
            S.append(t[b, k, 1] - t[b, k, 0])
            G.append(t[b, k, 2] - t[b, k, 1])
            Cc.append(t[b, k + 1, 0] - t[b, k, 2])
            k += 1
        ntiles.append(k)
        ends.append(t[b, k, 0] - t0)
    us = lambda x: float(np.mean(x) / 1e3) if x else None
    print(json.dumps({
        "mode": "trace", "workload": w.name, "N": w.N, "D": w.D, "V": w.V, "filter_eps": w.filter_eps,
        "status": st, "ctas": sms, "tiles_per_cta_mean": float(np.mean(ntiles)), "tiles_per_cta_max": int(max(ntiles)),
        "kernel_span_us": float(max(ends) / 1e3), "first_cta_end_us": float(min(ends) / 1e3),
        "wait_for_logits_us": us(S), "gradient_tile_us": us(G), "contraction_and_drain_us": us(Cc)}), flush=True)
    return 0


def run_trace_stripes(args, w):
    """Per-task timeline of one dense (filter-off) stripe backward launch
    through the trace hook: per task kind, the time between the completions
    of consecutive accumulators of a CTA pair (the tensor cores' time per
    task, bubbles included), how long the pair's producer waited for the
    task's inputs, and how often a task was handed out only after the
    previous accumulator was complete (a pipeline bubble).  One JSON object
    (documentation, not the contract line)."""
    import torch
    import linear_cross_entropy_05_b200 as L
    from linear_cross_entropy_05_b200 import synth
    dev = torch.device("cuda", 0)
    inp = synth.make_inputs(w)
    E = torch.from_numpy(inp["E"].view(np.int16)).view(torch.bfloat16).to(dev)
    C = torch.from_numpy(inp["C"].view(np.int16)).view(torch.bfloat16).to(dev)
    y = torch.from_numpy(inp["y"]).to(dev)
    dl = torch.from_numpy(synth.mean_dloss(inp["y"])).to(dev)
    wf, wb = L.Workspace(dev), L.Workspace(dev)
    loss, lse = L.forward(E, C, y, IGN, workspace=wf)
    dE = torch.empty((w.N, w.D), device=dev)
    dC = torch.empty((w.V, w.D), device=dev)
    for _ in range(2):
        L.backward(E, C, y, lse, dl, 0.0, IGN, workspace=wb, out=(dE, dC), stripes=True)
    cap = 4096
    pairs = torch.cuda.get_device_properties(dev).multi_processor_count // 2
    tr = torch.zeros(pairs * cap * 4, dtype=torch.int64, device=dev)
    L.cce_debug_set_backward_trace(tr.data_ptr(), cap)
    try:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        L.backward(E, C, y, lse, dl, 0.0, IGN, workspace=wb, out=(dE, dC), stripes=True)
        e1.record()
        torch.cuda.synchronize()
    finally:
        L.cce_debug_set_backward_trace(0, 1)
    st = L.read_status(wb)
    t = tr.view(pairs, cap, 4).cpu().numpy().astype(np.int64)
    names = {0: "A recompute + G store", 1: "B dC tile", 2: "C dE tile"}
    per = {k: {"n": 0, "acc_interval_us": [], "dep_wait_us": [], "epilogue_us": [], "bubbles": 0} for k in names}
    t_first = t[:, 0, 0][t[:, 0, 0] > 0].min()
    ends = []
    for p in range(pairs):
        k = 0
        while k < cap and t[p, k, 0] > 0:
            kind = int(t[p, k, 3] & 0xFF)
            d = per[kind]
            d["n"] += 1
            d["dep_wait_us"].append((t[p, k, 3] >> 8) / 1e3)
            if t[p, k, 2] > 0 and t[p, k, 1] > 0:
                d["epilogue_us"].append((t[p, k, 2] - t[p, k, 1]) / 1e3)
            if k > 0 and t[p, k, 1] > 0 and t[p, k - 1, 1] > 0:
                d["acc_interval_us"].append((t[p, k, 1] - t[p, k - 1, 1]) / 1e3)
                if t[p, k, 0] > t[p, k - 1, 1]:
                    d["bubbles"] += 1
            k += 1
        if k:
            ends.append((t[p, k - 1, 2] - t_first) / 1e3)
    flop = {0: 2.0 * 256 * 256 * w.D, 1: 2.0 * 256 * 256 * -(-w.N // 256) * 256,
            2: 2.0 * 256 * 256 * min(STRIPE_COLS, -(-w.V // 256) * 256)}
    peaks, _ = measured_peaks()
    pair_peak = float(peaks["bf16_tflops"]) * 1e12 / pairs
    out = {"mode": "trace-stripes", "workload": w.name, "N": w.N, "D": w.D, "V": w.V, "status": st,
           "launch_ms": e0.elapsed_time(e1), "pairs": pairs, "first_pair_done_us": float(min(ends)),
           "last_pair_done_us": float(max(ends)), "kinds": {}}
    for k, nm in names.items():
        d = per[k]
        out["kinds"][nm] = {
            "tasks": d["n"], "acc_interval_us_mean": float(np.mean(d["acc_interval_us"])) if d["acc_interval_us"] else None,
            "at_burst_peak_us": flop[k] / pair_peak * 1e6,
            "dep_wait_us_mean": float(np.mean(d["dep_wait_us"])) if d["dep_wait_us"] else None,
            "epilogue_us_mean": float(np.mean(d["epilogue_us"])) if d["epilogue_us"] else None,
            "handed_out_after_previous_done": d["bubbles"]}
    print(json.dumps(out), flush=True)
    return 0


def run_memory(args, w):
    """Classifier-head training step through the autograd wrapper: peak extra
    device memory and time of `linear_cross_entropy(E, C, y).backward()`
    against the same step with materialised logits (E C^T in bf16, then
    torch's fp32 cross-entropy), the usual head a user would replace.  The
    torch step is a comparison only; it runs nothing of this library.  One
    JSON object (documentation, not the contract line)."""
    import torch
    import torch.nn.functional as F
    import linear_cross_entropy_05_b200 as L
    from linear_cross_entropy_05_b200 import synth
    dev = torch.device("cuda", 0)
    inp = synth.make_inputs(w)
    E0 = torch.from_numpy(inp["E"].view(np.int16)).view(torch.bfloat16).to(dev)
    C0 = torch.from_numpy(inp["C"].view(np.int16)).view(torch.bfloat16).to(dev)
    y = torch.from_numpy(inp["y"]).to(dev)

    def cce_step(E, C):
        return L.linear_cross_entropy(E, C, y, IGN, w.filter_eps)

    def torch_step(E, C):
        return F.cross_entropy((E @ C.t()).float(), y, ignore_index=IGN)

    def measure(step, reps=5):
        E = E0.clone().requires_grad_(True)
        C = C0.clone().requires_grad_(True)
        out = {}
        for i in range(reps + 1):
            E.grad = None
            C.grad = None
            torch.cuda.synchronize()
            base = torch.cuda.memory_allocated(dev)
            torch.cuda.reset_peak_memory_stats(dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            loss = step(E, C)
            loss.backward()
            e1.record()
            torch.cuda.synchronize()
            if i == 0:        # first call: module load / allocator warm-up
                continue
            out.setdefault("ms", []).append(e0.elapsed_time(e1))
            out["peak_extra_bytes"] = max(out.get("peak_extra_bytes", 0),
                                          torch.cuda.max_memory_allocated(dev) - base)
        out["loss"] = float(loss)
        out["dE"], out["dC"] = E.grad.float(), C.grad.float()
        out["ms"] = float(np.median(out["ms"]))
        return out

    a = measure(cce_step)
    b = measure(torch_step)
    rel = lambda x, r: float((x - r).norm() / r.norm())
    grads = (w.N + w.V) * w.D * 2
    res = {
        "mode": "memory", "workload": w.name, "N": w.N, "D": w.D, "V": w.V, "filter_eps": w.filter_eps,
        "gradient_bytes_bf16": grads,
        "cce": {"peak_extra_bytes": int(a["peak_extra_bytes"]), "ms_per_step": a["ms"],
                "tokens_per_s": w.N / a["ms"] * 1e3},
        "materialised_torch": {"peak_extra_bytes": int(b["peak_extra_bytes"]), "ms_per_step": b["ms"],
                               "tokens_per_s": w.N / b["ms"] * 1e3,
                               "what": "logits = E @ C^T (bf16), F.cross_entropy(logits.float()), backward"},
        "loss_abs_diff": abs(a["loss"] - b["loss"]),
        "dE_rel_diff": rel(a["dE"], b["dE"]), "dC_rel_diff": rel(a["dC"], b["dC"]),
    }
    print(json.dumps(res), flush=True)
    return 0


def run_suite(args):
    """Per-workload table (not the contract line): fwd-only and fwd+bwd time,
    executed tensor fraction, tiles visited, extra global memory against the
    size of the materialised fp32 logits.  One JSON object per workload."""
    import torch
    import linear_cross_entropy_05_b200 as L
    from linear_cross_entropy_05_b200 import synth
    dev = torch.device("cuda", 0)
    peaks, _ = measured_peaks()
    peak = float(peaks["bf16_tflops"])   # burst: every call here is timed alone
    cases = [synth.TINY, synth.GEMMA2_2B, synth.LLAMA3_8B, synth.SMALL_LARGE_VOCAB,
             synth.SMALL_LARGE_VOCAB.__class__(**{**synth.SMALL_LARGE_VOCAB.__dict__, "filter_eps": 0.0,
                                                   "name": "small-model-large-vocab[filter off]"})] + \
            [synth.SWEEP.with_sizes(N=n, name=f"long-batch-sweep[N={n}]") for n in synth.SWEEP_NS]
    for w in cases:
        inp = synth.make_inputs(w)
        N, D, V = w.N, w.D, w.V
        E = torch.from_numpy(inp["E"].view(np.int16)).view(torch.bfloat16).to(dev)
        C = torch.from_numpy(inp["C"].view(np.int16)).view(torch.bfloat16).to(dev)
        y = torch.from_numpy(inp["y"]).to(dev)
        dl = torch.from_numpy(synth.mean_dloss(inp["y"])).to(dev)
        wsf, wsb = L.Workspace(dev), L.Workspace(dev)
        # the forward's row maxima feed the filter's pre-pass (as in the step)
        rm = torch.empty(N, device=dev) if (w.filter_eps > 0 and not args.no_row_max) else None
        loss, lse = L.forward(E, C, y, IGN, workspace=wsf, row_max=rm)
        dE, dC = L.backward(E, C, y, lse, dl, w.filter_eps, IGN, workspace=wsb, row_max=rm)
        st = L.read_status(wsb)
        reps = 5
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        torch.cuda.synchronize()
        tf = tb = 0.0
        for _ in range(reps):
            ev[0].record()
            L.forward(E, C, y, IGN, workspace=wsf, out=(loss, lse), row_max=rm)
            ev[1].record()
            L.backward(E, C, y, lse, dl, w.filter_eps, IGN, workspace=wsb, out=(dE, dC), row_max=rm)
            ev[2].record()
            torch.cuda.synchronize()
            tf += ev[0].elapsed_time(ev[1]) / reps
            tb += ev[1].elapsed_time(ev[2]) / reps
        unit = 2.0 * FU[0] * FU[1] * D
        executed = (2.0 * N * D * V + st["logit_tiles"] * 2.0 * BM * BN * D +
                    (st["live_tiles"] - st["flat_units"]) * 2.0 * unit)
        print(json.dumps({
            "workload": w.name, "N": N, "D": D, "V": V, "filter_eps": w.filter_eps,
            "fwd_ms": tf, "fwd_tokens_per_s": N / tf * 1e3, "fwd_frac_of_peak": 2.0 * N * D * V / tf / 1e9 / peak,
            "fwd_bwd_ms": tf + tb, "fwd_bwd_tokens_per_s": N / (tf + tb) * 1e3,
            "executed_frac_of_peak": executed / (tf + tb) / 1e9 / peak,
            "bwd_ms": tb, "bwd_executed_frac_of_peak": (executed - 2.0 * N * D * V) / tb / 1e9 / peak,
            "tiles": {k: st[k] for k in ("live_tiles", "dead_tiles", "pruned_tiles", "logit_tiles", "flat_units")},
            "extra_hbm_bytes": {"forward_workspace": wsf.buf.numel(), "backward_workspace": wsb.buf.numel()},
            "materialised_logits_fp32_bytes": N * V * 4, "peak_tflops": peak}), flush=True)
        del E, C, y, dl, dE, dC, loss, lse, wsf, wsb
        torch.cuda.empty_cache()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["cce", "reference"], default="cce")
    ap.add_argument("--cpu-rows", type=int, default=1024, help="tokens in the CPU-oracle baseline sample")
    ap.add_argument("--ref-rows", type=int, default=128, help="tokens per step of the reference (oracle) arm")
    ap.add_argument("--ref-budget-s", type=float, default=150.0,
                    help="the reference arm shrinks its per-step sample (to >= 32 tokens) to stay within this time")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end timing")
    ap.add_argument("--workload", default="gemma2-2b-head",
                    help="workload name (the default is the headline Gemma-2-2B-shaped head)")
    ap.add_argument("--N", type=int, default=None, help="override tokens (profiling cases)")
    ap.add_argument("--V", type=int, default=None, help="override vocabulary (profiling cases)")
    ap.add_argument("--bwd-variant", type=int, choices=[0, 1, 2, 3], default=0,
                    help="backward kernel: 0 = 3 stages / 1 staging buffer (default), 1 = 2 stages / 2 buffers, "
                         "2 = 2 stages / 8 epilogue warps, 3 = as 0 with load/store-path reductions")
    ap.add_argument("--deterministic", action="store_true",
                    help="bitwise reproducible backward (fixed-point accumulation)")
    ap.add_argument("--bf16-grads", action="store_true", help="bf16 dE/dC outputs (fixed-point accumulation)")
    ap.add_argument("--no-overlap-zero", action="store_true",
                    help="let the backward zero dE/dC itself instead of a side stream during the forward")
    ap.add_argument("--no-prepare", action="store_true",
                    help="let the backward compute max_v |C_v| itself instead of cce_backward_prepare on the side "
                         "stream during the forward")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense (filter-off) backward measurement")
    ap.add_argument("--dense-fused", action="store_true",
                    help="measure the dense backward on the fused per-tile kernel instead of the stripe kernel")
    ap.add_argument("--fwd-variant", choices=["single", "pair"], default="pair",
                    help="forward kernel: CTA pairs (default) or single CTAs (A/B measurement)")
    ap.add_argument("--prefetch", type=int, nargs=2, default=None, metavar=("FWD", "BWD"),
                    help="L2 prefetch distances in K slices for the forward / backward operand streams (A/B)")
    ap.add_argument("--reduce-prefetch", type=int, default=None, metavar="SLICES",
                    help="L2 prefetch distance of the filtered backward's reduction targets (A/B; 0 = off)")
    ap.add_argument("--l2-hints", action="store_true",
                    help="L2 eviction priorities in the filtered backward (A/B)")
    ap.add_argument("--fwd-schedule", type=int, nargs=4, default=None,
                    metavar=("SPLITS", "GROUP_M", "L2_HINTS", "STAGES"),
                    help="forward schedule (A/B): vocabulary splits per token block and token blocks per raster "
                         "group (0 = chosen per shape), L2 hints of the pair kernel (bit 0: E evict_last, bit 1: C "
                         "evict_first), its operand stages (0 = default 7, or 6)")
    ap.add_argument("--fwd-order", type=int, choices=[0, 1], default=None,
                    help="unit order of the pair forward (A/B): 0 round-robin, 1 one queue per L2 half")
    ap.add_argument("--e-scale", type=float, default=None, metavar="F",
                    help="stress variant, not one of the workloads: E multiplied by F (a peaky softmax whose token "
                         "blocks are not flat)")
    ap.add_argument("--no-row-max", action="store_true",
                    help="let the filter's pre-pass bound the logits by Cauchy-Schwarz instead of the forward's "
                         "per-token maximum logits (A/B)")
    ap.add_argument("--bwd-stripes", action="store_true",
                    help="take the backward through the stripe kernel (CCE_BWD_STRIPES) also with the filter on")
    ap.add_argument("--trace", action="store_true",
                    help="per-tile timeline of one backward launch (recompute wait, gradient tile, contraction)")
    ap.add_argument("--dense-trace", action="store_true",
                    help="with --trace: per-task timeline of the dense stripe backward (filter off)")
    ap.add_argument("--memory", action="store_true",
                    help="classifier-head training step: peak memory and time, CCE vs materialised logits")
    ap.add_argument("--vocab-parallel", action="store_true",
                    help="vocabulary-parallel form over the launched ranks (classifier sharded by rows, NCCL "
                         "exchange) instead of independent replicas")
    ap.add_argument("--suite", action="store_true",
                    help="per-workload table instead of the benchmark line (documentation)")
    args = ap.parse_args(argv)
    if args.impl == "cce" and (args.fwd_variant != "pair" or args.bwd_variant or args.prefetch or
                               args.reduce_prefetch is not None or args.l2_hints or args.fwd_schedule or
                               args.fwd_order is not None):
        import linear_cross_entropy_05_b200 as L
        L.cce_debug_set_forward_variant(1 if args.fwd_variant == "pair" else 0)
        L.cce_debug_set_backward_variant(args.bwd_variant)
        if args.prefetch:
            L.cce_debug_set_prefetch(*args.prefetch)
        if args.reduce_prefetch is not None:
            L.cce_debug_set_reduce_prefetch(args.reduce_prefetch)
        if args.l2_hints:
            L.cce_debug_set_l2_hints(True)
        if args.fwd_schedule:
            L.cce_debug_set_forward_schedule(*args.fwd_schedule)
        if args.fwd_order is not None:
            L.cce_debug_set_forward_order(args.fwd_order)
    if args.suite:
        return run_suite(args)
    if args.memory or args.trace:
        from linear_cross_entropy_05_b200 import synth
        w = synth.WORKLOADS[args.workload]
        w = w.with_sizes(N=args.N, V=args.V) if (args.N or args.V) else w
        if args.memory:
            return run_memory(args, w)
        return run_trace_stripes(args, w) if args.dense_trace else run_trace(args, w)
    if args.warmup < 3:
        args.warmup = 3
    from linear_cross_entropy_05_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if args.N or args.V:
        w = w.with_sizes(N=args.N, V=args.V)
    if args.impl == "reference":
        return run_reference(args, w)
    if args.vocab_parallel:
        return run_vocab_parallel(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
