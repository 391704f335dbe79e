#!/usr/bin/env python3
"""Benchmark of the fused SDPA forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--per-config]

One step = one pass of the whole hot path over one batch: the fused forward
(Q/K/V tiles in, rel-pos projections, QK^T, bias/mask, online softmax, PV,
epilogue) on the SAM ViT-B global-attention workload (B=1, 12 heads, 64x64
patch grid -> 4096 tokens, head_dim 64, bf16, decomposed rel-pos bias), with
inputs resident in HBM.  Several independent input sets (together larger than
the 126 MB L2) are cycled so consecutive steps never hit a warm L2.

Multi-GPU (torchrun, one process per GPU): every rank runs its own
independent problem (weak scaling, no collective on the data path); the time
is the max over ranks.

Rank 0 prints ONE JSON line.  ``--impl reference`` times the fp64 CPU oracle
(the slow, plain definition) on a bounded sample of the same workload.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attention_sdpa_fwd_b200 import workloads as W  # noqa: E402

METRIC = "attention TFLOP/s and % of B200 bf16 peak (or HBM GB/s %) per config, 1 GPU"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def max_over_ranks(values, device):
    """Element-wise max of per-rank floats over all ranks (identity at one rank)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def aggregate_throughput(flops_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job TFLOP/s: every rank runs its own problem (weak scaling), the
    job takes as long as the slowest rank."""
    return world * flops_per_rank / (ms_max * 1e-3) / 1e12


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ---------------------------------------------------------------------------
# clocks sampler (NVML read-only queries during the timed region)
# ---------------------------------------------------------------------------
class ClockSampler:
    """Polls the SM clock and the active clock-event reasons every ~1 ms on a
    background thread (NVML reads only; no setting is touched).  The timed
    region of one bench step is short (well under a second), so a 1 ms cadence
    is what puts samples inside it.  Falls back to ``nvidia-smi -lms 50``."""
    REASONS = (("hw_slowdown", "HwSlowdown"), ("hw_thermal_slowdown", "HwThermalSlowdown"),
               ("sw_thermal_slowdown", "SwThermalSlowdown"), ("sw_power_cap", "SwPowerCap"),
               ("hw_power_brake", "HwPowerBrakeSlowdown"))
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []          # (time, sm_mhz, max_mhz, [reason names])
        self.source = "none"
        self._stop = threading.Event()
        self.thread = None
        self.proc = None

    def _nvml_handle(self, nv):
        try:
            pr = torch.cuda.get_device_properties(self.cuda_index)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return nv.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._nvml_handle(nv)
            mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            bits = [(name, getattr(nv, "nvmlClocksEventReason" + suffix, 0)) for name, suffix in self.REASONS]
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons

            def loop():
                while not self._stop.is_set():
                    try:
                        mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        r = get_reasons(h)
                    except Exception:
                        break
                    self.samples.append((time.time(), mhz, mx, [n for n, b in bits if b and (r & b)]))
                    time.sleep(0.001)
            self.source = "nvml"
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.cuda_index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            return
        self.source = "nvidia-smi"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

        def read():
            for line in self.proc.stdout:
                parts = [x.strip() for x in line.split(",")]
                try:
                    self.samples.append((time.time(), float(parts[1]), float(parts[2]),
                                         [n for n, v in zip(names, parts[5:9]) if v.lower() == "active"]))
                except (ValueError, IndexError):
                    continue
        self.thread = threading.Thread(target=read, daemon=True)
        self.thread.start()

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float):
        rows = list(self.samples)
        inside = [r for r in rows if t0 <= r[0] <= t1]
        used = inside if inside else sorted(rows, key=lambda r: min(abs(r[0] - t0), abs(r[0] - t1)))[:3]
        if not used:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0,
                    "source": self.source}
        mhz = sorted(r[1] for r in used)
        reasons = sorted({n for r in used for n in r[3]})
        return {"sm_mhz": mhz[len(mhz) // 2], "sm_max_mhz": max(r[2] for r in used), "reasons": reasons,
                "samples": len(used), "samples_in_window": len(inside), "source": self.source}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
# sources of the tensor-core kernel the bench times (the traffic figure in
# profiles/traffic.json is valid only for these exact sources)
TC_SOURCES = ("flash_tc.cu", "common.cuh", "sm100.cuh", "softmax_tile.cuh", "tmap.h")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "attention_sdpa_fwd_b200", "csrc")
    for name in TC_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_hash: str, workload: str):
    """Per-launch DRAM bytes of the dominant kernel from the committed ncu
    summary, or None when absent or taken on a different kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel_source_hash") != kernel_hash:
        return None
    return e.get("dram_bytes_per_launch")


def make_device_sets(spec: W.Spec, device, nsets: int, seed_base: int):
    sets = []
    for s in range(nsets):
        wl = W.make(spec, seed=seed_base + s)
        t = lambda x: None if x is None else x.to(device, non_blocking=False).contiguous()
        sets.append(dict(q=t(wl.q), k=t(wl.k), v=t(wl.v), rh=t(wl.rel_pos_h), rw=t(wl.rel_pos_w),
                         mask=t(wl.mask), out=torch.empty_like(wl.q, device=device)))
    return sets


def launch(S, spec: W.Spec, st, stream, path):
    m = S.make_mask(spec.mask_kind, offset=spec.offset, window=spec.window, tensor=st["mask"])
    import ctypes
    rc = S.sdpa_fwd_ex(st["q"].data_ptr(), st["k"].data_ptr(), st["v"].data_ptr(), st["out"].data_ptr(),
                       S.SDPA_BF16 if spec.dtype == torch.bfloat16 else S.SDPA_F32,
                       spec.B, spec.Hq, spec.Hkv, spec.Tq, spec.Tkv, spec.d, spec.scale, spec.mask_kind,
                       ctypes.byref(m) if m is not None else None,
                       st["rh"].data_ptr() if st["rh"] is not None else None,
                       st["rw"].data_ptr() if st["rw"] is not None else None,
                       spec.q_hw, spec.k_hw, None, path, stream.cuda_stream)
    if rc != 0:
        raise RuntimeError(f"sdpa_fwd_ex failed: {S.STATUS.get(rc, rc)}")


def auto_path_name(S, spec: W.Spec) -> str:
    """The kernel family AUTO dispatches this workload to (host-side query: the
    library validates but never dereferences the placeholder addresses, which
    are 2^40 bytes apart so that no two spans overlap)."""
    import ctypes
    base = 1 << 40
    data = base * 7 if spec.mask_kind in (W.MASK_FLOAT, W.MASK_BOOL) else None
    m = None
    if spec.mask_kind != W.MASK_NONE:
        m = S.sdpa_mask_t(offset=spec.offset, window=spec.window, data=data)
        if data is not None:  # strides of the workload's contiguous [B, mask_heads, Tq, Tkv] mask
            m.stride_b = 0 if spec.B == 1 else spec.mask_heads * spec.Tq * spec.Tkv
            m.stride_h = 0 if spec.mask_heads == 1 else spec.Tq * spec.Tkv
            m.stride_q = spec.Tkv
    rel = spec.q_hw is not None
    rc = S.sdpa_select_path(base, base * 2, base * 3, base * 4,
                            S.SDPA_BF16 if spec.dtype == torch.bfloat16 else S.SDPA_F32,
                            spec.B, spec.Hq, spec.Hkv, spec.Tq, spec.Tkv, spec.d, spec.mask_kind,
                            ctypes.byref(m) if m is not None else None,
                            base * 5 if rel else None, base * 6 if rel else None, spec.q_hw, spec.k_hw)
    names = {v: k for k, v in S.PATHS.items()}
    return names.get(rc, f"status {rc}")


def n_input_sets(spec: W.Spec) -> int:
    """Input sets to rotate so that consecutive launches never find their
    inputs in the 126 MB L2 (together at least twice its size)."""
    return min(64, max(2, math.ceil(2 * L2_BYTES / max(spec.bytes(), 1))))


def time_workload(S, spec: W.Spec, device, steps: int, warmup: int, rank: int, ws: int, path=0, sets=None,
                  per_launch: bool = True):
    """K launches back to back on the current stream between two CUDA events.
    ``per_launch`` also brackets every launch with its own pair of events
    (for a per-launch median).  Those events sit between consecutive
    launches, so the headline measurement leaves them out: its launches follow
    one another as a caller's consecutive calls on a stream do."""
    per_set = spec.bytes()
    if sets is None:
        sets = make_device_sets(spec, device, n_input_sets(spec), seed_base=spec.seed + 1000 * rank)
    nsets = len(sets)
    stream = torch.cuda.current_stream(device)
    for i in range(warmup):
        launch(S, spec, sets[i % nsets], stream, path)
    torch.cuda.synchronize(device)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    t0 = time.time()
    e0.record(stream)
    for i in range(steps):
        if per_launch:
            starts[i].record(stream)
        launch(S, spec, sets[i % nsets], stream, path)
        if per_launch:
            ends[i].record(stream)
    e1.record(stream)
    torch.cuda.synchronize(device)
    t1 = time.time()
    if ws > 1:
        torch.distributed.barrier()
    total_ms = e0.elapsed_time(e1)
    launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)] if per_launch else [total_ms / steps] * steps
    return dict(total_ms=total_ms, launch_ms=launch_ms, t0=t0, t1=t1, nsets=nsets,
                set_bytes=per_set)


def time_graph(S, spec: W.Spec, device, launches: int = 40, reps: int = 5, sets=None):
    """Per-launch device time from CUDA-graph replays of `launches` back-to-back
    launches (rotating input sets): strips the host launch overhead that
    dominates per-launch events for the microsecond-sized workloads."""
    if sets is None:
        sets = make_device_sets(spec, device, n_input_sets(spec), seed_base=spec.seed)
    nsets = len(sets)
    side = torch.cuda.Stream(device)
    with torch.cuda.stream(side):
        for i in range(3):
            launch(S, spec, sets[i % nsets], side, 0)
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for i in range(launches):
            launch(S, spec, sets[i % nsets], side, 0)
    g.replay()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize(device)
    return e0.elapsed_time(e1) / (reps * launches)


def time_e2e(S, spec: W.Spec, device, steps: int, warmup: int):
    """Same forward through the host-buffer C entry point: pinned host inputs,
    H2D copies, kernel, D2H copy of the output, all inside the timed region."""
    wl = W.make(spec, seed=spec.seed + 777)
    pin = lambda x: None if x is None else x.contiguous().pin_memory()
    q, k, v, rh, rw = (pin(x) for x in (wl.q, wl.k, wl.v, wl.rel_pos_h, wl.rel_pos_w))
    out = torch.empty_like(q).pin_memory()
    stream = torch.cuda.current_stream(device)
    import ctypes
    mask_h = pin(wl.mask)
    m = None
    if spec.mask_kind != W.MASK_NONE:
        m = S.sdpa_mask_t(offset=spec.offset, window=spec.window, data=None, stride_b=0, stride_h=0, stride_q=0)
        if mask_h is not None:
            m.data = mask_h.data_ptr()
            m.stride_b = 0 if mask_h.shape[0] == 1 else mask_h.stride(0)
            m.stride_h = 0 if mask_h.shape[1] == 1 else mask_h.stride(1)
            m.stride_q = mask_h.stride(2)

    def call():
        rc = S.sdpa_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             S.SDPA_BF16 if spec.dtype == torch.bfloat16 else S.SDPA_F32,
                             spec.B, spec.Hq, spec.Hkv, spec.Tq, spec.Tkv, spec.d, spec.scale, spec.mask_kind,
                             ctypes.byref(m) if m is not None else None,
                             rh.data_ptr() if rh is not None else None,
                             rw.data_ptr() if rw is not None else None,
                             spec.q_hw, spec.k_hw, 0, stream.cuda_stream)
        if rc != 0:
            raise RuntimeError(f"sdpa_fwd_host failed: {S.STATUS.get(rc, rc)}")

    for _ in range(warmup):
        call()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / steps
    h2d = sum(x.numel() * x.element_size() for x in (q, k, v, rh, rw, mask_h) if x is not None)
    d2h = out.numel() * out.element_size()
    return ms, h2d, d2h


def time_pinned_copies(device, h2d_bytes: int, d2h_bytes: int, reps: int = 10):
    """The box's own floor for the host-buffer call: plain pinned copies of the
    same byte counts (one upload of h2d_bytes, one download of d2h_bytes), on
    one stream, timed with CUDA events (median of reps)."""
    up_h = torch.empty(h2d_bytes, dtype=torch.uint8).pin_memory()
    down_h = torch.empty(d2h_bytes, dtype=torch.uint8).pin_memory()
    up_d = torch.empty(h2d_bytes, dtype=torch.uint8, device=device)
    down_d = torch.empty(d2h_bytes, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def med(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize(device)
        ts = []
        for _ in range(reps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(device)
            ts.append(a.elapsed_time(b))
        return sorted(ts)[len(ts) // 2]
    up_ms = med(lambda: up_d.copy_(up_h, non_blocking=True))
    down_ms = med(lambda: down_h.copy_(down_d, non_blocking=True))
    return up_ms, down_ms


# What bounds each workload's kernel (the algorithmic work counts live in
# workloads.Spec.flops / bytes): the dense contractions run against the bf16
# tensor peak, the streaming shapes against HBM bandwidth, and the two tiny
# problems (33 KB) are latency-bound and reported in microseconds only.
BOUND = {"tiny_relpos_f32": "latency", "sam_global": "tensor", "sam_windowed": "hbm",
         "decoder_token_to_image": "hbm", "decoder_image_to_token": "hbm", "decoder_self": "latency",
         "gqa_causal": "tensor", "gqa_sliding": "tensor", "gqa_float_mask": "tensor"}


def bias_name(spec: W.Spec) -> str:
    parts = []
    if spec.rel:
        parts.append("decomposed rel-pos")
    if spec.mask_kind != W.MASK_NONE:
        m = W.MASK_NAMES[spec.mask_kind]
        if spec.mask_kind == W.MASK_SLIDING:
            m += f" w={spec.window}"
        parts.append(m + " mask")
    return " + ".join(parts) if parts else "none"


def dtype_name(spec: W.Spec) -> str:
    return "bf16" if spec.dtype == torch.bfloat16 else "f32"


def time_copy_floor(device, nbytes: float, launches: int = 40, reps: int = 3) -> float:
    """Per-copy device time (us) of a plain device-to-device copy that reads
    and writes nbytes / 2 each, in CUDA-graph replays of back-to-back copies
    over rotating buffers larger than L2 in all: the practical floor of a
    memory-bound launch of that much traffic on this GPU."""
    n = max(16, int(nbytes / 2) // 16 * 16)
    nbuf = min(16, max(2, math.ceil(2 * L2_BYTES / n)))
    src = [torch.empty(n, dtype=torch.uint8, device=device) for _ in range(nbuf)]
    dst = [torch.empty(n, dtype=torch.uint8, device=device) for _ in range(nbuf)]
    side = torch.cuda.Stream(device)
    with torch.cuda.stream(side):
        for i in range(3):
            dst[i % nbuf].copy_(src[i % nbuf])
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for i in range(launches):
            dst[i % nbuf].copy_(src[i % nbuf])
    g.replay()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize(device)
    return e0.elapsed_time(e1) / (reps * launches) * 1e3


def per_config_table(S, device, peaks, steps: int):
    """Every benchmark workload through AUTO: median per-launch CUDA-event time
    (rotating inputs larger than L2), per-launch time from CUDA-graph replays,
    and the fraction of the workload's roofline (bf16 burst tensor peak or HBM
    copy bandwidth) from the graph time."""
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    bf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    table = {}
    for name, sp in W.SPECS.items():
        sets = make_device_sets(sp, device, n_input_sets(sp), seed_base=sp.seed + 500)
        rr = time_workload(S, sp, device, steps, 3, 0, 1, sets=sets)
        lm = sorted(rr["launch_ms"])[len(rr["launch_ms"]) // 2]
        gm = time_graph(S, sp, device, launches=20 if sp.flops() > 1e11 else 40, reps=3, sets=sets)
        del sets
        torch.cuda.empty_cache()
        tf = sp.flops() / (gm * 1e-3) / 1e12
        gbs = sp.bytes() / (gm * 1e-3) / 1e9
        bound = BOUND.get(name, "tensor")
        e = dict(path=auto_path_name(S, sp), bias=bias_name(sp), dtype=dtype_name(sp),
                 us_events_median=lm * 1e3, us_graph=gm * 1e3, flops=sp.flops(), bytes=sp.bytes(),
                 tflops=tf, gbs=gbs, bound=bound)
        if bound == "tensor":
            e.update(frac=tf / bf, peak=bf, peak_unit="TFLOP/s")
        elif bound == "hbm":
            e.update(frac=gbs / hbm, peak=hbm, peak_unit="GB/s")
            # context for the HBM fraction of a few-MB launch: a plain copy of the same traffic
            cu = time_copy_floor(device, sp.bytes())
            e.update(copy_floor_us=cu, copy_floor_frac_hbm=sp.bytes() / (cu * 1e-6) / 1e9 / hbm,
                     us_graph_over_copy_floor=gm * 1e3 / cu)
        else:
            e.update(frac=None, peak=None, peak_unit=None)
        table[name] = e
    return table


_WL_CACHE = {}


def cpu_oracle_sample(spec: W.Spec, budget_s: float = 12.0):
    """Time the fp64 oracle on the host cores on a bounded row sample."""
    import oracle
    if spec.name not in _WL_CACHE:
        _WL_CACHE[spec.name] = W.make(spec)
    wl = _WL_CACHE[spec.name]
    kw = dict(mask_kind=spec.mask_kind, offset=spec.offset, window=spec.window)
    if spec.mask_kind in (W.MASK_FLOAT, W.MASK_BOOL):
        kw["mask"] = wl.mask
    if spec.rel:
        kw.update(rel_pos_h=wl.rel_pos_h, rel_pos_w=wl.rel_pos_w, q_hw=spec.q_hw, k_hw=spec.k_hw)
    # probe with a small sample, then size the real one to about budget_s:
    # a row subset when the whole workload takes longer, else whole passes
    probe = list(range(0, spec.Tq, max(1, spec.Tq // 16)))
    t = time.time()
    oracle.sdpa(wl.q, wl.k, wl.v, spec.scale, rows=probe, **kw)
    dt = max(time.time() - t, 1e-4)
    per_row = dt / len(probe)
    nrows = int(min(spec.Tq, max(len(probe), budget_s / per_row)))
    stride = max(1, spec.Tq // nrows)
    rows = list(range(0, spec.Tq, stride))[:nrows]
    passes = 1
    t = time.time()
    if len(rows) == spec.Tq:
        rows = None
        oracle.sdpa(wl.q, wl.k, wl.v, spec.scale, **kw)
        passes = max(1, int(round(budget_s / max(time.time() - t, 1e-4))))
        for _ in range(passes - 1):
            oracle.sdpa(wl.q, wl.k, wl.v, spec.scale, **kw)
    else:
        oracle.sdpa(wl.q, wl.k, wl.v, spec.scale, rows=rows, **kw)
    sec = time.time() - t
    nr = spec.Tq if rows is None else len(rows)
    flops = spec.flops() * nr / spec.Tq * passes
    what = (f"{passes} full pass(es) of the workload" if rows is None else
            f"all {spec.B * spec.Hq} (b,h) x {nr} of {spec.Tq} query rows")
    return dict(value=flops / sec / 1e12, unit="TFLOP/s", cores=oracle.num_threads(), kind="oracle",
                sample=f"{spec.name}: {what} (fp64, {sec:.1f} s)", seconds=sec)


def run_profile_launches(args):
    """Untimed launches for an ncu capture: one input set of the workload with
    its batch scaled by --batch-mult (so a small case can still exceed L2),
    --profile-launches calls, then the device error word.  Prints one status
    line, not a bench line."""
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    import attention_sdpa_fwd_b200 as S
    S.lib()
    spec = W.spec_named(args.workload)
    spec = W.scaled(spec, B=args.batch if args.batch > 0 else spec.B * args.batch_mult)
    st = make_device_sets(spec, device, 1, seed_base=spec.seed)[0]
    stream = torch.cuda.current_stream(device)
    for _ in range(args.profile_launches):
        launch(S, spec, st, stream, 0)
    torch.cuda.synchronize(device)
    rc = S.sdpa_last_device_error(stream.cuda_stream)
    print(f"profile launches: {spec.name} B={spec.B} x{args.profile_launches} "
          f"({spec.bytes() / 1e6:.1f} MB per launch) device error {rc}", flush=True)
    if rc != 0:
        sys.exit(1)


def run_ours(args):
    ws, rank, local = dist_env()
    if ws > 1:
        torch.cuda.set_device(local)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import attention_sdpa_fwd_b200 as S
    from attention_sdpa_fwd_b200 import build
    if rank == 0 or ws == 1:
        pass
    S.lib()  # fails loudly if the extension is missing
    peaks, peaks_src = load_peaks()
    spec = W.spec_named(args.workload)

    sampler = ClockSampler(torch.cuda.current_device() if ws == 1 else local)
    sampler.start()
    time.sleep(0.3)
    # one step = one launch; the K steps run back to back between two events,
    # as a caller's consecutive calls on a stream would
    r = time_workload(S, spec, device, args.steps, args.warmup, rank, ws, per_launch=False)
    clocks = sampler.summary(r["t0"], r["t1"])
    sampler.stop()

    ms = r["total_ms"] / args.steps
    launch_avg = sum(r["launch_ms"]) / len(r["launch_ms"])
    ms, launch_avg = max_over_ranks([ms, launch_avg], device)
    flops = spec.flops()
    value = aggregate_throughput(flops, ms, ws)

    e2e_ms, h2d, d2h = time_e2e(S, spec, device, max(3, min(args.steps, 20)), 2)
    e2e_ms, = max_over_ranks([e2e_ms], device)
    e2e = aggregate_throughput(flops, e2e_ms, ws)
    up_ms, down_ms = time_pinned_copies(device, int(h2d), int(d2h))

    per_config = {}
    if not args.no_per_config and ws == 1:
        per_config = per_config_table(S, device, peaks, max(10, args.steps))

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_sample(spec, budget_s=args.cpu_budget)
        cpu.pop("seconds", None)

    bound = BOUND.get(spec.name, "tensor")
    if bound == "hbm":
        achieved = spec.bytes() / (launch_avg * 1e-3) / 1e9
        peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        r_unit, peak_key = "GB/s", "hbm_gbs (copy)"
    else:
        achieved = flops / (launch_avg * 1e-3) / 1e12
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        r_unit, peak_key = "TFLOP/s", "bf16_tflops (burst)"
    khash = kernel_source_hash()
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dtype_name(spec),
        "data": f"synthetic (seeded normal q, k, v with std {spec.qkv_std:.3g}"
                + (f"; rel-pos tables std {spec.rel_std}" if spec.rel else "") + ")",
        "config": {"workload": spec.name, "B": spec.B, "H": spec.Hq, "Hkv": spec.Hkv, "Tq": spec.Tq,
                   "Tkv": spec.Tkv, "head_dim": spec.d,
                   "grid": list(spec.q_hw) if spec.q_hw else None, "bias": bias_name(spec),
                   "l2": f"{r['nsets']} rotating input sets of {r['set_bytes'] / 1e6:.1f} MB (> L2)",
                   "parallelism": f"replica x{ws} (independent problems per GPU)"},
        "roofline": {"bound": "tensor" if bound != "hbm" else "hbm", "achieved": achieved, "peak": peak,
                     "unit": r_unit, "frac": achieved / peak, "peak_source": f"{peaks_src} {peak_key}",
                     "traffic": ncu_traffic(khash, spec.name),
                     "flops_per_launch": flops, "launch_ms": launch_avg,
                     "frac_of_spec_sheet": achieved / (7700.0 if bound == "hbm" else 2250.0)},
        "e2e": {"value": e2e, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms,
                # plain pinned copies of the same bytes on this machine: the transfer floor of the call
                "pinned_upload_ms": up_ms, "pinned_download_ms": down_ms,
                "pinned_h2d_gbs": h2d / (up_ms * 1e-3) / 1e9, "pinned_d2h_gbs": d2h / (down_ms * 1e-3) / 1e9,
                "ms_over_serial_copy_floor": e2e_ms / (up_ms + down_ms)},
        "cpu_baseline": cpu,
        "gpu_launches": args.steps,
        "clocks": clocks,
        "kernel_source_hash": khash,
    }
    if per_config:
        line["per_config"] = per_config
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_reference(args):
    ws, rank, local = dist_env()
    if rank != 0:
        return
    spec = W.spec_named(args.workload)
    vals = []
    info = None
    # about 150 s of oracle work in all, whatever --steps / --warmup ask for
    budget = max(0.1, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    for i in range(args.warmup + args.steps):
        info = cpu_oracle_sample(spec, budget_s=budget)
        if i >= args.warmup:
            vals.append(info["value"])
    value = sum(vals) / len(vals)
    secs = info.pop("seconds")
    info["value"] = value
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": secs * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": spec.name, "B": spec.B, "H": spec.Hq, "T": spec.Tq, "head_dim": spec.d},
        "cpu_baseline": info,
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="sam_global", choices=sorted(W.SPECS) + sorted(W.EXTRA_SPECS))
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-workload table (every benchmark workload timed through AUTO)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--profile-launches", type=int, default=0,
                    help="only run this many untimed launches (for ncu) and exit")
    ap.add_argument("--batch-mult", type=int, default=1,
                    help="with --profile-launches: multiply the workload's batch")
    ap.add_argument("--batch", type=int, default=0,
                    help="with --profile-launches: set the workload's batch (overrides --batch-mult)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.profile_launches > 0:
        run_profile_launches(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
