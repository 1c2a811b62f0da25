#!/usr/bin/env python3
"""Benchmark of sparse-mask scaled dot-product attention on B200.

One step = the whole hot path over one batch of synthetic input: build the mask
on the device from its pattern parameters (with its row schedule and tile
plan), then the fused forward (scores on the mask's nonzeros + additive
mask/bias, running max/sum softmax, weighted sum of V, normalisation, out +
lse).

Default workload: block-local + strided + global tokens, B=1, H=16, n=16384,
d=128, bf16 Q/K/V ~ N(0, 0.5^2); mask = same 64-token block, j = i (mod 128),
and the first 32 tokens global (the largest of the five workloads).

Metric: masked-attention TFLOP/s = 4 * nnz * d / step time, nnz summed over
(b, h). ``--impl reference`` times the fp64 CPU oracle on the host cores instead.
Multi-GPU (torchrun): independent replicas, one per GPU (no collective on the
data path); ``value`` is the work of all ranks over the slowest rank's time.

Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "masked-attention TFLOP/s (4*nnz*d)"
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=3, help="workload index 0..5 (default 3)")
    ap.add_argument("--settle-seconds", type=float, default=1.0,
                    help="untimed load before the warm-up, so the clock sampler sees the GPU under load")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads' forward timings")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-baseline sample budget")
    return ap.parse_args()


def measured_peaks():
    """(HBM GB/s, dense bf16 TFLOP/s burst, source): the measured copy
    bandwidth and cuBLAS bf16 GEMM of this machine's B200s, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 1590.0)), "measured"
    return 6650.0, 1590.0, "fallback"


SMS = 148
MUFU_EX2_PER_CLK_PER_SM = 16   # B200 special-function unit: 4 per SM sub-partition


def mask_nnz_total(wl, nnz_per_mask):
    """nnz summed over every (b, h): each batch element uses its mask, every head shares it."""
    if wl.mask.num_masks == 1:
        return int(nnz_per_mask[0]) * wl.B * wl.H
    return int(sum(nnz_per_mask)) * wl.H


def effective_bytes(wl, nnz_total):
    """The per-nonzero operand bytes of the method (what a gather of every
    nonzero's rows moves): per nonzero a K row and a V row plus the column
    index (plus one mask and one bias element when present); per query row q_i,
    out_i, lse_i and its row pointer. Kernels that reuse rows from L1/L2, or
    compute whole tiles, move far fewer DRAM bytes than this."""
    es = 2 if wl.dtype == workloads.BF16 else 4
    per_nnz = 2 * wl.d * es + 4
    if wl.add_mask is not None:
        per_nnz += 2 if wl.add_mask.dtype == workloads.BF16 else 4
    if wl.bias is not None:
        per_nnz += 2 if wl.bias.dtype == workloads.BF16 else 4
    rows = wl.B * wl.H * wl.n
    return nnz_total * per_nnz + rows * (2 * wl.d * es + 4 + 4), per_nnz


def compulsory_bytes(wl, nnz_masks):
    """Bytes a forward cannot avoid moving through HBM: Q, K, V read and out
    written once, lse written, the additive mask and bias read once as stored,
    and the mask as the path stores it (a CSR: row pointers + column indices;
    an interval mask: one [lo, hi) pair per row; a closed-form pattern:
    nothing)."""
    es = 2 if wl.dtype == workloads.BF16 else 4
    rows = wl.B * wl.H * wl.n
    b = 4 * rows * wl.d * es + 4 * rows
    for t in (wl.add_mask, wl.bias):
        if t is not None:
            b += t.raw.nbytes
    mrows = wl.mask.num_masks * wl.n
    if wl.mask.kind in ("sliding", "varwin", "dense"):
        b += 8 * mrows
    elif wl.mask.kind in ("coo", "csr"):
        b += 4 * (mrows + 1) + 4 * nnz_masks
    return b


def roofline_entry(wl, t_ms, nnz_total, tiles_total, hbm_peak, tc_peak, peak_src, clk_mhz, kernel,
                   traffic=None, t_warm_ms=None):
    """Roofline of one forward launch: its algorithmic work (4*nnz*d FLOPs,
    the compulsory bytes) over the measured time against the measured peaks.
    ``bound`` follows the arithmetic intensity of that work: below the ridge
    (peak FLOP/s over peak bytes/s) the forward is bound by HBM, above it by
    the tensor cores. Beside it, the fractions of each unit the kernels drive:
    the MMA work executed (whole 128 x 128 tiles, two MMAs each), the exp count
    on the special-function unit (an upper bound: every element of every tile;
    the kernels skip 32-key chunks that hold no entry) and, for gathered
    entries, the per-nonzero effective bytes (served mostly by L2)."""
    t = t_ms * 1e-3
    flops = 4.0 * nnz_total * wl.d
    comp = compulsory_bytes(wl, nnz_total // (wl.B * wl.H if wl.mask.num_masks == 1 else wl.H))
    eff, per_nnz = effective_bytes(wl, nnz_total)
    mma = tiles_total * 4.0 * 128 * 128 * wl.d
    ex2_ub = tiles_total * 128.0 * 128
    clk = (clk_mhz or 1965.0) * 1e6
    intensity = flops / comp
    ridge = tc_peak * 1e12 / (hbm_peak * 1e9)
    bound = "tensor" if intensity > ridge else "hbm"
    src = "measured MEASURED_PEAKS.json" if peak_src == "measured" else "fallback"
    if bound == "tensor":
        achieved, peak, unit = flops / t / 1e12, tc_peak, "TFLOP/s"
        psrc = f"bf16_tflops ({src}, burst: the kernel runs for well under a second)"
    else:
        achieved, peak, unit = comp / t / 1e9, hbm_peak, "GB/s"
        psrc = f"hbm_gbs ({src})"
    e = {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
         "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": kernel,
         "algorithmic_flop_per_launch": flops, "compulsory_bytes_per_launch": int(comp),
         "arithmetic_intensity_flop_per_byte": round(intensity, 1), "ridge_flop_per_byte": round(ridge, 1),
         "fwd_ms": round(t_ms, 4), "peak_source": psrc,
         "fractions": {
             "useful_flop_of_bf16_peak": round(flops / t / 1e12 / tc_peak, 4),
             "executed_mma_of_bf16_peak": round(mma / t / 1e12 / tc_peak, 4),
             "compulsory_bytes_of_hbm_peak": round(comp / t / 1e9 / hbm_peak, 4),
             "ex2_upper_bound_of_mufu_peak": round(ex2_ub / t / (SMS * MUFU_EX2_PER_CLK_PER_SM * clk), 4),
         },
         "tc_tiles_per_launch": int(tiles_total), "mma_flop_executed_per_launch": mma}
    if t_warm_ms is not None:
        e["fwd_ms_warm_l2"] = round(t_warm_ms, 4)
    if tiles_total == 0:   # every entry gathered: the per-nonzero operand bytes, L2-served
        e["effective_gbs_l2_served"] = round(eff / t / 1e9, 1)
        e["effective_bytes_per_nnz"] = per_nnz
    return e


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples every 20 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_id: str):
        self.device_id = device_id
        self.proc = None
        self.lines = []
        self.start = 0
        self.end = None

    def mark(self):
        """Only samples taken after this call (and before the sampler stops) count."""
        self.start = len(self.lines)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20", "-i", self.device_id],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            # let nvidia-smi finish starting up (NVML initialisation) before the
            # timed region, so that it does not stall the first timed step
            t0 = time.perf_counter()
            while not self.lines and time.perf_counter() - t0 < 3.0:
                time.sleep(0.01)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        self.end = len(self.lines)  # samples after this are of an idle GPU
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        window = self.lines[self.start:self.end]
        for ln in window if window else self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- traffic
# source files (under sparse_mask_scaled_b200/csrc) whose contents a kernel's
# ncu summary was taken on: the kernel's own file and the headers it includes
KERNEL_SOURCES = {
    "k_fwd_pp": ["fwd_pp.cu", "bsg_plan.cuh", "sm100_ptx.cuh", "spattn_internal.cuh"],
    "k_fwd_tc": ["fwd_tc.cu", "sm100_ptx.cuh", "spattn_internal.cuh"],
    "k_fwd_tc_quad": ["fwd_tc.cu", "sm100_ptx.cuh", "spattn_internal.cuh"],
    "k_fwd_short": ["fwd_gather.cu", "spattn_internal.cuh"],
}


def kernel_source_hash(base: str):
    """First 16 hex digits of the SHA-256 over the kernel's source files in
    order (None for a kernel not listed)."""
    files = KERNEL_SOURCES.get(base)
    if not files:
        return None
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "sparse_mask_scaled_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload (profiles/<kernel base name>_<workload>.md), or None when there is
    none or the kernel's sources changed since the capture."""
    base = kernel.split("<")[0]
    path = os.path.join(ROOT, "profiles", f"{base}_{workload}.md")
    want = kernel_source_hash(base)
    if not want or not os.path.exists(path):
        return None
    vals = {}
    for ln in open(path):
        if ":" in ln and ln.strip().startswith("- "):
            k, v = ln.strip()[2:].split(":", 1)
            v = v.strip()
            if v.startswith("`"):  # `value` (note)
                v = v[1:].split("`", 1)[0]
            vals[k.strip()] = v
    if vals.get("source_sha256_16") != want:
        return None
    try:
        return int(float(vals["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- CPU side
def cpu_oracle_rate(wl, seconds: float, threads: int):
    """Time the oracle (as it stands) on a bounded random sample of the
    workload's rows; returns (TFLOP/s, rows, nnz, elapsed)."""
    import oracle
    rp, ci = oracle.mask_from_params(wl.mask)
    lens = np.diff(rp)
    B, H, n = wl.B, wl.H, wl.n
    rng = np.random.default_rng(12345)
    total_rows = B * H * n

    def run(rows):
        t0 = time.perf_counter()
        oracle.masked_sdpa(wl.q.raw, wl.k.raw, wl.v.raw, rp, ci, wl.mask.num_masks, wl.scale,
                           add_mask=None if wl.add_mask is None else wl.add_mask.raw,
                           bias=None if wl.bias is None else wl.bias.raw, rows=rows,
                           threads=threads)
        return time.perf_counter() - t0

    def nnz_of(rows):
        bh, i = rows // n, rows % n
        b = bh // H
        m = b if wl.mask.num_masks > 1 else np.zeros_like(b)
        return int(lens[m * n + i].sum())

    probe = np.sort(rng.choice(total_rows, size=min(total_rows, 512), replace=False))
    t = run(probe)
    per_row = max(t / probe.size, 1e-7)
    count = int(min(total_rows, max(probe.size, seconds / per_row)))
    rows = np.sort(rng.choice(total_rows, size=count, replace=False))
    t = run(rows)
    nz = nnz_of(rows)
    return 4.0 * nz * wl.d / t / 1e12, count, nz, t


def cpu_model():
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ---------------------------------------------------------------- GPU side
def _to_device(t, torch):
    if t.dtype == workloads.BF16:
        x = torch.from_numpy(np.ascontiguousarray(t.raw).view(np.int16)).view(torch.bfloat16)
    else:
        x = torch.from_numpy(np.ascontiguousarray(t.raw))
    return x.cuda()


class GpuWorkload:
    def __init__(self, wl, torch, sp):
        self.wl, self.torch, self.sp = wl, torch, sp
        self.q, self.k, self.v = (_to_device(x, torch) for x in (wl.q, wl.k, wl.v))
        self.am = _to_device(wl.add_mask, torch) if wl.add_mask is not None else None
        self.bias = _to_device(wl.bias, torch) if wl.bias is not None else None
        mp = wl.mask
        self.hw = self.crp = self.ccols = None
        if mp.kind == "varwin":
            self.hw = torch.from_numpy(np.ascontiguousarray(mp.half_widths, np.int32).ravel()).cuda()
        if mp.kind == "coo":
            self.crp = torch.from_numpy(mp.cand_row_ptr.astype(np.int32)).cuda()
            self.ccols = torch.from_numpy(mp.cand_cols.astype(np.int32)).cuda()
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(wl.B * wl.H * wl.n, dtype=torch.float32, device="cuda")

    def create(self, hw=None, crp=None, ccols=None, tile_min_nnz=0):
        mp = self.wl.mask
        return self.sp.spattn_create_csr_mask(
            mp.kind, mp.n, mp.num_masks, window=mp.window, block=mp.block, stride=mp.stride,
            n_global=mp.n_global, add_diagonal=mp.add_diagonal,
            half_widths=self.hw if hw is None else hw,
            in_row_ptr=self.crp if crp is None else crp,
            in_col_idx=self.ccols if ccols is None else ccols, tile_min_nnz=tile_min_nnz,
            asynchronous=True)

    def fwd(self, m, q=None, k=None, v=None, out=None, lse=None):
        return self.sp.spattn_fwd_mask(self.q if q is None else q, self.k if k is None else k,
                                       self.v if v is None else v, m, add_mask=self.am,
                                       bias=self.bias, scale=self.wl.scale,
                                       out=self.out if out is None else out,
                                       lse=self.lse if lse is None else lse)


def replica_seed(config: int, rank: int) -> int:
    """Each rank runs its own replica of the workload (rank 0: the standard seed)."""
    return 1000 + config + 7919 * rank


def max_over_ranks(values, torch, device, world: int):
    """Element-wise maximum of per-rank timings (the slowest rank sets the time)."""
    if world <= 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_value(world: int, flop_per_step: float, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: the work of all ranks over the slowest rank's step time."""
    return world * flop_per_step / (ms_per_step * 1e-3) / 1e12


def kernel_name(wl, m_tiles):
    """The forward's dominant kernel for the workload (see the library's routing
    in spattn_fwd_mask_kpad: closed-form block + strided + global masks and
    d = 128 interval masks without additive terms take the persistent kernel,
    d <= 64 the four-CTAs-per-SM tile kernel, d = 128 with additive terms and
    CSR masks the per-block tile kernel)."""
    if m_tiles == 0 or wl.dtype != workloads.BF16:
        return f"k_fwd_short<{'bf16' if wl.dtype == workloads.BF16 else 'f32'},{wl.d}>"
    extra = wl.add_mask is not None or wl.bias is not None
    if wl.mask.kind in ("dense", "sliding", "varwin") and wl.d == 128 and not extra:
        return f"k_fwd_pp<{wl.d},0,0>"
    if wl.mask.kind == "bsg" and not extra and wl.d in (64, 128):
        return f"k_fwd_pp<{wl.d},0,1>"
    if wl.d <= 64:
        # with additive terms the bench's (bf16, aligned) per-row term is staged by TMA
        return f"k_fwd_tc_quad<{wl.d},{int(extra)},{int(extra)}>"
    return f"k_fwd_tc<{wl.d}>"


def time_forward(g, m, torch, flush, reps=20, warm=3):
    """Median forward time (ms) with L2 flushed before each call, and with L2
    warm (the same call repeated back to back)."""
    stream = torch.cuda.current_stream()
    for _ in range(warm):
        g.fwd(m)

    def once(do_flush):
        if do_flush:
            flush.zero_()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        g.fwd(m)
        e.record(stream)
        return s, e

    cold = [once(True) for _ in range(reps)]
    hot = [once(False) for _ in range(reps)]
    torch.cuda.synchronize()
    return (statistics.median(a.elapsed_time(b) for a, b in cold),
            statistics.median(a.elapsed_time(b) for a, b in hot))


def bench_ours(args, rank, world, torch, sp):
    dev = torch.cuda.current_device()
    wl = workloads.make(args.config, seed=replica_seed(args.config, rank))
    g = GpuWorkload(wl, torch, sp)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    # mask statistics (same for every step)
    with g.create() as m0:
        nnz_masks = m0.nnz
        tiles_masks = m0.tc_tiles
        plan = {"tensor_core_tiles": tiles_masks}
    rep = wl.B * wl.H if wl.mask.num_masks == 1 else wl.H   # every head shares its batch element's mask
    nnz_total = nnz_masks * rep
    tiles_total = tiles_masks * rep
    flops = 4.0 * nnz_total * wl.d

    def step():
        m = g.create()
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        g.fwd(m)
        ev1.record(stream)
        m.close()
        return ev0, ev1

    starts, ends, fwd_evs = [], [], []
    smi_id = _smi_id(torch, dev)
    with ClockSampler(smi_id) as clk:
        clk.mark()
        # untimed load first, long enough for the sampler to see the clocks
        # under this work, then the warm-up right before the timed steps
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < args.settle_seconds:
            for _ in range(20):
                step()
            torch.cuda.synchronize()
        for _ in range(args.warmup):
            flush.zero_()
            step()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        launches0 = sp.spattn_launch_count()
        for it in range(args.steps):
            flush.zero_()                      # evict L2 between steps (outside the events)
            if it == 0:
                # the GPU starts idle: a second flush gives the host time to queue
                # the first step, as it is ahead for every later one
                flush.zero_()
            s = torch.cuda.Event(enable_timing=True)
            e = torch.cuda.Event(enable_timing=True)
            s.record(stream)
            fwd_evs.append(step())
            e.record(stream)
            starts.append(s)
            ends.append(e)
        torch.cuda.synchronize()
    launches = sp.spattn_launch_count() - launches0    # kernels the library enqueued while timed
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    fwd_ms = [a.elapsed_time(b) for a, b in fwd_evs]
    t_total = sum(step_ms)
    t_fwd = sum(fwd_ms) / len(fwd_ms)
    with g.create() as mw:
        _, t_warm = time_forward(g, mw, torch, flush)

    # ---- end to end: pinned host inputs -> device -> step -> host result
    e2e = e2e_measure(args, g, torch, stream, flush, flops)

    t_max, e2e["ms_per_step"] = max_over_ranks([t_total, e2e["ms_per_step"]], torch, "cuda", world)
    ms_per_step = t_max / args.steps
    value = job_value(world, flops, ms_per_step)
    e2e_value = job_value(world, flops, e2e["ms_per_step"])

    hbm_peak, tc_peak, peak_src = measured_peaks()
    clocks = clk.summary()
    kname = kernel_name(wl, tiles_total)
    roofline = roofline_entry(wl, t_fwd, nnz_total, tiles_total, hbm_peak, tc_peak, peak_src,
                              clocks.get("sm_mhz"), kname, traffic=committed_traffic(kname, wl.name),
                              t_warm_ms=t_warm)

    result = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == workloads.BF16 else "f32",
        "data": "synthetic (seeded numpy PCG64; no dataset)",
        "config": {"workload": f"{wl.name} B={wl.B} H={wl.H} n={wl.n} d={wl.d}", "B": wl.B, "H": wl.H,
                   "n": wl.n, "d": wl.d, "mask": wl.mask.kind, "num_masks": wl.mask.num_masks,
                   "nnz_total": nnz_total, "flop_per_step": flops,
                   "l2": "flushed before every timed step (256 MiB write; twice before the first)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "step": "device mask build (pattern -> mask with row schedule and tile plan) + fused forward",
                   "clocks_window": f"{args.settle_seconds:.1f} s of untimed steps, the warm-up and the timed steps",
                   "plan_per_mask_set": plan},
        "step_ms": {"min": round(min(step_ms), 4), "median": round(statistics.median(step_ms), 4),
                    "max": round(max(step_ms), 4)},
        "fwd": {"ms": round(t_fwd, 4), "ms_warm_l2": round(t_warm, 4),
                "tflops": round(flops / (t_fwd * 1e-3) / 1e12, 3)},
        "roofline": roofline,
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": e2e["h2d"],
                "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": round(e2e["ms_per_step"], 4)},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    return result, wl


def e2e_measure(args, g, torch, stream, flush, flops):
    """Same step through the public API, with the inputs in pinned host memory
    copied in and the result (out and lse) copied back inside the timed region."""
    wl = g.wl
    hq, hk, hv = (x.to("cpu").pin_memory() for x in (g.q, g.k, g.v))
    hhw = g.hw.to("cpu").pin_memory() if g.hw is not None else None
    hcrp = g.crp.to("cpu").pin_memory() if g.crp is not None else None
    hcc = g.ccols.to("cpu").pin_memory() if g.ccols is not None else None
    hout = torch.empty(g.out.shape, dtype=g.out.dtype).pin_memory()
    hlse = torch.empty(g.lse.shape, dtype=g.lse.dtype).pin_memory()
    dq, dk, dv = torch.empty_like(g.q), torch.empty_like(g.k), torch.empty_like(g.v)
    dhw = torch.empty_like(g.hw) if g.hw is not None else None
    dcrp = torch.empty_like(g.crp) if g.crp is not None else None
    dcc = torch.empty_like(g.ccols) if g.ccols is not None else None
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hhw, hcrp, hcc) if x is not None)
    d2h = hout.numel() * hout.element_size() + hlse.numel() * hlse.element_size()

    def one():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        if dhw is not None:
            dhw.copy_(hhw, non_blocking=True)
        if dcrp is not None:
            dcrp.copy_(hcrp, non_blocking=True)
            dcc.copy_(hcc, non_blocking=True)
        m = g.create(hw=dhw, crp=dcrp, ccols=dcc)
        g.fwd(m, q=dq, k=dk, v=dv)
        m.close()
        hout.copy_(g.out, non_blocking=True)
        hlse.copy_(g.lse, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        one()
    torch.cuda.synchronize()
    times = []
    steps = max(3, min(args.steps, 10))
    for _ in range(steps):
        flush.zero_()
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        one()
        e.record(stream)
        e.synchronize()
        times.append(s.elapsed_time(e))
    return {"ms_per_step": sum(times) / len(times), "h2d": int(h2d), "d2h": int(d2h)}


def backward_timing(args, torch, sp):
    """The backward pass (spattn_bwd_mask) on the benchmark workload: the mask and
    the forward's out / lse are prepared once, then each timed call computes dq,
    dk, dv (and dbias when the workload has a bias) with L2 flushed before it.
    FLOPs are counted as 2.5 x the forward's (10 * nnz * d: the score and
    dout . v recomputed, and the dq, dk, dv products)."""
    wl = workloads.make(args.config, seed=replica_seed(args.config, 0))
    g = GpuWorkload(wl, torch, sp)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    gen = torch.Generator(device="cuda").manual_seed(5)
    dout = torch.randn(g.q.shape, generator=gen, device="cuda").to(g.q.dtype)
    with g.create() as m:
        nnz_total = m.nnz * (wl.B * wl.H if wl.mask.num_masks == 1 else wl.H)
        out, lse = g.fwd(m)
        dq, dk, dv = (torch.empty_like(g.q) for _ in range(3))
        dbias = torch.empty(g.bias.shape, dtype=torch.float32, device="cuda") if g.bias is not None else None

        def one():
            sp.spattn_bwd_mask(g.q, g.k, g.v, m, out, lse, dout, add_mask=g.am, bias=g.bias, scale=wl.scale,
                               dq=dq, dk=dk, dv=dv, dbias=dbias)
        for _ in range(3):
            one()
        ts = []
        for _ in range(10):
            flush.zero_()
            s = torch.cuda.Event(enable_timing=True)
            e = torch.cuda.Event(enable_timing=True)
            s.record(stream)
            one()
            e.record(stream)
            e.synchronize()
            ts.append(s.elapsed_time(e))
    t = statistics.median(ts)
    es = 2 if wl.dtype == workloads.BF16 else 4
    rows = wl.B * wl.H * wl.n
    # the method's bytes: per nonzero a K and a V row (row pass) and a Q and a dout
    # row (column pass) plus the two indices and lse_i, D_i; per row q, dout, out,
    # dq read/written once and k, v, dk, dv likewise, plus lse and D
    alg = nnz_total * (4 * wl.d * es + 16) + rows * (8 * wl.d * es + 12)
    hbm_peak, _, _ = measured_peaks()
    return {"workload": wl.name, "ms": round(t, 4), "flop": 10.0 * nnz_total * wl.d,
            "tflops": round(10.0 * nnz_total * wl.d / (t * 1e-3) / 1e12, 3),
            "effective_gbs": round(alg / (t * 1e-3) / 1e9, 1),
            "frac_hbm_effective": round(alg / (t * 1e-3) / 1e9 / hbm_peak, 4),
            "path": "CUDA cores: row pass (dq) + column pass over the transposed mask (dk, dv)"}


def key_padding_lengths(wl):
    """Per-batch key lengths when the workload's additive mask is a key-padding
    mask [B, 1, 1, n] of 0 then -inf, else None."""
    if wl.add_mask is None or wl.add_mask.raw.shape[1:3] != (1, 1):
        return None
    keep = wl.add_mask.f64()[:, 0, 0, :] == 0
    lengths = keep.sum(axis=1)
    if not np.array_equal(keep, np.arange(wl.n)[None, :] < lengths[:, None]):
        return None
    return [int(x) for x in lengths]


def fusion_ablation(args, torch, sp):
    """The fused gather forward (spattn_fwd) against the proposal's three separate
    stages (spattn_fwd_unfused) on the benchmark workload's CSR, both on CUDA
    cores, L2 flushed before each call; the unfused path's score buffer is the
    nnz-sized memory the fused one never allocates."""
    wl = workloads.make(args.config, seed=replica_seed(args.config, 0))
    g = GpuWorkload(wl, torch, sp)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    with g.create() as m:
        rp, ci = m.csr()
        nnz_mask = m.nnz
    nm = wl.mask.num_masks
    nnz_total = nnz_mask * (wl.B * wl.H if nm == 1 else wl.H)
    res = {}
    for name, fn in (("fused_gather", sp.spattn_fwd), ("unfused", sp.spattn_fwd_unfused)):
        call = lambda: fn(g.q, g.k, g.v, rp, ci, nm, add_mask=g.am, bias=g.bias, scale=wl.scale,
                          out=g.out, lse=g.lse)
        for _ in range(3):
            call()
        ts = []
        for _ in range(10):
            flush.zero_()
            s = torch.cuda.Event(enable_timing=True)
            e = torch.cuda.Event(enable_timing=True)
            s.record(stream)
            call()
            e.record(stream)
            e.synchronize()
            ts.append(s.elapsed_time(e))
        res[name + "_ms"] = round(statistics.median(ts), 4)
    res["fusion_speedup"] = round(res["unfused_ms"] / res["fused_gather_ms"], 3)
    res["unfused_score_buffer_bytes"] = 4 * nnz_total
    res["fused_state_bytes_per_row"] = 4 * (wl.d + 2)
    return res


def contiguous_runs(torch, sp):
    """Contiguous column runs two ways, on the variable-window workload (every row
    one run of up to 513 keys): gathered by the CUDA-core kernel (a mask built
    with tile_min_nnz < 0: each lane group loads its nonzeros' K and V rows into
    registers), and as the default 128 x 128 tiles whose K and V tiles TMA stages
    in shared memory for the tensor cores. Forward only, L2 flushed."""
    wl = workloads.make(1, seed=replica_seed(1, 0))
    g = GpuWorkload(wl, torch, sp)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    res = {"workload": wl.name}
    for name, tmn in (("gathered", -1), ("tma_staged_tiles", 0)):
        with g.create(tile_min_nnz=tmn) as m:
            res[name + "_ms"] = round(time_forward(g, m, torch, flush, reps=10)[0], 4)
    res["tiles_speedup"] = round(res["gathered_ms"] / res["tma_staged_tiles_ms"], 2)
    return res


def other_workloads(torch, sp, skip, clk_mhz):
    """Forward-only timings of the other workloads and the extra dense d = 128
    case (device-resident inputs; L2 flushed, and warm), each with its roofline."""
    res = {}
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    hbm_peak, tc_peak, peak_src = measured_peaks()
    for cfg in range(6):
        if cfg == skip:
            continue
        try:
            wl = workloads.make(cfg)
            g = GpuWorkload(wl, torch, sp)
            rep = wl.B * wl.H if wl.mask.num_masks == 1 else wl.H
            with g.create() as m:
                nnz_total = m.nnz * rep
                tiles_total = m.tc_tiles * rep if wl.dtype == workloads.BF16 else 0
                t, t_warm = time_forward(g, m, torch, flush)
                t_kpad = None
                lengths = key_padding_lengths(wl)
                if lengths is not None:   # the same forward with the padding given as lengths
                    sl = torch.tensor(lengths, dtype=torch.int32, device="cuda")

                    class K:
                        def fwd(self_, mm):
                            sp.spattn_fwd_mask_kpad(g.q, g.k, g.v, mm, sl, bias=g.bias, scale=wl.scale,
                                                    out=g.out, lse=g.lse)
                    t_kpad, _ = time_forward(K(), m, torch, flush)
            tb = time.perf_counter()
            m2 = g.create()
            torch.cuda.synchronize()
            build_ms = (time.perf_counter() - tb) * 1e3
            m2.close()
            kname = kernel_name(wl, tiles_total)
            entry = roofline_entry(wl, t, nnz_total, tiles_total, hbm_peak, tc_peak, peak_src, clk_mhz, kname,
                                   traffic=committed_traffic(kname, wl.name), t_warm_ms=t_warm)
            entry.update({"nnz_total": nnz_total,
                          "tflops": round(4.0 * nnz_total * wl.d / (t * 1e-3) / 1e12, 3),
                          "mask_build_wall_ms": round(build_ms, 3),
                          "shape": f"B={wl.B} H={wl.H} n={wl.n} d={wl.d} {wl.dtype}"})
            if t_kpad is not None:
                entry["fwd_ms_seqlen_k"] = round(t_kpad, 4)
            if cfg == 5:
                entry["note"] = "extra to the five workloads: all-ones mask, d = 128"
            res[wl.name] = entry
            del g
        except Exception as ex:  # keep the headline line even if one extra case fails
            res[f"cfg{cfg}"] = {"error": str(ex)[:200]}
    return res


def _smi_id(torch, dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev)


def reference_arm(args, rank, world):
    """The fp64 CPU oracle, as it stands, on the host cores: each step a bounded
    random sample of the workload's rows."""
    if rank != 0:
        return None
    wl = workloads.make(args.config)
    threads = os.cpu_count() or 1
    per_step = max(1.0, min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_oracle_rate(wl, per_step / 4, threads)
    rates, rows, times = [], 0, []
    for _ in range(args.steps):
        r, cnt, nz, t = cpu_oracle_rate(wl, per_step, threads)
        rates.append(r)
        rows += cnt
        times.append(t)
    value = statistics.mean(rates)
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * statistics.mean(times), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded numpy PCG64)",
        "config": {"workload": f"{wl.name} B={wl.B} H={wl.H} n={wl.n} d={wl.d}"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows} random query rows over {args.steps} steps (fp64 oracle, "
                                   f"{cpu_model()})"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = reference_arm(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return

    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    import sparse_mask_scaled_b200 as sp
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    result, wl = bench_ours(args, rank, world, torch, sp)
    if rank == 0:
        if not args.no_extra and world == 1:
            result["other_workloads_fwd"] = other_workloads(torch, sp, args.config,
                                                            result["clocks"].get("sm_mhz"))
            try:
                result["backward"] = backward_timing(args, torch, sp)
            except Exception as ex:  # keep the headline line
                result["backward"] = {"error": str(ex)[:200]}
            try:
                result["fusion_ablation"] = fusion_ablation(args, torch, sp)
            except Exception as ex:
                result["fusion_ablation"] = {"error": str(ex)[:200]}
            try:
                result["contiguous_runs"] = contiguous_runs(torch, sp)
            except Exception as ex:
                result["contiguous_runs"] = {"error": str(ex)[:200]}
        if not args.no_cpu_baseline and world == 1:
            threads = os.cpu_count() or 1
            rate, cnt, nz, t = cpu_oracle_rate(wl, args.cpu_seconds, threads)
            rate1, cnt1, nz1, t1 = cpu_oracle_rate(wl, max(1.0, args.cpu_seconds / 4), 1)
            result["cpu_baseline"] = {"value": round(rate, 6), "unit": "TFLOP/s", "cores": threads,
                                      "kind": "oracle",
                                      "sample": f"{cnt} random query rows ({nz} nonzeros) of the same "
                                                f"workload, {t:.1f} s wall, fp64, {cpu_model()}",
                                      "one_thread": {"value": round(rate1, 6), "cores": 1,
                                                     "sample": f"{cnt1} random query rows ({nz1} nonzeros), "
                                                               f"{t1:.1f} s wall"}}
        print(json.dumps(result), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
