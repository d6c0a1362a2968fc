#!/usr/bin/env python3
"""Benchmark of the NVFP4 hot path on B200.

One step = the prefill linear-layer path on the 8192 x 8192 x 8192 workload
(activations bf16 [8192, 8192] N(0,1) with 0.5% outlier channels x30,
weights N(0, 0.02)): quantize the activations and run the block-scaled GEMM
against the pre-quantized weights, bf16 output: the amax pass, then one
kernel whose extra warps quantize A (scales in the tensor-core layout) row
block by row block while its tensor cores multiply the blocks already done.  value = 2*M*N*K per step
over the device time of the step, summed over ranks (weak scaling: every
rank runs its own replica; the path needs no exchange).

Also reported on rank 0: that kernel's roofline (live CUDA events),
end-to-end throughput through host buffers and SM clocks during the timed
region; at N = 1 also the quantize-bandwidth, rotated and stochastic
quantize, decode-GEMV, long-K, MXFP4 and requantizing-GEMM workloads, and
the CPU oracle timed on a bounded sample of the same workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nvfp4_block_scaled_15_b200 import inputs  # noqa: E402

METRIC = "NVFP4 GEMM TFLOPS & fraction of FP4 peak; quantize/GEMV GB/s vs HBM"
M = N = K = 8192
FLOPS_STEP = 2.0 * M * N * K
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0            # nominal dense ratio (9 PFLOP/s FP4 : 2.25 PFLOP/s BF16)
NOMINAL_FP4_TFLOPS = 9000.0    # B200 dense FP4, nominal (the 18 PFLOP/s figure is with 2:4 sparsity)
GEMM_SOURCES = ["gemm.cu", "ptx.cuh", "tc_common.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-parts", action="store_true", help="skip the quantize/GEMV/long-K sub-benchmarks")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--part", choices=["quantize", "hadamard", "stochastic", "gemv", "longk", "gemm", "quantgemm",
                                       "mxquantize", "mxgemm", "requant"],
                    default=None,
                    help="run one workload alone, --steps times (for profiling); prints its timing")
    ap.add_argument("--record-traffic", nargs=4, metavar=("NAME", "RAW_CSV", "LAUNCHES", "SOURCES"),
                    help="store DRAM bytes per launch of an ncu capture in profiles/traffic.json: NAME, the "
                         "CSV of 'ncu -i REPORT --page raw --csv', the number of captured launches, and the "
                         "kernel's csrc files, comma-separated; the capture command follows as --traffic-command")
    ap.add_argument("--traffic-command", default="", help="the ncu command of --record-traffic's capture")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _code_only(text: str) -> str:
    """C/C++/CUDA source without comments and with whitespace runs collapsed:
    edits to comments or layout do not change it."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_code_hash(files):
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "nvfp4_block_scaled_15_b200", "csrc", name), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")


def profile_entry(name):
    """One ncu capture's figures for a kernel, kept in profiles/traffic.json by
    ``--record-traffic``; None when the kernel's code (comments and layout
    aside) changed after the capture."""
    if not os.path.exists(TRAFFIC_JSON):
        return None
    with open(TRAFFIC_JSON) as f:
        entry = json.load(f).get(name)
    if not entry or entry.get("code_hash") != kernel_code_hash(entry["sources"]):
        return None
    return entry


def profile_traffic(name):
    """DRAM bytes per launch of a kernel from its ncu capture (or None)."""
    entry = profile_entry(name)
    return None if entry is None else int(entry["dram_bytes_per_launch"])


def record_traffic(name, raw_csv, sources, launches, command):
    """Store one capture's DRAM traffic per launch (dram__bytes_read.sum +
    dram__bytes_write.sum, averaged over the captured launches) from the CSV
    that ``ncu -i REPORT --page raw --csv`` prints, with the code hash of the
    kernel's sources at capture time."""
    import csv
    with open(raw_csv, newline="") as f:
        rows = list(csv.reader(f))
    head = next(r for r in rows if "dram__bytes_read.sum" in r)
    i_r, i_w = head.index("dram__bytes_read.sum"), head.index("dram__bytes_write.sum")
    units_row = rows[rows.index(head) + 1]
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    vals = []
    pct = {"tensor_pipe_busy_pct": "sm__pipe_tensor_cycles_active.avg.pct_of_peak_sustained_elapsed",
           "dram_throughput_pct": "gpu__dram_throughput.avg.pct_of_peak_sustained_elapsed"}
    pct_vals = {k: [] for k in pct}
    for r in rows[rows.index(head) + 2:]:
        if len(r) > max(i_r, i_w) and r[i_r]:
            vals.append(float(r[i_r].replace(",", "")) * scale[units_row[i_r]]
                        + float(r[i_w].replace(",", "")) * scale[units_row[i_w]])
            for k, metric in pct.items():
                if metric in head and r[head.index(metric)]:
                    pct_vals[k].append(float(r[head.index(metric)].replace(",", "")))
    if len(vals) != launches:
        raise SystemExit(f"{len(vals)} launches in {raw_csv}, expected {launches}")
    data = {}
    if os.path.exists(TRAFFIC_JSON):
        with open(TRAFFIC_JSON) as f:
            data = json.load(f)
    data[name] = {"dram_bytes_per_launch": int(round(sum(vals) / len(vals))), "sources": sources,
                  "code_hash": kernel_code_hash(sources), "launches": launches, "command": command}
    for k, v in pct_vals.items():
        if len(v) == launches:
            data[name][k] = round(sum(v) / len(v), 2)
    with open(TRAFFIC_JSON, "w") as f:
        json.dump(data, f, indent=1, sort_keys=True)
        f.write("\n")
    return data[name]


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x10: "sync_boost",
            0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples = []          # (t, sm_mhz, reasons_bitmask)
        self.period = period_s
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _reasons(self):
        nv = self._nv
        for fn in ("nvmlDeviceGetCurrentClocksEventReasons", "nvmlDeviceGetCurrentClocksThrottleReasons"):
            if hasattr(nv, fn):
                return getattr(nv, fn)(self._h)
        return 0

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM)
                self.samples.append((time.perf_counter(), mhz, int(self._reasons())))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self._nv is not None:
            self._t.start()
        return self

    def stop(self):
        self._stop.set()
        if self._nv is not None:
            self._t.join(timeout=2)

    def summary(self, t0, t1):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        timed = [s for s in self.samples if t0 <= s[0] <= t1]
        use = timed if len(timed) >= 3 else self.samples
        bits = 0
        for s in use:
            bits |= s[2]
        return {"sm_mhz": statistics.median(s[1] for s in use), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(v for k, v in _REASONS.items() if bits & k),
                "samples": len(use), "window": "timed" if use is timed else "warmup+timed"}


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample
# ---------------------------------------------------------------------------
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


class OracleSample:
    """The prefill step restated by the oracle on a slice: tensor amax of the
    full activations, quantization of ``rows`` activation rows, and the fp64
    block-scaled GEMM of those rows against ``cols`` pre-quantized weight rows."""

    def __init__(self, a_bits, w_bits, rows, cols):
        from oracle import nvfp4_oracle as O
        self.O = O
        self.a = a_bits
        self.rows, self.cols = rows, cols
        gw = O.global_scale(O.amax(w_bits))
        cw, sw = O.quantize_with_scale(w_bits[:cols], gw)
        self.w = (O.pack_codes(cw), sw, gw)

    def step(self):
        O = self.O
        ga = O.global_scale(O.amax(self.a))
        ca, sa = O.quantize_with_scale(self.a[:self.rows], ga)
        d, s, alpha = O.gemm_ref(O.pack_codes(ca), sa, ga, *self.w)
        return d

    def flops(self):
        return 2.0 * self.rows * self.cols * K


def time_oracle(sample: OracleSample, reps: int = 1):
    t = time.perf_counter()
    for _ in range(reps):
        sample.step()
    return (time.perf_counter() - t) / reps


# ---------------------------------------------------------------------------
# multi-rank timing (one process per GPU; replicas, no data-path collective)
# ---------------------------------------------------------------------------
def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's step time: every rank contributes its own mean."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, ms: float) -> float:
    """Whole-job TFLOP/s: every rank runs one prefill step per step time."""
    return world * FLOPS_STEP / (ms * 1e-3) / 1e12


# ---------------------------------------------------------------------------
# reference arm: the oracle, timed on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, rank):
    if rank != 0:
        return
    a, w = inputs.prefill_gemm()
    sample = OracleSample(a, w, rows=256, cols=512)
    for _ in range(args.warmup):
        sample.step()
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        sample.step()
        times.append(time.perf_counter() - t)
    sec = statistics.mean(times)
    value = sample.flops() / sec / 1e12
    desc = (f"oracle prefill step on a slice: amax of A [8192,8192], quantize {sample.rows} rows of A, "
            f"fp64 GEMM against {sample.cols} pre-quantized weight rows (K=8192)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_block(n_gpus):
    return {"workload": "prefill GEMM 8192x8192x8192: activation quantize (amax pass, then quantization "
                        "inside the GEMM kernel, tcgen05 scale layout) + block-scaled NVFP4 GEMM, weights "
                        "pre-quantized, bf16 out",
            "M": M, "N": N, "K": K, "activations": "bf16 N(0,1), 0.5% outlier channels x30, seed 4",
            "weights": "bf16 N(0,0.02), seed 5", "l2": "flushed before every step (256 MiB write)",
            "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "single GPU"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if args.record_traffic:
        name, raw_csv, launches, sources = args.record_traffic
        print(json.dumps(record_traffic(name, raw_csv, sources.split(","), int(launches), args.traffic_command)))
        return
    if args.part:
        run_part(args)
        return

    # host inputs first (the generator's process pool starts before CUDA)
    a_bits, w_bits = inputs.prefill_gemm()
    parts_inputs = None
    # the single-GPU workloads run at N = 1 only: with N > 1 the other ranks
    # would sit in the closing barrier for their whole duration
    if rank == 0 and world == 1 and not args.no_parts:
        parts_inputs = {"quant": inputs.quantize_bandwidth(),
                        "gemv": inputs.decode_gemv(16),
                        "longk": inputs.long_k()}

    import torch
    import torch.distributed as dist
    from nvfp4_block_scaled_15_b200 import nvfp4 as nv

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    peaks, peaks_src = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    hbm_peak = peaks["hbm_gbs"]

    a = to_dev(a_bits)
    w = to_dev(w_bits)
    qw = nv.quantize(w, nv.SF_TCGEN05)
    qa = nv.empty_quantized(M, K, nv.SF_TCGEN05, dev)
    d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws_bytes = nv.nvfp4_workspace_bytes(nv.OP_GEMM_QUANT_A, M, N, K)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    # The step: A's amax pass (prepare), then the quantize-and-GEMM kernel
    # (run), issued back to back as nvfp4_gemm_quant_a issues them (the
    # kernel's programmatic launch overlaps the amax pass's tail).
    def prepare():
        nv.nvfp4_gemm_quant_a_prepare(a, K, M, N, K, ws, ws_bytes)

    def run():
        nv.nvfp4_gemm_quant_a_run(a, K, qw.codes, qw.sf, qw.g, M, N, K, d, N, nv.OUT_BF16, ws, ws_bytes)

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        prepare()
        run()
    torch.cuda.synchronize(dev)
    assert nv.nvfp4_check_device_status() == nv.OK

    def timed_steps(split):
        """K steps between a barrier and a synchronize on both sides, the L2
        flushed before each; with ``split`` an event between the amax pass and
        the kernel times the kernel on its own (the event ends the programmatic
        overlap, so the step itself is timed without it)."""
        ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for e0, e1, e2 in ev:
            flush.zero_()
            e0.record(stream)
            prepare()
            if split:
                e1.record(stream)
            run()
            e2.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        return ev, t0, time.perf_counter()

    sampler = ClockSampler(local, period_s=0.005).start()
    ev, t0, t1 = timed_steps(split=False)
    step_ms = [e0.elapsed_time(e2) for e0, e1, e2 in ev]
    ms = statistics.mean(step_ms)
    if world > 1:
        ms = max_over_ranks(ms, dist, dev)
    value = job_value(world, ms)
    # second timed pass: the kernel alone, for its roofline.  An idle half
    # second first, so that it starts from the power state the first pass
    # started from (after a pass of back-to-back steps the 1 kW limit has
    # already pulled the SM clock down).
    time.sleep(0.5)
    ev_split, t0s, t1s = timed_steps(split=True)
    sampler.stop()
    status = nv.nvfp4_check_device_status()
    amax_ms = [e0.elapsed_time(e1) for e0, e1, e2 in ev_split]
    fused_ms = [e1.elapsed_time(e2) for e0, e1, e2 in ev_split]

    # end to end through the public API with pinned host buffers
    e2e = None
    if rank == 0:
        e2e = bench_e2e(nv, torch, dev, a_bits, qw, min(args.steps, 30))

    result = None
    if rank == 0:
        fused_avg = statistics.mean(fused_ms)
        achieved = FLOPS_STEP / (fused_avg * 1e-3) / 1e12
        prof = profile_entry("quant_gemm_prefill_8192")
        traffic = None if prof is None else int(prof["dram_bytes_per_launch"])
        result = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic", "config": config_block(world),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                         "frac": achieved / fp4_peak, "traffic": traffic,
                         "frac_of_nominal_dense_fp4": achieved / NOMINAL_FP4_TFLOPS,
                         "tensor_pipe_busy_pct_ncu": None if prof is None else prof.get("tensor_pipe_busy_pct"),
                         "kernel": "gemm_pair_kernel<quantize A> (extra warps quantize the bf16 A row block by "
                                   "row block; tcgen05.mma.cta_group::2 kind::mxf4nvf4, 256x256 tiles, 8192^3)",
                         "peak_source": f"{peaks_src} bf16 burst {peaks['bf16_tflops']} TFLOP/s x {FP4_OVER_BF16} "
                                        "(nominal FP4:BF16 dense ratio)",
                         "algorithmic": "2*M*N*K = 1.0995e12 FLOP per launch (the quantization of A inside the "
                                        "kernel is not counted)",
                         "timing": "CUDA events around the kernel in a second timed pass of the same steps, an "
                                   "event between the amax pass and the kernel, after 0.5 s idle",
                         "clocks": sampler.summary(t0s, t1s)},
            "e2e": e2e,
            "gpu_launches": 2 * args.steps,
            "clocks": sampler.summary(t0, t1),
            "wall_ms_per_step": (t1 - t0) * 1e3 / args.steps,
            "step_breakdown_ms": {"amax_pass": statistics.mean(amax_ms), "quantize_and_gemm": fused_avg,
                                  "step_with_event_between": statistics.mean(e0.elapsed_time(e2)
                                                                             for e0, e1, e2 in ev_split)},
            "device_status": nv.nvfp4_status_string(status),
        }
    if rank == 0 and parts_inputs is not None:
        parts_inputs["prefill"] = (a, w)
        result["parts"] = bench_parts(nv, torch, dev, flush, parts_inputs, hbm_peak, fp4_peak, peaks_src)
        # the same step as two kernels after the amax pass (quantize pass, then
        # the plain GEMM), and the plain GEMM alone
        ms_q = _timed(torch, dev, flush, lambda: nv.quantize(a, nv.SF_TCGEN05, out=qa), 20)
        ms_g = _timed(torch, dev, flush, lambda: nv.gemm(qa, qw, out=d), 20)
        ms_two = _timed(torch, dev, flush, lambda: (nv.quantize(a, nv.SF_TCGEN05, out=qa), nv.gemm(qa, qw, out=d)), 20)
        result["parts"]["prefill_step_two_kernels"] = {
            "ms": ms_two, "tflops": FLOPS_STEP / (ms_two * 1e-3) / 1e12, "quantize_ms": ms_q, "gemm_ms": ms_g,
            "note": "amax + quantize passes, then gemm_pair_kernel; median of 20, L2 flushed"}
        result["parts"]["gemm_only"] = {
            "ms": ms_g, "tflops": FLOPS_STEP / (ms_g * 1e-3) / 1e12,
            "frac_fp4_peak": FLOPS_STEP / (ms_g * 1e-3) / 1e12 / fp4_peak,
            "traffic": profile_traffic("gemm_prefill_8192"),
            "tensor_pipe_busy_pct_ncu": (profile_entry("gemm_prefill_8192") or {}).get("tensor_pipe_busy_pct")}
    if rank == 0 and world == 1 and not args.no_cpu:
        sample = OracleSample(a_bits, w_bits, rows=8192, cols=2048)
        sec = time_oracle(sample)
        result["cpu_baseline"] = {
            "value": sample.flops() / sec / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"oracle prefill step on a slice: amax of A [8192,8192], quantize {sample.rows} rows, "
                      f"fp64 GEMM against {sample.cols} pre-quantized weight rows, K=8192 "
                      f"({sec:.1f} s on the host)"}
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def bench_e2e(nv, torch, dev, a_bits, qw, steps):
    """The step through host buffers: every step copies A [8192, 8192] bf16 from
    pinned host memory, quantizes and multiplies it (nvfp4_gemm_quant_a) and
    copies D back to pinned host memory.  Steps are double-buffered on three streams (upload, compute,
    download), as a serving loop overlaps them: step i+1's upload and step
    i-1's download run while step i computes, each buffer reused only after
    the work that read it has finished."""
    a_host = torch.from_numpy(np.ascontiguousarray(a_bits).view(np.int16)).view(torch.bfloat16).pin_memory()
    d_host = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    a_dev = [torch.empty((M, K), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    d_dev = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    ws_bytes = nv.nvfp4_workspace_bytes(nv.OP_GEMM_QUANT_A, M, N, K)
    wss = [torch.empty(ws_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    up, comp, down = (torch.cuda.Stream(dev) for _ in range(3))
    uploaded = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    downloaded = [torch.cuda.Event() for _ in range(2)]

    def run(n):
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(computed[b])          # a_dev[b] no longer read
                a_dev[b].copy_(a_host, non_blocking=True)
                uploaded[b].record(up)
            with torch.cuda.stream(comp):
                comp.wait_event(uploaded[b])
                if i >= 2:
                    comp.wait_event(downloaded[b])      # d_dev[b] copied out
                nv.gemm_quant_a(a_dev[b], qw, out=d_dev[b], workspace=wss[b], stream=comp)
                computed[b].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(computed[b])
                d_host[b].copy_(d_dev[b], non_blocking=True)
                downloaded[b].record(down)

    run(4)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(up)
    run(steps)
    down.wait_stream(up)
    down.wait_stream(comp)
    e1.record(down)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    return {"value": FLOPS_STEP / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms, "steps": steps,
            "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
            "pipelining": "double-buffered: upload, compute and download of consecutive steps overlap"}


def _timed(torch, dev, flush, fn, reps):
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        flush.zero_()
        fn()
    ts = []
    for _ in range(reps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        ts.append((e0, e1))
    torch.cuda.synchronize(dev)
    return statistics.median(e0.elapsed_time(e1) for e0, e1 in ts)


def bench_parts(nv, torch, dev, flush, pin, hbm_peak, fp4_peak, peaks_src):
    out = {"peaks": f"{peaks_src}: HBM {hbm_peak} GB/s, FP4 {fp4_peak:.1f} TFLOP/s (bf16 x4)"}
    reps = 20

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    # quantize bandwidth [16384, 8192]
    x = to_dev(pin["quant"])
    rows, k = x.shape
    q = nv.empty_quantized(rows, k, nv.SF_TCGEN05, dev)
    ms_all = _timed(torch, dev, flush, lambda: nv.quantize(x, nv.SF_TCGEN05, out=q), reps)
    ms_amax = _timed(torch, dev, flush, lambda: nv.nvfp4_amax(x, rows, k, k, q.amax), reps)
    ms_q1 = _timed(torch, dev, flush, lambda: nv.nvfp4_quantize(x, rows, k, k, q.codes, q.sf, nv.SF_TCGEN05, q.g,
                                                                q.amax, 1), reps)
    two_pass = rows * k * 2 * 2 + rows * k // 2 + rows * k // 16
    one_pass = rows * k * 2 + rows * k // 2 + rows * k // 16
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(10):
        nv.quantize(x, nv.SF_TCGEN05, out=q)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_b2b = e0.elapsed_time(e1) / 10
    out["quantize_16384x8192"] = {
        "back_to_back_ms": ms_b2b, "back_to_back_gbs_two_pass": two_pass / ms_b2b / 1e6,
        "back_to_back_frac_hbm": two_pass / ms_b2b / 1e6 / hbm_peak,
        "ms": ms_all, "gbs_two_pass": two_pass / ms_all / 1e6, "frac_hbm": two_pass / ms_all / 1e6 / hbm_peak,
        "gbs_strict_one_read": one_pass / ms_all / 1e6,
        "amax_ms": ms_amax, "amax_gbs": rows * k * 2 / ms_amax / 1e6,
        "quantize_pass_ms": ms_q1, "quantize_pass_gbs": one_pass / ms_q1 / 1e6,
        "quantize_pass_frac_hbm": one_pass / ms_q1 / 1e6 / hbm_peak}
    del x, q

    # Hadamard-rotated quantize of the same input (orders 16 and 128): two
    # passes, the transform computed in both; same algorithmic bytes
    x = to_dev(pin["quant"])
    q = nv.empty_quantized(rows, k, nv.SF_TCGEN05, dev)
    had = {}
    for order in (16, 128):
        ms_h = _timed(torch, dev, flush, lambda: nv.quantize_hadamard(x, order, nv.SF_TCGEN05, out=q), reps)
        ms_h1 = _timed(torch, dev, flush, lambda: nv.nvfp4_quantize_hadamard(
            x, rows, k, k, order, q.codes, q.sf, nv.SF_TCGEN05, q.g, q.amax, 1), reps)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(10):
            nv.quantize_hadamard(x, order, nv.SF_TCGEN05, out=q)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_hb = e0.elapsed_time(e1) / 10
        had[f"order={order}"] = {
            "ms": ms_h, "gbs_two_pass": two_pass / ms_h / 1e6, "frac_hbm": two_pass / ms_h / 1e6 / hbm_peak,
            "back_to_back_ms": ms_hb, "back_to_back_frac_hbm": two_pass / ms_hb / 1e6 / hbm_peak,
            "quantize_pass_ms": ms_h1, "quantize_pass_frac_hbm": one_pass / ms_h1 / 1e6 / hbm_peak}
    ms_hs = _timed(torch, dev, flush, lambda: nv.quantize_hadamard_stochastic(x, 16, 1234, 0, nv.SF_TCGEN05, out=q),
                   reps)
    had["order=16_stochastic"] = {"ms": ms_hs, "gbs_two_pass": two_pass / ms_hs / 1e6,
                                  "frac_hbm": two_pass / ms_hs / 1e6 / hbm_peak}
    ms_hs = _timed(torch, dev, flush, lambda: nv.quantize_hadamard_stochastic(x, 128, 1234, 0, nv.SF_TCGEN05, out=q),
                   reps)
    had["order=128_stochastic"] = {"ms": ms_hs, "gbs_two_pass": two_pass / ms_hs / 1e6,
                                   "frac_hbm": two_pass / ms_hs / 1e6 / hbm_peak}
    out["hadamard_quantize_16384x8192"] = had
    del x, q
    # stochastic rounding of the codes (Philox4x32-10 in the kernel), same input and bytes
    x = to_dev(pin["quant"])
    q = nv.empty_quantized(rows, k, nv.SF_TCGEN05, dev)
    ms_s = _timed(torch, dev, flush, lambda: nv.quantize_stochastic(x, 1234, 0, nv.SF_TCGEN05, out=q), reps)
    ms_s1 = _timed(torch, dev, flush, lambda: nv.nvfp4_quantize_stochastic(
        x, rows, k, k, q.codes, q.sf, nv.SF_TCGEN05, q.g, q.amax, 1, 1234, 0), reps)
    out["stochastic_quantize_16384x8192"] = {
        "ms": ms_s, "gbs_two_pass": two_pass / ms_s / 1e6, "frac_hbm": two_pass / ms_s / 1e6 / hbm_peak,
        "quantize_pass_ms": ms_s1, "quantize_pass_frac_hbm": one_pass / ms_s1 / 1e6 / hbm_peak}
    del x, q

    # decode GEMV: W [28672, 8192] pre-quantized, x [M, 8192] quantized in the
    # call.  Three weight copies (396 MB, more than L2) in rotation, so no call
    # finds its weights in L2 without a flush.
    xg, wg = pin["gemv"]
    n, k = wg.shape
    wqs = [nv.quantize(to_dev(wg), nv.SF_TCGEN05) for _ in range(3)]
    stream = torch.cuda.current_stream(dev)
    res, thr = {}, {}
    for m in (1, 8, 16):
        xm = to_dev(xg[:m])
        y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(nv.nvfp4_workspace_bytes(nv.OP_GEMV_BATCHED, m, n, k), dtype=torch.uint8, device=dev)
        algo = n * k // 2 + n * k // 16 + m * k * 2 + m * n * 2
        for i in range(6):
            nv.gemv_batched(xm, wqs[i % 3], out=y, workspace=ws)
        # per call: one call per event pair, the weights cold by rotation
        ts = []
        for i in range(21):
            c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            c0.record(stream)
            nv.gemv_batched(xm, wqs[i % 3], out=y, workspace=ws)
            c1.record(stream)
            ts.append((c0, c1))
        torch.cuda.synchronize(dev)
        ms_c = statistics.median(c0.elapsed_time(c1) for c0, c1 in ts)
        # decode throughput: calls back to back (as layers follow one another)
        calls = 30
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(calls):
            nv.gemv_batched(xm, wqs[i % 3], out=y, workspace=ws)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / calls
        # the same 30 calls captured once in a CUDA graph and replayed (how a
        # decode step issues its layers), so no per-launch host work sits between them
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(calls):
                nv.gemv_batched(xm, wqs[i % 3], out=y, workspace=ws)
        graph.replay()
        torch.cuda.synchronize(dev)
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        graph.replay()
        graph.replay()
        g1.record(stream)
        torch.cuda.synchronize(dev)
        ms_g = g0.elapsed_time(g1) / (2 * calls)
        del graph
        thr[f"M={m}"] = {"ms_per_call": ms, "gbs": algo / ms / 1e6, "frac_hbm": algo / ms / 1e6 / hbm_peak,
                         "graph_ms_per_call": ms_g, "graph_frac_hbm": algo / ms_g / 1e6 / hbm_peak}
        # per call with a 256 MiB L2 flush (a write) before each, last: the
        # flush's dirty lines are written back while the call streams the
        # weights (and would be during the next measurement)
        ms_f = _timed(torch, dev, flush, lambda: nv.gemv_batched(xm, wqs[0], out=y, workspace=ws), reps)
        res[f"M={m}"] = {"ms": ms_c, "gbs": algo / ms_c / 1e6, "frac_hbm": algo / ms_c / 1e6 / hbm_peak,
                         "l2": "inputs larger than L2: three weight copies (396 MB) in rotation, no flush",
                         "ms_l2_flushed": ms_f, "frac_hbm_l2_flushed": algo / ms_f / 1e6 / hbm_peak,
                         "algorithmic_bytes": algo}
        for i in range(6):                      # write the flush's dirty lines back before the next M
            nv.gemv_batched(xm, wqs[i % 3], out=y, workspace=ws)
    out["gemv_28672x8192"] = res
    # the fixed cost an event pair sees around any one launch on this machine: a
    # one-element torch fill timed the same way as the per-call numbers
    tiny = torch.empty(1, dtype=torch.int32, device=dev)
    ts = []
    for i in range(21):
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        tiny.fill_(i)
        c1.record(stream)
        ts.append((c0, c1))
    torch.cuda.synchronize(dev)
    thr["per_call_floor_ms"] = statistics.median(c0.elapsed_time(c1) for c0, c1 in ts)
    thr["note"] = ("ms_per_call: 30 calls between one event pair; graph: the same calls replayed from a CUDA "
                   "graph; both with three weight copies in rotation (396 MB, more than L2); "
                   "per_call_floor_ms: an event pair around a one-element fill")
    out["gemv_28672x8192_back_to_back"] = thr
    del wqs

    # long-K: A [4096, 28672] bf16 quantized in the call, W [8192, 28672] pre-quantized
    al, wl = pin["longk"]
    am, k = al.shape
    nn = wl.shape[0]
    wq = nv.quantize(to_dev(wl), nv.SF_TCGEN05)
    ad = to_dev(al)
    dd = torch.empty((am, nn), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(nv.nvfp4_workspace_bytes(nv.OP_GEMM_QUANT_A, am, nn, k), dtype=torch.uint8, device=dev)
    ms = _timed(torch, dev, flush, lambda: nv.gemm_quant_a(ad, wq, out=dd, workspace=ws), 10)
    fl = 2.0 * am * nn * k
    # the same work as two kernels after the amax pass: the quantize pass, then the plain GEMM
    qa_l = nv.empty_quantized(am, k, nv.SF_TCGEN05, dev)
    ms_two = _timed(torch, dev, flush, lambda: (nv.quantize(ad, nv.SF_TCGEN05, out=qa_l), nv.gemm(qa_l, wq, out=dd)),
                    10)
    out["long_k_4096x8192x28672"] = {"ms": ms, "tflops": fl / ms / 1e9, "frac_fp4_peak": fl / ms / 1e9 / fp4_peak,
                                     "kernel": "amax pass + quantize-and-GEMM kernel (grouped schedule)",
                                     "two_kernels_ms": ms_two, "two_kernels_tflops": fl / ms_two / 1e9}
    del wq, ad, dd, ws, qa_l

    # MXFP4 (E8M0 scale per 32, no global scale): one-pass quantize of the
    # same [16384, 8192] input and the 8192^3 GEMM on MXFP4 operands
    x = to_dev(pin["quant"])
    rows, k = x.shape
    qm = nv.mxfp4_quantize(x, nv.SF_TCGEN05)
    ms = _timed(torch, dev, flush, lambda: nv.mxfp4_quantize(x, nv.SF_TCGEN05, out=qm), reps)
    one_pass = rows * k * 2 + rows * k // 2 + rows * k // 32
    out["mxfp4_quantize_16384x8192"] = {"ms": ms, "gbs": one_pass / ms / 1e6,
                                        "frac_hbm": one_pass / ms / 1e6 / hbm_peak, "algorithmic_bytes": one_pass}
    del x, qm
    a, w = pin["prefill"]
    qa, qw = nv.mxfp4_quantize(a, nv.SF_TCGEN05), nv.mxfp4_quantize(w, nv.SF_TCGEN05)
    d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ms = _timed(torch, dev, flush, lambda: nv.mxfp4_gemm(qa, qw, out=d), reps)
    out["mxfp4_gemm_8192"] = {"ms": ms, "tflops": FLOPS_STEP / ms / 1e9,
                              "frac_fp4_peak": FLOPS_STEP / ms / 1e9 / fp4_peak}
    del qa, qw, d

    # 8192^3 GEMM whose epilogue writes the output quantized for the next
    # layer (NVFP4, tensor-core scales, amax) or as FP8, under an output scale
    # g_d; against the unfused chain GEMM (bf16 D) + quantize of D
    qa, qw = nv.quantize(a, nv.SF_TCGEN05), nv.quantize(w, nv.SF_TCGEN05)
    h = nv.empty_quantized(M, N, nv.SF_TCGEN05, dev)
    h.g.fill_(2688.0 / 40.0)
    ms_rq = _timed(torch, dev, flush, lambda: nv.nvfp4_gemm_requant(
        qa.codes, qa.sf, qa.g, qw.codes, qw.sf, qw.g, M, N, K, h.g, h.codes, N // 2, h.sf, nv.SF_TCGEN05, h.amax),
        reps)
    d8 = torch.empty((M, N), dtype=torch.float8_e4m3fn, device=dev)
    ms_f8 = _timed(torch, dev, flush, lambda: nv.nvfp4_gemm_fp8_out(
        qa.codes, qa.sf, qa.g, qw.codes, qw.sf, qw.g, M, N, K, h.g, d8, N, h.amax), reps)
    d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    hq = nv.empty_quantized(M, N, nv.SF_TCGEN05, dev)
    ms_unfused = _timed(torch, dev, flush, lambda: (nv.gemm(qa, qw, out=d), nv.quantize(d, nv.SF_TCGEN05, out=hq)),
                        reps)
    out["gemm_requant_8192"] = {
        "nvfp4_out_ms": ms_rq, "nvfp4_out_tflops": FLOPS_STEP / ms_rq / 1e9,
        "nvfp4_out_frac_fp4_peak": FLOPS_STEP / ms_rq / 1e9 / fp4_peak,
        "fp8_out_ms": ms_f8, "fp8_out_tflops": FLOPS_STEP / ms_f8 / 1e9,
        "unfused_gemm_bf16_then_quantize_ms": ms_unfused}
    assert nv.nvfp4_check_device_status() == nv.OK
    return out


def run_part(args):
    """One workload alone: generate its inputs, run it ``--steps`` times with the
    L2 flushed in between, print the median time."""
    if args.part in ("quantize", "mxquantize", "hadamard", "stochastic"):
        x_bits = inputs.quantize_bandwidth()
    elif args.part == "gemv":
        xg, wg = inputs.decode_gemv(16)
    elif args.part == "longk":
        al, wl = inputs.long_k()
    else:
        a_bits, w_bits = inputs.prefill_gemm()
    import torch
    from nvfp4_block_scaled_15_b200 import nvfp4 as nv
    dev = torch.device("cuda", 0)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    out = {"part": args.part}
    if args.part == "quantize":
        x = to_dev(x_bits)
        q = nv.empty_quantized(*x.shape, nv.SF_TCGEN05, dev)
        out["ms"] = _timed(torch, dev, flush, lambda: nv.quantize(x, nv.SF_TCGEN05, out=q), args.steps)
    elif args.part == "hadamard":
        x = to_dev(x_bits)
        q = nv.empty_quantized(*x.shape, nv.SF_TCGEN05, dev)
        for order in (16, 128):
            out[f"ms_order{order}"] = _timed(torch, dev, flush,
                                             lambda: nv.quantize_hadamard(x, order, nv.SF_TCGEN05, out=q), args.steps)
        out["ms_order128_stochastic"] = _timed(
            torch, dev, flush, lambda: nv.quantize_hadamard_stochastic(x, 128, 1234, 0, nv.SF_TCGEN05, out=q),
            args.steps)
    elif args.part == "stochastic":
        x = to_dev(x_bits)
        q = nv.empty_quantized(*x.shape, nv.SF_TCGEN05, dev)
        out["ms"] = _timed(torch, dev, flush, lambda: nv.quantize_stochastic(x, 1234, 0, nv.SF_TCGEN05, out=q),
                           args.steps)
    elif args.part == "gemv":
        wq = nv.quantize(to_dev(wg), nv.SF_TCGEN05)
        n, k = wg.shape
        for m in (1, 8, 16):
            xm = to_dev(xg[:m])
            y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(nv.nvfp4_workspace_bytes(nv.OP_GEMV_BATCHED, m, n, k), dtype=torch.uint8, device=dev)
            out[f"ms_M{m}"] = _timed(torch, dev, flush, lambda: nv.gemv_batched(xm, wq, out=y, workspace=ws),
                                     args.steps)
    elif args.part == "longk":
        wq = nv.quantize(to_dev(wl), nv.SF_TCGEN05)
        ad = to_dev(al)
        dd = torch.empty((al.shape[0], wl.shape[0]), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(nv.nvfp4_workspace_bytes(nv.OP_GEMM_QUANT_A, al.shape[0], wl.shape[0], al.shape[1]),
                         dtype=torch.uint8, device=dev)
        out["ms"] = _timed(torch, dev, flush, lambda: nv.gemm_quant_a(ad, wq, out=dd, workspace=ws), args.steps)
    elif args.part == "mxquantize":
        x = to_dev(x_bits)
        q = nv.mxfp4_quantize(x, nv.SF_TCGEN05)
        out["ms"] = _timed(torch, dev, flush, lambda: nv.mxfp4_quantize(x, nv.SF_TCGEN05, out=q), args.steps)
    elif args.part == "requant":
        qa = nv.quantize(to_dev(a_bits), nv.SF_TCGEN05)
        qw = nv.quantize(to_dev(w_bits), nv.SF_TCGEN05)
        h = nv.empty_quantized(M, N, nv.SF_TCGEN05, dev)
        h.g.fill_(2688.0 / 40.0)
        out["ms"] = _timed(torch, dev, flush, lambda: nv.nvfp4_gemm_requant(
            qa.codes, qa.sf, qa.g, qw.codes, qw.sf, qw.g, M, N, K, h.g, h.codes, N // 2, h.sf, nv.SF_TCGEN05,
            h.amax), args.steps)
    elif args.part == "quantgemm":
        qw = nv.quantize(to_dev(w_bits), nv.SF_TCGEN05)
        a = to_dev(a_bits)
        d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(nv.nvfp4_workspace_bytes(nv.OP_GEMM_QUANT_A, M, N, K), dtype=torch.uint8, device=dev)
        out["ms"] = _timed(torch, dev, flush, lambda: nv.gemm_quant_a(a, qw, out=d, workspace=ws), args.steps)
    elif args.part == "mxgemm":
        qa = nv.mxfp4_quantize(to_dev(a_bits), nv.SF_TCGEN05)
        qw = nv.mxfp4_quantize(to_dev(w_bits), nv.SF_TCGEN05)
        d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        out["ms"] = _timed(torch, dev, flush, lambda: nv.mxfp4_gemm(qa, qw, out=d), args.steps)
    else:
        qa = nv.quantize(to_dev(a_bits), nv.SF_TCGEN05)
        qw = nv.quantize(to_dev(w_bits), nv.SF_TCGEN05)
        d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        out["ms"] = _timed(torch, dev, flush, lambda: nv.gemm(qa, qw, out=d), args.steps)
    out["device_status"] = nv.nvfp4_status_string(nv.nvfp4_check_device_status())
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
