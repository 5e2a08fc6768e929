#!/usr/bin/env python3
"""Benchmark of the fused attention hot path on B200.

Headline (``value``): useful prefill TFLOP/s of ``attn_fwd`` on the causal multi-head
workload (B=8, H=32, N=4096, d=128, causal): 4*d flops per visible (query, key) pair.
One step is one ``attn_fwd`` call, which performs every prefill row of the hot path in one
kernel (tile classification, TMA loads, QK^T, mask, online softmax, PV, epilogue).
The ``decode`` object reports the split-KV decode workload (B=64, Hq=32, Hkv=8, T=32768,
d=128): KV-cache GB/s and tokens/s of one ``attn_decode_splitkv`` call (split + merge).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); the (batch, head) units are independent, so each
rank runs its own slice of every workload -- whole batch entries, or whole KV-head groups
when the batch does not divide -- with no collective on the data path; the value is all
ranks' work divided by the slowest rank's device time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402
from workloads import accounting  # noqa: E402

METRIC = "prefill useful TFLOPS & decode KV GB/s on 1 B200, as % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Vendor figures per GPU, for the second fraction the lines report: dense bf16 tensor
# throughput and HBM3e bandwidth (8 TB/s; 7.7 TB/s on HGX boards).
SPEC_PEAKS = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}
L2_BYTES = 126 * 2 ** 20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks during timing
class ClockSampler:
    """Samples the SM clock and the throttle reasons of one GPU while the timed region runs:
    NVML every 5 ms (the timed regions are tens of milliseconds), else nvidia-smi."""
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.sm = []
        self.max_mhz = None
        self.reasons = set()
        self._stop = False
        self._thread = None
        self._nvml = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = None
            try:
                import torch
                pr = torch.cuda.get_device_properties(self.gpu)
                h = pynvml.nvmlDeviceGetHandleByPciBusId(
                    f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0")
            except Exception:
                h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self._nvml = (pynvml, h)
        except Exception:
            self._nvml = None
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def _run(self):
        if self._nvml is not None:
            pynvml, h = self._nvml
            while not self._stop:
                try:
                    self.sm.append(float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)))
                    bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    for name, mask in self.REASONS.items():
                        if bits & mask:
                            self.reasons.add(name)
                except Exception:
                    pass
                time.sleep(0.005)
            return
        fields = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={fields}",
                                     "--format=csv,noheader,nounits", "-lms", "100"],
                                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        while not self._stop:
            line = proc.stdout.readline()
            if not line:
                break
            parts = [x.strip() for x in line.split(",")]
            try:
                self.sm.append(float(parts[0]))
                self.max_mhz = float(parts[1])
            except (ValueError, IndexError):
                continue
            for name, val in zip(names, parts[2:6]):
                if val.lower().startswith("active"):
                    self.reasons.add(name)
        proc.terminate()

    def __exit__(self, *exc):
        self._stop = True
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self):
        return {"sm_mhz": statistics.median(self.sm) if self.sm else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.sm)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(n_gpus: int, backend: str | None = None):
    """One process per GPU under torchrun: NCCL when CUDA is present (gloo only for the
    CPU tests of this plumbing). Returns (world, rank, local rank)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend is None:
        backend = "nccl" if torch.cuda.is_available() else "gloo"
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, x: float) -> float:
    """The slowest rank's figure (all ranks take part; every rank gets the result)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """All ranks' units over the slowest rank's time (every rank runs an equal part)."""
    return units_per_rank * world / (ms_max * 1e-3)


def my_part(w: workloads.Workload, world: int) -> workloads.Workload:
    """This rank's part of a workload: its own batch entries or KV-head groups (no exchange
    between ranks), or the whole workload when neither divides evenly."""
    return workloads.rank_part(w, world, int(os.environ.get("RANK", "0")))


def split_note(w_full: workloads.Workload, w: workloads.Workload, world: int) -> str:
    if world == 1:
        return "1 GPU, the whole workload"
    if w.B != w_full.B:
        return f"{world} ranks, each its own {w.B} of the {w_full.B} batch entries, no collective"
    if w.Hkv != w_full.Hkv:
        return (f"{world} ranks, each its own {w.Hkv} of the {w_full.Hkv} KV heads (with their "
                f"query heads), no collective")
    return f"{world} replicas of the whole workload (B and Hkv not divisible), no collective"


# ----------------------------------------------------------------------- CPU baseline
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_prefill_sample(w: workloads.Workload, budget_s: float, max_heads: int = 256):
    """Times the fp64 oracle on whole heads of the workload until ``budget_s`` is spent.
    Returns (useful TFLOP/s, heads done, seconds)."""
    import oracle
    q, k, v = (x.float().numpy() for x in _cpu_head_inputs(w, 0))
    docs = workloads.workload_doc_offsets(w)
    pairs = accounting.visible_pairs(w.Nq, w.Nk, w.mask_kind, w.window, docs)
    G = w.Hq // w.Hkv
    rows = np.arange(w.Nq)
    done, t0 = 0, time.perf_counter()
    while done < max_heads:
        h = done % w.Hq
        for r0 in range(0, w.Nq, 256):
            rr = rows[r0:r0 + 256]
            oracle.attention_head(q[h, rr], rr, k[h // G], v[h // G], w.scale, w.mask_kind,
                                  w.window, w.softcap, docs)
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return 4 * w.d * pairs * done / dt / 1e12, done, dt


def _cpu_head_inputs(w: workloads.Workload, b: int):
    """q[b], k[b], v[b] of the workload, drawn on the CPU (same seeds as make_inputs)."""
    q = workloads.randn_bf16((1, w.Hq, w.Nq, w.d), w.seed, 0, w.input_std)[0]
    k = workloads.randn_bf16((1, w.Hkv, w.Nk, w.d), w.seed, 1, w.input_std)[0]
    v = workloads.randn_bf16((1, w.Hkv, w.Nk, w.d), w.seed, 2, w.input_std)[0]
    return q, k, v


# ----------------------------------------------------------------- traffic from ncu
def recorded_traffic(kernel_key: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current
    kernel source (the summary stores a hash of the sources it measured)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel_key)
    except (OSError, ValueError):
        return None
    if not rec:
        return None
    from io_aware_softmax_b200 import build as _b
    import hashlib
    h = hashlib.sha256()
    for name in rec.get("sources", []):
        with open(os.path.join(_b.CSRC, name), "rb") as f:
            h.update(f.read())
    return rec.get("bytes_per_launch") if h.hexdigest() == rec.get("sha256") else None


# ----------------------------------------------------------------------------- our arm
def time_launches(fn, steps: int, world: int):
    import torch
    stream = torch.cuda.current_stream()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    t_all0 = torch.cuda.Event(enable_timing=True)
    t_all1 = torch.cuda.Event(enable_timing=True)
    t_all0.record(stream)
    for i in range(steps):
        starts[i].record(stream)
        fn()
        ends[i].record(stream)
    t_all1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = t_all0.elapsed_time(t_all1)
    return total_ms, per


def run_ours(args, world, rank, local):
    import torch
    import io_aware_softmax_b200 as attn

    peaks, peak_src = load_peaks()
    if args.only == "decode":
        return bench_decode(args, world, local, peaks, peak_src)
    if args.only == "extras":
        return {"extras": bench_extras(args, world, local, peaks, peak_src)}
    if args.workload:
        # one prefill workload alone (profiler captures of a single kernel)
        return bench_prefill_variant(workloads.BY_NAME[args.workload], args, world, local,
                                     peaks, peak_src, steps=args.steps)
    w_full = workloads.CAUSAL_MHA
    w = my_part(w_full, world)
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = workloads.make_inputs(w, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    flops = accounting.prefill_useful_flops(w.B, w.Hq, w.Nq, w.Nk, w.d, w.mask_kind)
    executed = accounting.prefill_executed_flops(w.B, w.Hq, w.Nq, w.Nk, w.d, w.mask_kind)

    def step():
        attn.attn_fwd(q, k, v, scale=w.scale, mask=w.mask_kind, out=o, lse=lse)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if attn.device_status() != 0:
        raise RuntimeError("device status not ok after warm-up")
    with ClockSampler(local) as clk:
        total_ms, per = time_launches(step, args.steps, world)
    if attn.device_status() != 0:
        raise RuntimeError("device status not ok after timed steps")
    ms_step = max_over_ranks(world, total_ms / args.steps)
    kernel_ms = max_over_ranks(world, sum(per) / len(per))
    value = whole_job_rate(flops, world, ms_step) / 1e12
    clocks = clk.summary()
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "strong" if w is not w_full or world == 1 else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": w_full.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.Nq,
                   "d": w.d, "mask": "causal",
                   "useful_tflop_per_step": round(flops * world / 1e12, 4),
                   "executed_tflop_per_step": round(executed * world / 1e12, 4),
                   "l2": "inputs larger than L2 (q+k+v %.0f MB > 126 MB per GPU)" %
                         (3 * q.numel() * 2 / 1e6),
                   "parallelism": split_note(w_full, w, world),
                   "seed": w.seed},
        "roofline": prefill_roofline(flops, executed, kernel_ms, peaks, peak_src, clocks,
                                     "attn_fwd_sm100_kernel<128>",
                                     recorded_traffic("prefill_causal_mha"),
                                     torch.cuda.get_device_properties(dev).multi_processor_count),
        "gpu_launches": args.steps,
    }
    out["clocks"] = clocks

    if not args.no_e2e:
        out["e2e"] = e2e_prefill(w, args, world, q, k, v)
    del q, k, v, o, lse
    torch.cuda.empty_cache()
    if args.only == "all":
        # the other two prefill workloads: sliding-window GQA and packed documents + soft-cap
        out["configs"] = {x.name: bench_prefill_variant(x, args, world, local, peaks, peak_src)
                          for x in (workloads.SWA_GQA, workloads.DOC_SOFTCAP)}
    if not args.no_decode and args.only == "all":
        out["decode"] = bench_decode(args, world, local, peaks, peak_src)
    if not args.no_extras and args.only == "all":
        out["extras"] = bench_extras(args, world, local, peaks, peak_src)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, heads, dt = oracle_prefill_sample(w, args.cpu_budget)
        out["cpu_baseline"] = {"value": round(tf, 5), "unit": "TFLOP/s",
                               "cores": blas_threads(), "kind": "oracle",
                               "sample": f"{heads} whole heads (4096 query rows each, all keys) "
                                         f"of {w.name}, fp64, {dt:.1f} s"}
        if args.only == "all":
            out["cpu_baseline"]["per_workload"] = cpu_baselines_other(args.cpu_budget / 3)
    out["summary"] = summary_of(out)
    return out


def summary_of(out: dict) -> dict:
    """One short entry per line, [value, unit, ms per step, roofline fraction]: the whole
    line is long, so this compact copy goes last, where a reader of the output's tail sees
    every workload's figure."""
    def entry(x):
        r = x.get("roofline", {})
        return [x.get("value"), x.get("unit"), x.get("ms_per_step"), r.get("frac")]
    sm = {out["config"]["workload"]: entry(out)}
    for group in ("configs", "extras"):
        for name, x in out.get(group, {}).items():
            sm[name] = entry(x)
    if "decode" in out:
        sm[out["decode"]["workload"]] = entry(out["decode"])
    if "e2e" in out:
        sm["e2e"] = [out["e2e"]["value"], out["e2e"]["unit"], out["e2e"].get("ms_per_step"),
                     None]
    return sm


def cpu_baselines_other(budget_s: float) -> dict:
    """The oracle on bounded samples of the other three workloads, extrapolated to the whole
    workload: whole query-row blocks of a few heads (sliding GQA, documents) or whole
    sequences (decode), timed, scaled by the rows (sequences) the workload has."""
    res = {}
    for w in (workloads.SWA_GQA, workloads.DOC_SOFTCAP):
        per_row_s, rows, dt = oracle_rows_sample(w, budget_s)
        docs = workloads.workload_doc_offsets(w)
        flops = accounting.prefill_useful_flops(w.B, w.Hq, w.Nq, w.Nk, w.d, w.mask_kind,
                                                w.window, docs)
        total_s = per_row_s * w.B * w.Hq * w.Nq
        res[w.name] = {"value": round(flops / total_s / 1e12, 6), "unit": "TFLOP/s",
                       "sample": f"{rows} query rows in 256-row blocks over several heads, "
                                 f"{dt:.1f} s; extrapolated to all {w.B * w.Hq * w.Nq} rows"}
    w = workloads.DECODE
    seqs, dt = oracle_decode_sample(w, budget_s)
    kv = accounting.decode_kv_bytes(w.B, w.Hkv, w.Nk, w.d)
    per_seq = dt / seqs
    res[w.name] = {"value": round(kv / (per_seq * w.B) / 1e9, 4), "unit": "GB/s (KV cache)",
                   "sample": f"{seqs} whole sequences (all 32 heads, 32768 cached rows), "
                             f"{dt:.1f} s; extrapolated to all {w.B}"}
    return res


def oracle_rows_sample(w: workloads.Workload, budget_s: float):
    """Seconds per query row of the fp64 oracle on a prefill workload: 256-row blocks taken
    at seeded places over the heads of batch entry 0 until ``budget_s`` is spent."""
    import oracle
    q, k, v = (x.float().numpy() for x in _cpu_head_inputs(w, 0))
    docs = workloads.workload_doc_offsets(w)
    G = w.Hq // w.Hkv
    rng = np.random.default_rng(w.seed)
    rows, t0 = 0, time.perf_counter()
    while True:
        h = int(rng.integers(w.Hq))
        r0 = int(rng.integers(0, w.Nq // 256)) * 256
        rr = np.arange(r0, min(r0 + 256, w.Nq))
        oracle.attention_head(q[h, rr], rr, k[h // G], v[h // G], w.scale, w.mask_kind,
                              w.window, w.softcap, docs)
        rows += len(rr)
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return dt / rows, rows, dt


def oracle_decode_sample(w: workloads.Workload, budget_s: float):
    """Whole decode sequences (every query head against its KV head's full cache) through
    the fp64 oracle until ``budget_s`` is spent; returns (sequences, seconds)."""
    import oracle
    G = w.Hq // w.Hkv
    # sequence 0's inputs (the CPU draw of the same seeds), reused for every timed sequence
    q = workloads.randn_bf16((1, w.Hq, 1, w.d), w.seed, 0)[0].float().numpy()
    k = workloads.randn_bf16((1, w.Hkv, w.Nk, w.d), w.seed, 1)[0].float().numpy()
    v = workloads.randn_bf16((1, w.Hkv, w.Nk, w.d), w.seed, 2)[0].float().numpy()
    seqs, t0 = 0, time.perf_counter()
    while seqs < w.B:
        for h in range(w.Hq):
            oracle.attention_head(q[h], np.arange(1), k[h // G], v[h // G], w.scale)
        seqs += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return seqs, time.perf_counter() - t0


def l2_note(*tensors) -> str:
    """The L2 statement of a line's config: the inputs every step reads exceed the L2, so no
    flush is needed between timed steps."""
    nbytes = sum(t.numel() * t.element_size() for t in tensors)
    assert nbytes > L2_BYTES, "inputs fit in L2: the line would need an L2 flush"
    return "inputs larger than L2 (%.0f MB > %.0f MB)" % (nbytes / 1e6, L2_BYTES / 1e6)


def bench_extras(args, world, local, peaks, peak_src):
    """The rows beyond the headline: ALiBi and symmetric-window prefill, paged decode, the
    backward pass and the FP8 prefill, one line each (--extra picks one group of them)."""
    pick = getattr(args, "extra", None)
    ex = {}
    if pick in (None, "alibi"):
        ex[workloads.ALIBI_MHA.name] = bench_prefill_variant(workloads.ALIBI_MHA, args, world,
                                                             local, peaks, peak_src)
    if pick in (None, "sym"):
        ex[workloads.SWA_SYM_GQA.name] = bench_prefill_variant(workloads.SWA_SYM_GQA, args,
                                                               world, local, peaks, peak_src)
    if pick in (None, "paged"):
        paged = bench_decode_paged(args, world, local, peaks, peak_src)
        ex["paged_" + paged["config"]["workload"]] = paged
    if pick in (None, "backward"):
        for x in (workloads.CAUSAL_MHA, workloads.ALIBI_MHA, workloads.DOC_SOFTCAP):
            ex["backward_" + x.name] = bench_backward(x, args, world, local, peaks, peak_src)
    if pick in (None, "fp8"):
        ex["fp8_" + workloads.CAUSAL_MHA.name] = bench_fp8(
            workloads.CAUSAL_MHA, args, world, local, peaks, peak_src)
    return ex


def decode_workload(args, world: int = 1):
    """This rank's part of the decode workload, with the batch overridden by --decode-batch
    (smaller caches for profiler captures)."""
    import dataclasses
    w = workloads.DECODE
    if args.decode_batch:
        w = dataclasses.replace(w, B=args.decode_batch, name=w.name.replace(
            f"b{w.B}_", f"b{args.decode_batch}_"))
    return my_part(w, world)


def tensor_peak_at_clock(sm_mhz, n_sms: int) -> float | None:
    """Dense bf16 tensor throughput (TFLOP/s) of the chip at the sampled SM clock: one
    128x128x16 tcgen05 product (524288 flops) every 64 cycles per SM, measured with a probe,
    i.e. 8192 flops per cycle per SM."""
    if not sm_mhz:
        return None
    return 8192.0 * n_sms * sm_mhz * 1e6 / 1e12


def prefill_roofline(flops, executed, kernel_ms, peaks, peak_src, clocks, kernel, traffic,
                     n_sms):
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = flops / (kernel_ms * 1e-3) / 1e12
    exe = executed / (kernel_ms * 1e-3) / 1e12
    at_clk = tensor_peak_at_clock(clocks.get("sm_mhz"), n_sms)
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "peak_source": f"bf16_tflops (burst, {peak_src})",
            "frac_of_spec": round(achieved / SPEC_PEAKS["bf16_tflops"], 4),
            "executed_tflops": round(exe, 2),
            "tensor_peak_at_clock": round(at_clk, 1) if at_clk else None,
            "executed_frac_at_clock": round(exe / at_clk, 4) if at_clk else None,
            "kernel_ms": round(kernel_ms, 4), "kernel": kernel, "traffic": traffic}


def bench_prefill_variant(w, args, world, local, peaks, peak_src, steps=None):
    """Useful TFLOP/s of attn_fwd on a prefill workload other than the headline (sliding-
    window GQA, packed documents with soft-cap, ALiBi, symmetric window): the same timing as
    the headline, fewer steps."""
    import torch
    import io_aware_softmax_b200 as attn
    w_full, w = w, my_part(w, world)
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = workloads.make_inputs(w, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    slopes = (torch.tensor(workloads.workload_alibi_slopes(w), dtype=torch.float32, device=dev)
              if w.alibi else None)
    docs = workloads.workload_doc_offsets(w)
    doc_t = None if docs is None else torch.from_numpy(docs).to(dev)
    flops = accounting.prefill_useful_flops(w.B, w.Hq, w.Nq, w.Nk, w.d, w.mask_kind, w.window,
                                            docs)
    executed = accounting.prefill_executed_flops(w.B, w.Hq, w.Nq, w.Nk, w.d, w.mask_kind,
                                                 w.window, docs)

    def step():
        attn.attn_fwd(q, k, v, scale=w.scale, mask=w.mask_kind, window=w.window,
                      softcap=w.softcap, doc_offsets=doc_t, alibi_slopes=slopes, out=o, lse=lse)

    steps = steps or max(3, min(args.steps, 30))
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        total_ms, per = time_launches(step, steps, world)
    if attn.device_status() != 0:
        raise RuntimeError(f"device status not ok after {w.name}")
    ms = max_over_ranks(world, total_ms / steps)
    kernel_ms = max_over_ranks(world, sum(per) / len(per))
    clocks = clk.summary()
    kernel = "attn_fwd_sm100_kernel<%d>%s" % (w.d, " (ALiBi)" if w.alibi else "")
    cfg = {**w.describe(), "l2": l2_note(q, k, v), "parallelism": split_note(w_full, w, world)}
    if docs is not None:
        cfg["num_docs"] = len(docs) - 1
    res = {"config": cfg,
           "value": round(whole_job_rate(flops, world, ms) / 1e12, 2),
           "unit": "TFLOP/s", "ms_per_step": round(ms, 4), "steps": steps,
           "useful_tflop_per_step": round(flops / 1e12, 4),
           "executed_tflop_per_step": round(executed / 1e12, 4),
           "roofline": prefill_roofline(flops, executed, kernel_ms, peaks, peak_src, clocks,
                                        kernel, recorded_traffic("prefill_" + w.name),
                                        torch.cuda.get_device_properties(dev).multi_processor_count),
           "gpu_launches": steps, "clocks": clocks}
    del q, k, v, o, lse
    torch.cuda.empty_cache()
    return res


def bench_decode_paged(args, world, local, peaks, peak_src, page: int = 256):
    """The decode workload on a paged cache: 256-row pages placed by a seeded permutation,
    every sequence at full length (the same KV bytes as the contiguous line)."""
    import torch
    import io_aware_softmax_b200 as attn
    w = decode_workload(args, world)
    dev = torch.device("cuda", torch.cuda.current_device())
    max_pages = w.Nk // page
    num_pages = w.B * max_pages
    q = workloads.randn_bf16((w.B, w.Hq, 1, w.d), w.seed, 0, 1.0, dev)
    kp = workloads.randn_bf16((num_pages, w.Hkv, page, w.d), w.seed, 1, 1.0, dev)
    vp = workloads.randn_bf16((num_pages, w.Hkv, page, w.d), w.seed, 2, 1.0, dev)
    perm = np.random.default_rng(w.seed).permutation(num_pages).astype(np.int32)
    table = torch.from_numpy(perm.reshape(w.B, max_pages)).to(dev)
    lens = torch.full((w.B,), w.Nk, dtype=torch.int32, device=dev)
    S = attn.default_splits(w.B, w.Hkv, w.Nk, dev.index)
    ws = torch.empty(attn.decode_workspace_bytes(w.B, w.Hq, w.d, S), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, 1), dtype=torch.float32, device=dev)

    def step():
        attn.attn_decode_paged(q, kp, vp, table, lens, scale=w.scale, num_splits=S, workspace=ws,
                               out=o, lse=lse)

    steps = max(3, min(args.steps, 30))
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        total_ms, per = time_launches(step, steps, world)
    if attn.device_status() != 0:
        raise RuntimeError("device status not ok after paged decode")
    ms = max_over_ranks(world, total_ms / steps)
    call_ms = max_over_ranks(world, sum(per) / len(per))
    kv = accounting.decode_kv_bytes(w.B, w.Hkv, w.Nk, w.d)
    io = accounting.decode_io_bytes(w.B, w.Hq, w.Hkv, w.Nk, w.d) + w.B * max_pages * 4 + w.B * 4
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    res = {"config": {**w.describe(), "page_size": page, "num_pages": num_pages,
                      "l2": l2_note(kp, vp),
                      "placement": "seeded permutation", "seq_lens": "all T"},
           "value": round(whole_job_rate(kv, world, ms) / 1e9, 1), "unit": "GB/s (KV cache)",
           "tokens_per_s": round(w.B * world / (ms * 1e-3), 1), "ms_per_step": round(ms, 4),
           "steps": steps, "num_splits": S,
           "roofline": {"bound": "hbm", "achieved": round(io / (call_ms * 1e-3) / 1e9, 1),
                        "peak": peak, "unit": "GB/s",
                        "frac": round(io / (call_ms * 1e-3) / 1e9 / peak, 4),
                        "peak_source": f"hbm_gbs ({peak_src})",
                        "kernel": "attn_decode_split_kernel (paged) + attn_merge_kernel "
                                  "(one call)",
                        "traffic": recorded_traffic("paged_decode")},
           "gpu_launches": 2 * steps, "clocks": clk.summary()}
    del q, kp, vp, o, lse, ws
    torch.cuda.empty_cache()
    return res


def bench_backward(w, args, world, local, peaks, peak_src):
    """Useful TFLOP/s of attn_bwd (dQ, dK, dV from O, LSE and dO) on a prefill workload
    (attn_bwd_alibi when the workload carries ALiBi slopes; its documents and soft-cap too)."""
    import torch
    import io_aware_softmax_b200 as attn
    w = my_part(w, world)
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = workloads.make_inputs(w, device=dev)
    dout = workloads.randn_bf16((w.B, w.Hq, w.Nq, w.d), w.seed, 3, 1.0, dev, w.b0)
    slopes = (torch.tensor(workloads.workload_alibi_slopes(w), dtype=torch.float32, device=dev)
              if w.alibi else None)
    docs = workloads.workload_doc_offsets(w)
    doc_t = None if docs is None else torch.tensor(docs, dtype=torch.int32, device=dev)
    o, lse = attn.attn_fwd(q, k, v, scale=w.scale, mask=w.mask_kind, window=w.window,
                           alibi_slopes=slopes, softcap=w.softcap, doc_offsets=doc_t)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(attn.bwd_workspace_bytes(w.B, w.Hq, w.Nq), dtype=torch.uint8, device=dev)
    flops = accounting.backward_useful_flops(w.B, w.Hq, w.Nq, w.Nk, w.d, w.mask_kind, w.window,
                                             docs)

    def step():
        attn.attn_bwd(q, k, v, o, lse, dout, scale=w.scale, mask=w.mask_kind, window=w.window,
                      dq=dq, dk=dk, dv=dv, workspace=ws, alibi_slopes=slopes,
                      softcap=w.softcap, doc_offsets=doc_t)

    steps = max(3, min(args.steps, 20))
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        total_ms, per = time_launches(step, steps, world)
    if attn.device_status() != 0:
        raise RuntimeError("device status not ok after the backward pass")
    ms = max_over_ranks(world, total_ms / steps)
    call_ms = max_over_ranks(world, sum(per) / len(per))
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = flops / (call_ms * 1e-3) / 1e12
    res = {"config": {**w.describe(), "l2": l2_note(q, k, v, o, dout)},
           "value": round(whole_job_rate(flops, world, ms) / 1e12, 2),
           "unit": "TFLOP/s", "ms_per_step": round(ms, 4), "steps": steps,
           "useful_tflop_per_step": round(flops / 1e12, 4),
           "flop_accounting": "10 d per visible pair (S, dP, dV, dQ, dK)",
           "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                        "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                        "peak_source": f"bf16_tflops (burst, {peak_src})",
                        "kernel": "attn_bwd_rowdot + attn_bwd_dq + attn_bwd_dkdv (one call)"
                                  + (" (ALiBi)" if w.alibi else "")
                                  + (" (soft-cap)" if w.softcap else ""),
                        "traffic": (None if (w.alibi or w.softcap or w.docs)
                                    else recorded_traffic("backward"))},
           "gpu_launches": 3 * steps, "clocks": clk.summary()}
    del q, k, v, o, lse, dout, dq, dk, dv, ws, slopes, doc_t
    torch.cuda.empty_cache()
    return res


def bench_fp8(w, args, world, local, peaks, peak_src):
    """Useful TFLOP/s of attn_fwd_fp8 on a prefill workload: Q and K quantized per 128-row
    block after the seeded random-sign Hadamard rotation, V per head and transposed; the
    quantization runs before the timed region and is timed on its own."""
    import torch
    import io_aware_softmax_b200 as attn
    w = my_part(w, world)
    dev = torch.device("cuda", torch.cuda.current_device())
    q, k, v = workloads.make_inputs(w, device=dev)
    signs = torch.from_numpy(np.random.default_rng(w.seed).choice([-1.0, 1.0], w.d)
                             .astype(np.float32)).to(dev)

    def quant():
        q8, qs = attn.quantize_fp8(q, block_rows=128, signs=signs)
        k8, ks = attn.quantize_fp8(k, block_rows=128, signs=signs)
        vt8, vs = attn.quantize_fp8(v, block_rows=w.Nk, transpose=True)
        return q8, qs, k8, ks, vt8, vs[:, :, 0].contiguous()

    for _ in range(2):
        inputs = quant()
    torch.cuda.synchronize()
    qt_ms, _ = time_launches(quant, 3, world)
    q8, qs, k8, ks, vt8, vs = inputs
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    flops = accounting.prefill_useful_flops(w.B, w.Hq, w.Nq, w.Nk, w.d, w.mask_kind, w.window)

    def step():
        attn.attn_fwd_fp8(q8, qs, k8, ks, vt8, vs, scale=w.scale, mask=w.mask_kind,
                          window=w.window, out=o, lse=lse)

    steps = max(3, min(args.steps, 30))
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        total_ms, per = time_launches(step, steps, world)
    if attn.device_status() != 0:
        raise RuntimeError("device status not ok after the FP8 prefill")
    ms = max_over_ranks(world, total_ms / steps)
    call_ms = max_over_ranks(world, sum(per) / len(per))
    peak = 2.0 * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = flops / (call_ms * 1e-3) / 1e12
    # the whole FP8 path from bf16 inputs: quantize Q, K, V, then the FP8 prefill
    def full_step():
        q8_, qs_, k8_, ks_, vt8_, vs_ = quant()
        attn.attn_fwd_fp8(q8_, qs_, k8_, ks_, vt8_, vs_, scale=w.scale, mask=w.mask_kind,
                          window=w.window, out=o, lse=lse)

    for _ in range(2):
        full_step()
    torch.cuda.synchronize()
    full_ms, _ = time_launches(full_step, steps, world)
    full_ms = max_over_ranks(world, full_ms / steps)
    quant_bytes = 3 * q.numel() * 2 + 3 * q.numel()   # bf16 read, E4M3 written (Hq = Hkv)
    qt = max_over_ranks(world, qt_ms / 3)
    res = {"config": {**w.describe(), "dtype": "e4m3 (P e4m3), bf16 O",
                      "l2": l2_note(q8, k8, vt8),
                      "scales": "Q, K per 128 rows after Hadamard rotation; V per head"},
           "with_quantize": {"value": round(whole_job_rate(flops, world, full_ms) / 1e12, 2),
                             "unit": "TFLOP/s", "ms_per_step": round(full_ms, 4),
                             "note": "quantization of the bf16 Q, K, V inside the timed step"},
           "quantize": {"ms": round(qt, 4), "bytes": quant_bytes,
                        "gbs": round(quant_bytes / (qt * 1e-3) / 1e9, 1),
                        "frac_of_hbm": round(quant_bytes / (qt * 1e-3) / 1e9 /
                                             float(peaks.get("hbm_gbs",
                                                             FALLBACK_PEAKS["hbm_gbs"])), 4),
                        "launches": "Q, K, V: 1 each (V transposed, one scale per head, a cluster of 8 CTAs per head)",
                        "traffic": {"quant_rows (Q or K)": recorded_traffic("quant_rows"),
                                    "quant_vt (V)": recorded_traffic("quant_vt")}},
           "accuracy": fp8_accuracy(w),
           "value": round(whole_job_rate(flops, world, ms) / 1e12, 2), "unit": "TFLOP/s",
           "ms_per_step": round(ms, 4), "steps": steps,
           "useful_tflop_per_step": round(flops / 1e12, 4),
           "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                        "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                        "peak_source": f"2 x bf16_tflops (burst, {peak_src}): the nominal "
                                       "fp8 / bf16 ratio",
                        "kernel": "attn_fwd_sm100_kernel<128> (E4M3)",
                        "traffic": recorded_traffic("fp8")},
           "gpu_launches": steps, "clocks": clk.summary()}
    del q, k, v, q8, k8, vt8, o, lse
    torch.cuda.empty_cache()
    return res


def fp8_accuracy(w, heads: int = 4, n: int = 1024, seed: int = 71) -> dict:
    """FP8 output error against the bf16 path (attn_fwd) on the same inputs, with and without
    the Hadamard rotation: N(0,1) inputs whose Q and K carry 0.1 % outlier entries of std 10,
    causal, d = 128, a few heads of the workload's length scale."""
    import torch
    import io_aware_softmax_b200 as attn
    dev = torch.device("cuda", torch.cuda.current_device())
    gen = torch.Generator(device=dev).manual_seed(seed)
    q, k, v = (workloads.randn_bf16((1, heads, n, w.d), seed, i, 1.0, dev) for i in range(3))
    for t in (q, k):
        hit = torch.rand(t.shape, generator=gen, device=dev) < 1e-3
        t[hit] = (torch.randn(t.shape, generator=gen, device=dev)[hit] * 10.0).to(t.dtype)
    o_ref, l_ref = attn.attn_fwd(q, k, v, mask="causal")
    out = {"vs": "attn_fwd (bf16) on the same inputs",
           "input": f"1x{heads}x{n}x{w.d}, causal, N(0,1) with 0.1 % outlier entries (std 10) "
                    "in Q and K"}
    for name, rot in (("rotated", True), ("plain", False)):
        signs = (torch.from_numpy(np.random.default_rng(seed).choice([-1.0, 1.0], w.d)
                                  .astype(np.float32)).to(dev) if rot else None)
        q8, qs = attn.quantize_fp8(q, block_rows=128, signs=signs)
        k8, ks = attn.quantize_fp8(k, block_rows=128, signs=signs)
        vt8, vs = attn.quantize_fp8(v, block_rows=n, transpose=True)
        o, l = attn.attn_fwd_fp8(q8, qs, k8, ks, vt8, vs[:, :, 0].contiguous(), mask="causal")
        err = (o.float() - o_ref.float())
        out[name] = {"o_rmse": round(float(err.pow(2).mean().sqrt()), 6),
                     "o_max": round(float(err.abs().max()), 5),
                     "lse_max": round(float((l - l_ref).abs().max()), 6)}
    return out


def e2e_prefill(w, args, world, q, k, v):
    """Same metric through the public API with host buffers: every step copies q, k, v from
    pinned host memory, runs attn_fwd and reads O and LSE back.  Steps are pipelined over
    two device buffer sets and three streams, so step i + 1's host-to-device copies and
    step i - 1's device-to-host copies run while step i computes (PCIe is full duplex);
    the timed region spans the first step's copies in to the last step's copies out."""
    import torch
    import io_aware_softmax_b200 as attn
    hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
    ho = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    hl = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32).pin_memory()
    sets = [dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v),
                 o=torch.empty_like(q),
                 lse=torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=q.device))
            for _ in range(2)]
    s_in, s_run, s_out = (torch.cuda.Stream(device=q.device) for _ in range(3))
    ev = [{n: torch.cuda.Event() for n in ("in", "run", "out")} for _ in range(2)]
    used = [False, False]

    def step(i):
        b = i % 2
        d, e = sets[b], ev[b]
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(e["out"])          # this set's previous step fully done
                s_in.wait_event(e["run"])
            d["q"].copy_(hq, non_blocking=True)
            d["k"].copy_(hk, non_blocking=True)
            d["v"].copy_(hv, non_blocking=True)
            e["in"].record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(e["in"])
            attn.attn_fwd(d["q"], d["k"], d["v"], scale=w.scale, mask=w.mask_kind,
                          out=d["o"], lse=d["lse"])
            e["run"].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(e["run"])
            ho.copy_(d["o"], non_blocking=True)
            hl.copy_(d["lse"], non_blocking=True)
            e["out"].record(s_out)
        used[b] = True

    steps = max(3, min(args.steps, 10))
    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(steps):
        step(i)
    # the timed region ends when every stream has finished
    for st in (s_run, s_out):
        s_in.wait_stream(st)
    t1.record(s_in)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(world, t0.elapsed_time(t1) / steps)
    flops = accounting.prefill_useful_flops(w.B, w.Hq, w.Nq, w.Nk, w.d, w.mask_kind)
    return {"value": round(flops * world / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": (q.numel() + k.numel() + v.numel()) * 2,
            "d2h_bytes_per_step": q.numel() * 2 +
            w.B * w.Hq * w.Nq * 4, "steps": steps, "ms_per_step": round(ms, 3),
            "pipeline": "2 device buffer sets, copy-in / compute / copy-out streams"}


def bench_decode(args, world, local, peaks, peak_src):
    import torch
    import io_aware_softmax_b200 as attn
    w = decode_workload(args, world)
    dev = torch.device("cuda", torch.cuda.current_device())
    q, kc, vc = workloads.make_inputs(w, device=dev)
    S = attn.default_splits(w.B, w.Hkv, w.Nk, dev.index)
    ws = torch.empty(attn.decode_workspace_bytes(w.B, w.Hq, w.d, S), dtype=torch.uint8,
                     device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, 1), dtype=torch.float32, device=dev)

    def step():
        attn.attn_decode(q, kc, vc, scale=w.scale, num_splits=S, workspace=ws, out=o, lse=lse)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        total_ms, per = time_launches(step, args.steps, world)
    if attn.device_status() != 0:
        raise RuntimeError("device status not ok after decode steps")
    ms = max_over_ranks(world, total_ms / args.steps)
    call_ms = max_over_ranks(world, sum(per) / len(per))
    kv = accounting.decode_kv_bytes(w.B, w.Hkv, w.Nk, w.d)
    io = accounting.decode_io_bytes(w.B, w.Hq, w.Hkv, w.Nk, w.d)
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    gbs = whole_job_rate(kv, world, ms) / 1e9
    res = {"workload": w.name, "l2": l2_note(kc, vc), "value": round(gbs, 1),
           "unit": "GB/s (KV cache)",
           "tokens_per_s": round(w.B * world / (ms * 1e-3), 1), "ms_per_step": round(ms, 4),
           "num_splits": S, "kv_bytes_per_step": kv,
           "roofline": {"bound": "hbm", "achieved": round(io / (call_ms * 1e-3) / 1e9, 1),
                        "peak": peak, "unit": "GB/s", "frac": round(io / (call_ms * 1e-3) / 1e9
                                                                   / peak, 4),
                        "peak_source": f"hbm_gbs ({peak_src})",
                        "frac_of_spec": round(io / (call_ms * 1e-3) / 1e9 / SPEC_PEAKS["hbm_gbs"],
                                              4),
                        "kernel": "attn_decode_split_kernel + attn_merge_kernel (one call)",
                        "traffic": recorded_traffic("decode")},
           "gpu_launches": 2 * args.steps, "clocks": clk.summary()}
    if not args.no_e2e:
        hk, hv = kc.cpu().pin_memory(), vc.cpu().pin_memory()
        hq = q.cpu().pin_memory()
        ho = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        hl = torch.empty((w.B, w.Hq, 1), dtype=torch.float32).pin_memory()

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            kc.copy_(hk, non_blocking=True)
            vc.copy_(hv, non_blocking=True)
            attn.attn_decode(q, kc, vc, scale=w.scale, num_splits=S, workspace=ws, out=o,
                             lse=lse)
            ho.copy_(o, non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        e2e_step()
        total, _ = time_launches(e2e_step, 3, world)
        ems = max_over_ranks(world, total / 3)
        res["e2e"] = {"value": round(kv * world / (ems * 1e-3) / 1e9, 2), "unit": "GB/s",
                      "h2d_bytes_per_step": kv + q.numel() * 2,
                      "d2h_bytes_per_step": q.numel() * 2 + w.B * w.Hq * 4, "steps": 3}
    return res


# ------------------------------------------------------------------------ reference arm
def run_reference(args, world, rank):
    """The fp64 CPU oracle, as it stands, on the host cores: each step is one whole head of
    the causal multi-head workload (a bounded sample of the same workload)."""
    import oracle
    w = workloads.CAUSAL_MHA
    q, k, v = (x.float().numpy() for x in _cpu_head_inputs(w, 0))
    pairs = accounting.visible_pairs(w.Nq, w.Nk, w.mask_kind)
    rows = np.arange(w.Nq)

    def step(h):
        for r0 in range(0, w.Nq, 256):
            rr = rows[r0:r0 + 256]
            oracle.attention_head(q[h, rr], rr, k[h], v[h], w.scale, w.mask_kind)

    for i in range(args.warmup):
        step(i % w.Hq)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step((args.warmup + i) % w.Hq)
    dt = time.perf_counter() - t0
    ms = dt * 1e3 / args.steps
    value = 4 * w.d * pairs / (ms * 1e-3) / 1e12
    cores = blas_threads()
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.Nq, "d": w.d,
                   "mask": "causal", "sample_per_step": "one whole head (b=0), 4096 rows"},
        "cpu_baseline": {"value": round(value, 5), "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle", "sample": "one whole head of the workload per step"},
        "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the ALiBi and symmetric-window prefill lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle time")
    ap.add_argument("--only", choices=["all", "prefill", "decode", "extras"], default="all",
                    help="run one part only (profiling runs)")
    ap.add_argument("--workload", choices=sorted(n for n, x in workloads.BY_NAME.items()
                                                 if x.kind == "prefill"), default=None,
                    help="time attn_fwd on this prefill workload only (profiling runs)")
    ap.add_argument("--extra", choices=["alibi", "sym", "paged", "backward", "fp8"],
                    default=None, help="with --only extras: that line alone (profiling runs)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="decode batch size override (smaller caches for ncu captures)")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, world, rank)), flush=True)
        return 0
    world, rank, local = dist_setup(args.gpus)
    out = run_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
