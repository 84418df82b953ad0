#!/usr/bin/env python
"""Benchmark: FP8 NT GEMM with fine-grained scaling on B200 (one process per GPU).

One step = one call of the library's dense FP8 GEMM on the workload M=4096, N=7168, K=7168 (A and B e4m3
with power-of-two 1x128 / 128x128 scales, bf16 out; seeded synthetic inputs), the configuration the
headline metric is quoted on.  Other workloads can be timed with --workload for reference (the default line
is the contract line): 1 dense 128x256x512; 3 and 5 contiguous grouped; 4 masked grouped; 6 no-padding grouped;
7 contiguous with B in the NN orientation; 8 K-grouped with fp32 output; 9 contiguous W4A8 (B in E2M1);
10 workload 2 with fp32 (non-power-of-two) scales, through the fp32 scale-promotion path.  The default line
also times workloads 3, 4 and 5 (under "grouped", the M-grouped half of the metric) and workload 1 (under
"latency") in the same process with the same protocol.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload 2]

Timing: inputs resident in HBM; each step is bracketed by CUDA events on the launching stream; between
steps a 512 MB buffer is rewritten to flush the 126 MB L2 (outside the events).  The timed loop is
bracketed by a barrier and a device synchronise, and the per-step time is the max over ranks.  N > 1 runs
N independent replicas (weak scaling; the GEMM has no exchange step).

End to end (the "e2e" key): every step uploads its inputs from pinned host memory, runs the call and reads
its whole result back; steps are pipelined over an upload stream, the compute stream and a read-back stream
with two device buffer sets, so the bound is the busier PCIe direction.
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FP8_OVER_BF16 = 2.0  # nominal dense FP8 / BF16 tensor throughput ratio (4.5 / 2.25 PFLOP/s)
# Dense FP8 tensor FLOPs per SM per clock: a 128 x 224 x 32 block-scaled MMA issues every 112 cycles when nothing
# else holds it (an issue-loop micro-benchmark on this GPU); twice the 8192 of BF16 (the measured cuBLAS BF16 peak
# equals 148 x 8192 x the SM clock it ran at).
FP8_FLOP_PER_SM_CLOCK = 16384
METRIC = "FP8 GEMM TFLOPS (dense and M-grouped)"
GROUPED_WORKLOADS = (3, 4, 5)  # the M-grouped half of the metric, timed beside the dense headline
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["moe_grouped_gemm_03_b200/csrc/gemm_kernel.cuh", "moe_grouped_gemm_03_b200/csrc/ptx.cuh",
                  "moe_grouped_gemm_03_b200/csrc/dg_api.cu", "moe_grouped_gemm_03_b200/csrc/scale_pack.cuh",
                  "moe_grouped_gemm_03_b200/csrc/transpose.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=2, choices=[1, 2, 3, 4, 5, 6, 7, 8, 9, 10])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--grouped", default="auto",
                    help="comma-separated workloads timed after the main one and reported under 'grouped' "
                         "(auto: 3,4,5 when the main workload is 2 on one GPU; none: skip)")
    ap.add_argument("--latency", default="auto",
                    help="comma-separated latency-bound workloads timed after the grouped ones and reported under "
                         "'latency' (auto: 1 when the main workload is 2 on one GPU; none: skip)")
    ap.add_argument("--ref-seconds", type=float, default=30.0,
                    help="reference arm: wall time of all warm-up and timed oracle steps together")
    return ap.parse_args()


def strip_comments(src: str) -> str:
    """C/C++/CUDA source without comments and blank lines (string and character literals kept as written), so a
    comment edit does not count as a kernel change."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c in "\"'":  # a literal, up to its unescaped closing quote
            j = i + 1
            while j < n and src[j] != c:
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            while i < n and src[i] != "\n":
                i += 1
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    lines = [ln.rstrip() for ln in "".join(out).splitlines()]
    return "\n".join(ln for ln in lines if ln.strip())


def kernel_source_hash():
    """Hash of the kernel sources' code (comments and blank lines ignored): recorded ncu traffic is used only
    while it matches."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            h.update(strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def recorded_traffic(workload):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    rec = d.get(str(workload))
    if not rec or rec.get("kernel_hash") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(0.01)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def dist_setup(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    device = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(flops_per_rank, local_ms, world):
    """(slowest rank's ms per step, TFLOP/s of all ranks together): every rank runs its own replica of the
    workload, so the job processes world x flops_per_rank per step in the slowest rank's time."""
    ms = max_over_ranks(local_ms, world)
    return ms, world * flops_per_rank / (ms * 1e-3) / 1e12


def call_library(p, t, out):
    import moe_grouped_gemm_03_b200 as dg

    if p.kind == "dense":
        dg.fp8_gemm_nt((t["a"], t["sfa"]), (t["b"], t["sfb"]), out)
    elif p.kind == "contiguous":
        dg.m_grouped_fp8_gemm_nt_contiguous((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, t["m_indices"])
    elif p.kind == "k_grouped":  # D = the products (no C)
        dg.k_grouped_fp8_gemm_nt_contiguous((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, p.counts.tolist(), t["ks"])
    elif p.kind == "contiguous_w4a8":
        dg.m_grouped_fp8_fp4_gemm_nt_contiguous((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, t["m_indices"])
    elif p.kind == "contiguous_nn":
        dg.m_grouped_fp8_gemm_nn_contiguous((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, t["m_indices"])
    elif p.kind == "nopad":
        dg.m_grouped_fp8_gemm_nt_nopad((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, t["counts"])
    else:
        dg.m_grouped_fp8_gemm_nt_masked((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, t["masked_m"], p.expected_m)


LATENCY_WORKLOADS = (1,)  # the default line's latency-bound workload (the small dense call)
PROMOTION_WORKLOADS = (10,)  # run with fp32 scale promotion (their scales are not powers of two)


def launches_per_call(p, promotion=False):
    """The library's kernels one call launches: the scale pre-pass and the GEMM (the fp32 scale-promotion GEMM has no
    pre-pass; a short dense call -- K <= 2048 and 2MNK <= 2^34 -- runs that GEMM alone on its power-of-two
    scales).  The NN call reads B in place through the swapped-operand tiles when its 128-row blocks fit their
    tables (M_total / 128 <= 1024) and promotion is off; otherwise it transposes B first (one more launch)."""
    transpose = p.kind == "contiguous_nn" and (promotion or p.rows // 128 > 1024)
    short_dense = p.kind == "dense" and p.K <= 2048 and 2 * p.M * p.N * p.K <= 1 << 34
    return (2 if transpose else 1) + (0 if promotion or short_dense else 1)


def algorithmic_bytes(p):
    """Each valid A row once, each active group's B once, the scales of those, each valid D row once.
    K-grouped: A and B once, their per-row scales, fp32 D once (no C in the timed call)."""
    import numpy as np

    if p.kind == "contiguous_w4a8":  # B is half a byte per element, with one 4-byte scale per row per 128 K
        rows = p.valid_rows()
        groups = np.unique(p.row_groups(rows)) if len(rows) else []
        nkb = p.K // 128
        return int(len(rows) * p.K + len(groups) * p.N * p.K // 2 + len(rows) * nkb * 4
                   + len(groups) * p.N * nkb * 16 + len(rows) * p.N * 2)
    if p.kind == "k_grouped":
        nkb = p.K // 128
        return int((p.M + p.N) * p.K + (p.M + p.N) * nkb * 4 + p.G * p.M * p.N * 4)

    rows = p.valid_rows()
    nkb = p.K // 128
    groups = np.unique(p.row_groups(rows)) if len(rows) else []
    nnb = (p.N + 127) // 128
    return int(len(rows) * p.K + len(groups) * p.N * p.K + len(rows) * nkb * 4 + len(groups) * nnb * nkb * 4
               + len(rows) * p.N * 2)


def oracle_sample(p, seconds, rng_seed=0):
    """Time the oracle on a bounded random sample of valid rows (about `seconds` of CPU time)."""
    import numpy as np

    import oracle

    valid = p.valid_rows()
    rng = np.random.default_rng(rng_seed)
    n = min(len(valid), 4)
    t0 = time.perf_counter()
    oracle.problem_rows(p, np.sort(rng.choice(valid, n, replace=False)))
    dt = max(time.perf_counter() - t0, 1e-6)
    n = int(min(len(valid), max(n, n * seconds / dt)))
    rows = np.sort(rng.choice(valid, n, replace=False))
    t0 = time.perf_counter()
    oracle.problem_rows(p, rows)
    dt = time.perf_counter() - t0
    flops = 2.0 * n * p.N * p.K
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{n} random valid rows x all {p.N} columns of the workload (seed {rng_seed}); "
                      f"{dt:.2f} s wall for {flops / 1e9:.1f} GFLOP in fp64"}


def workload_config(p, world, promotion):
    """The `config` object of both arms: the workload, its scales and the timing protocol."""
    if promotion:
        scales = "fp32, promoted per 128-K block"
    elif launches_per_call(p) == 1:  # a short dense call: one kernel
        scales = "powers of two, applied per 128-K block by the promotion GEMM (short call: no pre-pass)"
    else:
        scales = "powers of two (UE8M0, block-scaled MMA)"
    return {"workload": p.name, "M": p.M, "N": p.N, "K": p.K, "G": p.G, "scales": scales,
            "l2": "flushed between steps (512 MB write outside the timed events)",
            "parallelism": f"{world} independent replicas" if world > 1 else "1 GPU"}


def run_reference(args, world, rank):
    """Reference arm: the CPU oracle, as it stands, on bounded samples of the same workload.  It runs the requested
    --warmup and --steps; every step times the oracle on a fresh random sample of valid rows (all columns), sized so
    that all warm-up and timed steps together take about --ref-seconds of wall time."""
    import synth

    if rank != 0:
        return
    p = synth.make_config(args.workload)
    import numpy as np

    import oracle

    valid = p.valid_rows()
    rng = np.random.default_rng(1)
    probe = time.perf_counter()
    oracle.problem_rows(p, np.sort(rng.choice(valid, 2, replace=False)))
    per_row = (time.perf_counter() - probe) / 2
    steps, warm = max(1, args.steps), max(0, args.warmup)
    per_step = min(3.0, max(0.01, args.ref_seconds / (steps + warm)))
    rows_per_step = int(max(1, min(len(valid), per_step / max(per_row, 1e-9))))
    for _ in range(warm):
        oracle.problem_rows(p, np.sort(rng.choice(valid, rows_per_step, replace=False)))
    times = []
    for _ in range(steps):
        rows = np.sort(rng.choice(valid, rows_per_step, replace=False))
        t0 = time.perf_counter()
        oracle.problem_rows(p, rows)
        times.append(time.perf_counter() - t0)
    flops = 2.0 * rows_per_step * p.N * p.K
    value = flops / statistics.mean(times) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warm, "ms_per_step": 1e3 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(p, world, args.workload in PROMOTION_WORKLOADS),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"{rows_per_step} random valid rows x all {p.N} columns per step "
                                   f"({2 * rows_per_step * p.N * p.K / 1e9:.1f} GFLOP in fp64)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def time_steps(p, t, out, flush, steps, warmup, world, promotion):
    """Warm up, then time `steps` calls, each bracketed by CUDA events on the launching stream with an L2 flush
    between them (outside the events).  NVML samples clocks during the timed loop, and the library's clock record
    gives the SM clock the GEMM launches themselves ran at (the board's power limit holds it below the maximum
    while the tensor cores are busy, a drop NVML's 10 ms samples mostly miss between the short launches)."""
    import torch

    import moe_grouped_gemm_03_b200 as dg

    stream = torch.cuda.current_stream()
    for _ in range(max(warmup, 3)):
        call_library(p, t, out)
    torch.cuda.synchronize()
    dg.check_device_error()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    clocks = ClockSampler(torch.cuda.current_device())
    dg.debug_clock_read(reset=True)
    barrier(world)
    torch.cuda.synchronize()
    dg.debug_clock_record(True)
    with clocks:
        for i in range(steps):
            flush.fill_(i)
            starts[i].record(stream)
            call_library(p, t, out)
            ends[i].record(stream)
        torch.cuda.synchronize()
    dg.debug_clock_record(False)
    barrier(world)
    dg.check_device_error()
    cycles, ns, launches = dg.debug_clock_read(reset=True)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    summary = clocks.summary()
    summary["sm_mhz_in_kernel"] = 1e3 * cycles / ns if ns else None
    summary["in_kernel_launches"] = launches
    return step_ms, summary


def roofline_for(p, workload, mean_ms, peaks, peak_src, clocks, num_sms):
    """Roofline of one workload's GEMM.  `peak` is the contract's: the measured bf16 burst peak x the nominal
    FP8/BF16 ratio 2.  `clock_consistent` restates it from the SM clock the GEMM ran at (the library's clock
    record) and from the maximum clock, at FP8_FLOP_PER_SM_CLOCK."""
    flops = p.flops()
    achieved = flops / (mean_ms * 1e-3) / 1e12
    fp8_peak = peaks["bf16_tflops"] * FP8_OVER_BF16
    nbytes = algorithmic_bytes(p)
    hbm_gbs = nbytes / (mean_ms * 1e-3) / 1e9
    mhz = clocks.get("sm_mhz_in_kernel")
    max_mhz = clocks.get("sm_max_mhz") or peaks.get("sm_max_mhz")
    at_clock = num_sms * FP8_FLOP_PER_SM_CLOCK * mhz / 1e6 if mhz else None
    at_max = num_sms * FP8_FLOP_PER_SM_CLOCK * max_mhz / 1e6 if max_mhz else None
    roof = {"bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
            "frac": achieved / fp8_peak, "traffic": recorded_traffic(workload),
            "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} x nominal fp8/bf16 ratio 2",
            "clock_consistent": {
                "fp8_flop_per_sm_clock": FP8_FLOP_PER_SM_CLOCK, "sms": num_sms,
                "sm_mhz_in_kernel": mhz, "peak_at_kernel_clock": at_clock,
                "frac_at_kernel_clock": achieved / at_clock if at_clock else None,
                "sm_max_mhz": max_mhz, "peak_at_max_clock": at_max,
                "frac_at_max_clock": achieved / at_max if at_max else None},
            "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": nbytes,
            "hbm_gbs_achieved": hbm_gbs, "hbm_peak_gbs": peaks["hbm_gbs"]}
    if p.kind in ("masked", "masked_w4a8"):
        roof.update(bound="hbm", achieved=hbm_gbs, peak=peaks["hbm_gbs"], unit="GB/s", frac=hbm_gbs / peaks["hbm_gbs"],
                    peak_source=f"{peak_src} HBM copy bandwidth", tflops_achieved=achieved)
    return roof


def run_grouped(workloads, args, world, local, flush, peaks, peak_src, num_sms):
    """The M-grouped half of the metric, timed in the same process with the same protocol as the main line."""
    import torch

    import synth

    res = {}
    for w in workloads:
        p = synth.make_config(w)
        promotion = w in PROMOTION_WORKLOADS
        import moe_grouped_gemm_03_b200 as dg

        dg.set_fp32_scale_promotion(promotion)
        t = synth.to_torch(p, f"cuda:{local}")
        out = torch.empty(p.out_shape(), dtype=torch.float32 if p.kind == "k_grouped" else torch.bfloat16,
                          device=f"cuda:{local}")
        step_ms, clocks = time_steps(p, t, out, flush, args.steps, args.warmup, world, promotion)
        ms, value = whole_job_throughput(p.flops(), statistics.mean(step_ms), world)
        res[str(w)] = {"workload": p.name, "value": value, "unit": "TFLOP/s", "ms_per_step": ms,
                       "steps": args.steps, "warmup": max(args.warmup, 3),
                       "roofline": roofline_for(p, w, statistics.mean(step_ms), peaks, peak_src, clocks, num_sms),
                       "clocks": clocks, "gpu_launches": args.steps * launches_per_call(p, promotion),
                       "config": workload_config(p, world, promotion)}
        del t, out
        torch.cuda.empty_cache()
    return res


def run_ours(args, world, rank, local):
    import torch

    import moe_grouped_gemm_03_b200 as dg
    import synth

    p = synth.make_config(args.workload)
    promotion = args.workload in PROMOTION_WORKLOADS
    dg.set_fp32_scale_promotion(promotion)
    t = synth.to_torch(p, f"cuda:{local}")
    out_dtype = torch.float32 if p.kind == "k_grouped" else torch.bfloat16
    out = torch.empty(p.out_shape(), dtype=out_dtype, device=f"cuda:{local}")
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.int32, device=f"cuda:{local}")
    stream = torch.cuda.current_stream()
    flops = p.flops()
    num_sms = torch.cuda.get_device_properties(local).multi_processor_count

    K = args.steps
    step_ms, clocks = time_steps(p, t, out, flush, K, args.warmup, world, promotion)
    ms, value = whole_job_throughput(flops, statistics.mean(step_ms), world)

    # End to end through the public API: every step copies its inputs from pinned host memory to the device,
    # runs the call and reads its whole result back to pinned host memory.  Steps are pipelined over three
    # streams (host->device copies, the call, device->host copies) with two device buffer sets, so one step's
    # upload overlaps the previous step's read-back (the two PCIe directions use separate copy engines).
    ref_bytes = out.cpu().view(torch.uint8)  # the device-timed result
    host = {k: v.cpu().pin_memory() for k, v in t.items()}
    host_outs = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = host_outs[0].numel() * host_outs[0].element_size()
    # (the second output starts as a copy of the first: rows a grouped call leaves unwritten match too)
    bufs = [(t, out), ({k: torch.empty_like(v) for k, v in t.items()}, out.clone())]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    e2e_steps = max(3, min(K, 20))
    total = e2e_steps + 2  # two untimed steps first
    ev = lambda: torch.cuda.Event()
    called, read_back = [None] * total, [None] * total
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(total):
        ti, oi = bufs[i % 2]
        if i == 2:
            torch.cuda.synchronize()
            barrier(world)
            e_start.record(s_in)
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(called[i - 2])  # the call two steps back has read this buffer set
            for k in ti:
                ti[k].copy_(host[k], non_blocking=True)
            uploaded = ev()
            uploaded.record(s_in)
        stream.wait_event(uploaded)
        if i >= 2:
            stream.wait_event(read_back[i - 2])  # its result has been read back before it is overwritten
        call_library(p, ti, oi)
        called[i] = ev()
        called[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(called[i])
            host_outs[i % 2].copy_(oi, non_blocking=True)
            read_back[i] = ev()
            read_back[i].record(s_out)
    s_out.wait_stream(s_in)
    s_out.wait_stream(stream)
    e_end.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end) / e2e_steps, world)
    # the results read back equal the device-timed result bit for bit (same inputs, same kernels)
    if not all(torch.equal(h.view(torch.uint8), ref_bytes) for h in host_outs):
        raise RuntimeError("end-to-end results differ from the device-timed result")
    del bufs, host, host_outs, t, out, ref_bytes
    torch.cuda.empty_cache()

    peaks, peak_src = load_peaks()
    roofline = roofline_for(p, args.workload, statistics.mean(step_ms), peaks, peak_src, clocks, num_sms)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": K, "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8e4m3", "data": "synthetic",
        "config": workload_config(p, world, promotion),
        "plan": {"block_n": 128 if promotion else dg.select_block_n(
                     p.G * ((p.expected_m + 127) // 128) if p.kind == "masked" else (p.rows + 127) // 128,
                     p.N, dg.get_num_sms()),
                 "tflops_frac_of_fp8_peak": roofline["achieved"] / roofline["peak"] if roofline["unit"] == "TFLOP/s"
                 else None},
        "roofline": roofline,
        "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": K * launches_per_call(p, promotion),
        "clocks": clocks,
    }
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = oracle_sample(p, args.cpu_seconds)
    grouped = args.grouped
    if grouped == "auto":
        grouped = ",".join(str(w) for w in GROUPED_WORKLOADS) if args.workload == 2 and world == 1 else ""
    workloads = [int(w) for w in grouped.split(",") if w.strip() and w.strip() != "none"]
    if workloads:
        del p
        line["grouped"] = run_grouped(workloads, args, world, local, flush, peaks, peak_src, num_sms)
    latency = args.latency
    if latency == "auto":
        latency = ",".join(str(w) for w in LATENCY_WORKLOADS) if args.workload == 2 and world == 1 else ""
    small = [int(w) for w in latency.split(",") if w.strip() and w.strip() != "none"]
    if small:
        # the small dense call: one launch (latency-bound; two CUDA events around one trivial kernel already
        # measure about 6 us on this protocol)
        line["latency"] = run_grouped(small, args, world, local, flush, peaks, peak_src, num_sms)
    dg.set_fp32_scale_promotion(False)
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args) if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if args.impl == "ours" and world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
