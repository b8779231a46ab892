"""Benchmark of the B200 exact attention forward (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--pass fwd|bwd|fp8|decode|seqpar]
                    [--no-cpu-baseline]

A step is one attention forward pass over the whole workload (default: the
non-causal B=1, H=32, N=16384, d=128 case the throughput target is set on),
i.e. one launch of the sm_100a kernel through the C ABI.  Inputs are seeded
synthetic bf16 tensors (``exact_io_aware_73_b200.workloads``), resident in
HBM before timing starts.  Metric: TFLOP/s with FLOPs = 4 B H N^2 d (halved
when causal), the convention of the two attention GEMMs.

Multi-GPU (torchrun, one rank per GPU): every rank runs the full workload
on its own GPU with its own seed -- independent problems, no collective on
the data path (weak scaling); value = all ranks' FLOPs / max-over-ranks time.

``--impl reference`` times the fp64 CPU oracle (the reference arm of this
repository: the pages ship no runnable code) on a bounded sample of rows of
the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_io_aware_73_b200 import replicas as R  # noqa: E402
from exact_io_aware_73_b200 import workloads as W  # noqa: E402

METRIC = "attention fwd TFLOP/s (bf16, causal/non-causal) and % of B200 dense BF16 peak"
METRIC_BWD = "attention bwd TFLOP/s (bf16; 2.5 x forward FLOPs)"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0}
KERNEL_NAME = "attn_fwd_sm100_kernel"
CSRC = os.path.join(ROOT, "exact_io_aware_73_b200", "csrc")


KERNEL_SOURCES = ("attn_fwd_kernel.cuh", "ptx_sm100.cuh")
DECODE_SOURCES = ("attn_decode_kernel.cuh", "attn_fwd_kernel.cuh", "ptx_sm100.cuh")
DECODE_MMA_SOURCES = ("attn_decode_mma_kernel.cuh", "attn_fwd_kernel.cuh", "ptx_sm100.cuh")
BWD_SOURCES = ("attn_bwd_kernel.cuh", "attn_fwd_kernel.cuh", "ptx_sm100.cuh")


def cpu_model() -> str:
    """Model name of the host CPU (first entry of /proc/cpuinfo), recorded
    beside the core count of every CPU baseline."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def pages_context(w) -> dict:
    """The pages' own figures for this path, quoted beside the result for
    context.  They are not targets: none was measured on a B200."""
    n_scores = w.B * w.H * w.N * w.N
    return {
        "note": "figures printed on the pages, for context only (not targets)",
        "hopper_fa2_vs_ampere_fa2": (
            "+20-50% FLOPs/s for the CUTLASS FlashAttention-2 forward on one "
            "H100 PCIe over the Ampere-tuned kernel (briefgpt.xyz keyword page "
            "'attention algorithm', abstract)"),
        "standard_attention_scores_fp16_gb_printed": 12.9,
        "standard_attention_scores_fp16_gb_computed": round(
            23400 * 23400 * 12 * 2 / 1e9, 2),
        "standard_attention_scores_source": (
            "23,400 one-second steps x 12 heads, fp16 S, under standard "
            "attention (marketmaker.cc post, introduction)"),
        "this_workload_scores_fp16_gb": round(n_scores * 2 / 1e9, 3),
    }


def _code_only(text: str) -> str:
    """C++ source without comments and with whitespace runs collapsed, so
    that editing a comment does not change the hash of the code."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"' or c == "'":  # string or character literal: copied as is
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash(sources=KERNEL_SOURCES) -> str:
    """Hash of the device code (comments and whitespace ignored); a committed
    traffic figure is only used while it matches (the counters describe that
    exact kernel)."""
    h = hashlib.sha256()
    for f in sources:
        with open(os.path.join(CSRC, f), encoding="utf-8") as fh:
            h.update(f.encode() + b"\0" + _code_only(fh.read()).encode())
    return h.hexdigest()[:16]


# The exponential roof: the softmax evaluates one exp2 per visible score, B H
# N^2 of them (halved under the causal mask, the FLOP convention's count), on
# the MUFU unit at 16 per clock per SM.  The kernel evaluates a fixed share of
# them (pairs out of every 8, per head dimension, read from its source) on
# the FMA pipe instead.
MUFU_EX2_PER_CLK_PER_SM = 16


def fma_pipe_pairs_per8(d: int) -> int:
    """Pairs of exponentials out of 8 that the forward kernel evaluates on
    the FMA pipe at head dimension d (its ATTN_EXP2_EMU_PER8_D<d> default)."""
    with open(os.path.join(CSRC, "attn_fwd_kernel.cuh"), encoding="utf-8") as fh:
        src = fh.read()
    m = re.search(r"#define ATTN_EXP2_EMU_PER8_D%d (\d+)" % d, src)
    if m is None:
        raise RuntimeError(f"no exponential split for d = {d} in the kernel source")
    return int(m.group(1))
DEFAULT_SM_MHZ = 1965.0


def exp_roof(flops: float, d: int, ms_per_step: float, sm_count: int,
             sm_mhz) -> dict:
    """The forward's second roof beside the tensor cores: algorithmic exp2
    per launch (flops / (4 d)) over the launch time, against the MUFU rate
    of all SMs at the SM clock sampled during the timed region (the maximum
    clock when no sample exists)."""
    mhz = float(sm_mhz) if sm_mhz else DEFAULT_SM_MHZ
    count = flops / (4.0 * d)
    achieved = count / (ms_per_step * 1e-3) / 1e9
    peak = MUFU_EX2_PER_CLK_PER_SM * sm_count * mhz * 1e6 / 1e9
    return {"unit": "Gexp2/s", "achieved": achieved, "peak": peak,
            "frac": achieved / peak, "exp2_per_launch": count,
            "peak_basis": (f"{MUFU_EX2_PER_CLK_PER_SM} ex2 per clock per SM x "
                           f"{sm_count} SMs x {mhz:.0f} MHz (median SM clock in "
                           "the timed region)"),
            "mufu_share": 1.0 - fma_pipe_pairs_per8(d) / 8.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(workload: str, prefix: str = "traffic_", sources=KERNEL_SOURCES):
    """DRAM bytes per launch from a committed ncu capture of this workload,
    or None when there is none or the kernel changed since it was taken."""
    path = os.path.join(ROOT, "profiles", f"{prefix}{workload}.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("kernel_source_hash") != kernel_source_hash(sources):
        return None
    return t.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and throttle reasons sampled every 10 ms through NVML
    (read-only queries; nvidia-smi is the fallback), each sample with its
    host time.  begin() / end() mark the timed region; the record keeps the
    samples inside it, or, when the region is shorter than the sampling
    needs, the last sample before it and the first after it."""
    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40,
               "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self._nvml = None
        self.t_begin = None
        self.t_end = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(
                h, pynvml.NVML_CLOCK_SM)
            self._nvml = (pynvml, h)
        except Exception:  # no NVML: fall back to one nvidia-smi query
            self._nvml = None
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()

    def _query(self):
        if self._nvml is not None:
            pynvml, h = self._nvml
            mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
            try:
                mask = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
            except AttributeError:
                mask = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
            return float(mhz), int(mask)
        out = subprocess.run(
            ["nvidia-smi", "-i", str(self.gpu),
             "--query-gpu=clocks.sm,clocks.max.sm,clocks_event_reasons.active",
             "--format=csv,noheader,nounits"], capture_output=True, text=True,
            timeout=10).stdout.strip().split(",")
        self.max_mhz = float(out[1])
        return float(out[0]), int(out[2].strip(), 16)

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz, mask = self._query()
                self.samples.append((time.monotonic(), mhz, mask))
            except Exception:
                return
            self._stop.wait(0.01 if self._nvml is not None else 0.2)

    def begin(self):
        self.t_begin = time.monotonic()

    def end(self):
        self.t_end = time.monotonic()

    def stop(self):
        if self.t_end is None:
            self.end()
        if self.t_begin is None:  # started right before the region
            self.t_begin = self.samples[0][0] if self.samples else self.t_end
        # keep sampling until one sample lies after the region
        for _ in range(50):
            if self.samples and self.samples[-1][0] >= self.t_end:
                break
            time.sleep(0.01)
        self._stop.set()
        if self._t:
            self._t.join(timeout=5)
        if not self.samples:
            return None
        inside = [x for x in self.samples if self.t_begin <= x[0] <= self.t_end]
        where = "inside the timed region"
        if len(inside) < 2:
            before = [x for x in self.samples if x[0] < self.t_begin][-1:]
            after = [x for x in self.samples if x[0] > self.t_end][:1]
            inside = inside + before + after
            where = "the region's own samples plus the nearest one on each side"
        reasons = sorted(n for n, bit in self.REASONS.items()
                         if any(m & bit for _, _, m in inside))
        return {"sm_mhz": statistics.median(c for _, c, _ in inside),
                "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(inside), "window": where,
                "region_ms": round((self.t_end - self.t_begin) * 1e3, 1),
                "source": "nvml" if self._nvml is not None else "nvidia-smi"}


def cpu_baseline(w, qkv, budget_s: float, seed: int = 11):
    """The fp64 oracle (as it stands) on sampled rows of the workload, all
    host cores; returns the baseline object for the JSON line."""
    import numpy as np
    import oracle
    q, k, v = qkv
    bits = [oracle.bf16_bits(t) for t in (q, k, v)]
    threads = len(os.sched_getaffinity(0))
    rng = np.random.default_rng(seed)
    total_rows = w.B * w.H * w.N

    def row_flops(rows):
        i = rows % w.N
        keys = (i + 1) if w.causal else np.full_like(i, w.N)
        return float(np.sum(4.0 * keys * w.d))

    # calibrate on a small batch, then run a batch sized to the budget
    done_rows, done_flops, elapsed = 0, 0.0, 0.0
    batch = max(threads, 8)
    while elapsed < budget_s:
        rows = rng.integers(0, total_rows, size=batch)
        t0 = time.perf_counter()
        oracle.attention_rows_bf16(*bits, w.causal, w.scale, rows, threads)
        dt = time.perf_counter() - t0
        elapsed += dt
        done_rows += batch
        done_flops += row_flops(rows)
        rate = batch / max(dt, 1e-6)
        batch = int(min(max(threads, rate * (budget_s - elapsed) * 0.9),
                        total_rows))
        if budget_s - elapsed < 0.5:
            break
    return {"value": done_flops / elapsed / 1e12, "unit": "TFLOP/s",
            "cores": threads, "cpu_model": cpu_model(), "kind": "oracle",
            "sample": f"{done_rows} random query rows of {w.name} "
                      f"({done_rows / total_rows:.2e} of the workload), fp64 "
                      f"two-pass oracle, {elapsed:.1f} s"}


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    qkv = W.make_qkv(w)
    per_step = max(0.2, min(args.cpu_budget_s, 20.0,
                            150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(w, qkv, per_step / 4)
    vals = []
    t0 = time.perf_counter()
    for s in range(args.steps):
        vals.append(cpu_baseline(w, qkv, per_step, seed=100 + s))
    wall = time.perf_counter() - t0
    value = statistics.mean(v["value"] for v in vals)
    cb = dict(vals[-1])
    cb["value"] = value
    cb["sample"] = (f"each step: {per_step:.0f} s of random query rows of "
                    f"{w.name}; " + vals[-1]["sample"])
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * wall / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "causal": w.causal, "parallelism": "host cores (OpenMP)"},
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline_bwd(w, budget_s: float):
    """fp64 backward oracle on a bounded slice of the workload: the first
    2048 positions of up to (host cores) heads, one head per thread."""
    import numpy as np
    import oracle
    threads = len(os.sched_getaffinity(0))
    H = max(1, min(w.H * w.B, threads))
    n = min(w.N, 2048)
    sub = W.shape_case(1, H, n, w.d, w.causal, seed=w.seed)
    q, k, v = (oracle.bf16_bits_to_f64(oracle.bf16_bits(t)) for t in W.make_qkv(sub))
    do = np.random.default_rng(5).standard_normal(q.shape)
    t0 = time.perf_counter()
    oracle.attention_backward(q, k, v, do, w.causal, w.scale, threads)
    dt = time.perf_counter() - t0
    flops = 2.5 * sub.flops()
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": threads,
            "cpu_model": cpu_model(),
            "kind": "oracle",
            "sample": f"fp64 backward of {H} heads x N={n}, d={w.d} "
                      f"({'causal' if w.causal else 'non-causal'}), {dt:.1f} s"}


def run_backward(args, w):
    """Time attn_bwd (prep + dQ + dK/dV kernels) on the workload; one GPU."""
    import torch
    from exact_io_aware_73_b200 import attn
    world, rank, local = R.env_ranks()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    R.init("nccl", world, device=dev)
    q, k, v = (t.to(dev) for t in W.make_qkv(w, seed=R.rank_seed(w.seed, rank)))
    g = torch.Generator().manual_seed(R.rank_seed(w.seed, rank) + 3)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16).to(dev)
    o, lse = attn.attn_fwd(q, k, v, causal=w.causal, scale=w.scale)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(attn.bwd_workspace_bytes(w.B, w.H, w.N), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    in_bytes = 6 * q.numel() * 2
    flush = None if in_bytes > L2_BYTES else torch.empty(
        2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def step():
        rc = attn.attn_bwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                               o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                               dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                               ws.data_ptr(), ws.numel(), w.B, w.H, w.N, w.d,
                               w.causal, w.scale, sh)
        if rc != 0:
            raise attn.AttnError(rc, "attn_bwd")

    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        step()
    if attn.status() != 0:
        raise RuntimeError("device status after warm-up")
    R.barrier(world)
    torch.cuda.synchronize(dev)
    clocks.begin()
    evs = []
    for _ in range(args.steps):
        if flush is not None:
            flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        evs.append((a, b))
    R.barrier(world)
    torch.cuda.synchronize(dev)
    clocks.end()
    clk = clocks.stop()
    if attn.status() != 0:
        raise RuntimeError("device status after the timed region")
    ms = R.max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, dev)
    ms_per_step = ms / args.steps
    flops = 2.5 * w.flops()
    value = R.job_throughput(flops, world, ms_per_step * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    achieved = flops / (ms_per_step * 1e-3) / 1e12
    cb = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cb = cpu_baseline_bwd(w, args.cpu_budget_s)
    if rank == 0:
        print(json.dumps({
            "metric": METRIC_BWD, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Gaussian/uniform bf16 inputs, N(0,1) dO)",
            "config": {"workload": w.name, "pass": "bwd", "B": w.B, "H": w.H,
                       "N": w.N, "d": w.d, "causal": w.causal,
                       "l2": ("inputs larger than L2" if flush is None else
                              "L2 flushed between steps (outside the events)"),
                       "parallelism": f"{world} independent replicas"},
            "roofline": {"bound": "tensor", "achieved": achieved,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"],
                         "peak_source": f"{peak_src} bf16 burst (cuBLAS)",
                         "traffic": load_traffic(w.name, "traffic_bwd_", BWD_SOURCES),
                         "note": "FLOPs = 2.5 x forward (5 GEMMs); the kernels "
                                 "run 7 (S and dP are recomputed in both the "
                                 "dQ and the dK/dV kernel); traffic is the "
                                 "dK/dV kernel's (the larger share), per launch"},
            "cpu_baseline": cb, "e2e": None,
            "gpu_launches": 3 * args.steps, "clocks": clk}), flush=True)
    R.finish(world)
    return 0


METRIC_FP8 = ("attention fwd TFLOP/s, FP8 (E4M3) operands with incoherent "
              "processing (rotation + block quantization inside the step)")
FP8_SIGN_SEED = 77


def cpu_baseline_fp8(w, qkv, signs, budget_s: float, seed: int = 13):
    """The FP8 oracle (as it stands) on head (0, 0) of the workload: its Q,
    K, V quantized (time amortised over the rows timed), then random query
    rows through the blocked E4M3 softmax, all host cores."""
    import numpy as np
    import oracle
    threads = len(os.sched_getaffinity(0))
    bits = [oracle.bf16_bits(t[:1, :1].contiguous()) for t in qkv]
    t0 = time.perf_counter()
    z = oracle.quantize_qkv_fp8(*bits, True, np.asarray(signs, dtype=np.int8))
    t_quant = time.perf_counter() - t0
    scale_qk = float(np.float32(w.scale)) * z["gain"]
    rng = np.random.default_rng(seed)
    rows_done, flops, elapsed = 0, 0.0, 0.0
    batch = max(threads, 8)
    while elapsed < budget_s:
        rows = rng.integers(0, w.N, size=batch)
        t1 = time.perf_counter()
        oracle.attention_fp8_rows(z["q8"], z["qs"], z["k8"], z["ks"], z["v8"],
                                  z["vs"], w.causal, scale_qk, rows,
                                  threads=threads, tau=oracle.FP8_KERNEL_TAU)
        dt = time.perf_counter() - t1
        elapsed += dt
        rows_done += batch
        keys = (rows + 1) if w.causal else np.full_like(rows, w.N)
        flops += float(np.sum(4.0 * keys * w.d))
        rate = batch / max(dt, 1e-6)
        batch = int(min(max(threads, rate * (budget_s - elapsed) * 0.9), w.N))
        if budget_s - elapsed < 0.5:
            break
    total = elapsed + t_quant * rows_done / w.N
    return {"value": flops / total / 1e12, "unit": "TFLOP/s", "cores": threads,
            "cpu_model": cpu_model(),
            "kind": "oracle",
            "sample": f"head (0,0) of {w.name}: quantized in {t_quant:.1f} s "
                      f"(amortised over the rows), {rows_done} random query "
                      f"rows through the FP8 oracle in {elapsed:.1f} s"}


def run_fp8(args, w):
    """Time the FP8 path: attn_fwd_fp8 = quantize Q, K (rotated, per tile)
    and V (per head: two launches), then the E4M3 attention kernel."""
    import torch
    from exact_io_aware_73_b200 import attn
    if w.d != 128:
        raise SystemExit("the FP8 path exists for d = 128 only")
    world, rank, local = R.env_ranks()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    R.init("nccl", world, device=dev)
    qkv_host = W.make_qkv(w, seed=R.rank_seed(w.seed, rank))
    q, k, v = (t.to(dev) for t in qkv_host)
    signs = W.make_signs(FP8_SIGN_SEED, w.d).tolist()
    lo, hi = attn.sign_mask(signs)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    ws = torch.empty(attn.fp8_workspace_bytes(w.B, w.H, w.N, w.d),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    in_bytes = 3 * q.numel() * 2
    flush = None if in_bytes > L2_BYTES else torch.empty(
        2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def step(qq=q, kk=k, vv=v, oo=o, ll=lse):
        rc = attn.attn_fwd_fp8_raw(qq.data_ptr(), kk.data_ptr(), vv.data_ptr(),
                                   oo.data_ptr(), ll.data_ptr(), w.B, w.H, w.N,
                                   w.d, w.causal, w.scale, 1, lo, hi,
                                   ws.data_ptr(), ws.numel(), sh)
        if rc != 0:
            raise attn.AttnError(rc, "attn_fwd_fp8")

    # the attention kernel alone, on codes made by the same path
    q8, qs = attn.fp8_quantize(q, True, signs)
    k8, ks = attn.fp8_quantize(k, True, signs)
    v8, vs = attn.fp8_quantize(v, False, per_head=True)
    fp8_fns = attn._fp8_fns()

    def kernel_only():
        rc = fp8_fns.attn_fwd_fp8_quantized(
            q8.data_ptr(), qs.data_ptr(), k8.data_ptr(), ks.data_ptr(),
            v8.data_ptr(), vs.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B,
            w.H, w.N, w.d, int(w.causal), float(w.scale / w.d), sh)
        if rc != 0:
            raise attn.AttnError(rc, "attn_fwd_fp8_quantized")

    def timed(fn, steps):
        evs = []
        for _ in range(steps):
            if flush is not None:
                flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            evs.append((a, b))
        R.barrier(world)
        torch.cuda.synchronize(dev)
        return sum(a.elapsed_time(b) for a, b in evs)

    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        step()
        kernel_only()
    if attn.status() != 0:
        raise RuntimeError("device status after warm-up")
    R.barrier(world)
    torch.cuda.synchronize(dev)
    clocks.begin()
    step_ms = timed(step, args.steps)
    kern_ms = timed(kernel_only, args.steps)
    clocks.end()
    clk = clocks.stop()
    if attn.status() != 0:
        raise RuntimeError("device status after the timed region")
    ms_per_step = R.max_over_ranks(step_ms, world, dev) / args.steps
    kern_ms_per = R.max_over_ranks(kern_ms, world, dev) / args.steps
    flops = w.flops()
    value = R.job_throughput(flops, world, ms_per_step * 1e-3) / 1e12

    # end to end through the host-buffer entry attn_fwd_fp8_host: pinned
    # host Q, K, V copied in, rotated, quantized and attended, O and lse
    # copied out, every step (the copies overlap the computation by chunks)
    qh, kh, vh = (x.pin_memory() for x in qkv_host)
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()
    hws = torch.empty(attn.fp8_host_workspace_bytes(w.B, w.H, w.N, w.d),
                      dtype=torch.uint8, device=dev)

    def e2e_step():
        attn.attn_fwd_fp8_host(qh, kh, vh, oh, lh, w.causal, w.scale, hws,
                               signs=signs, stream=stream)

    e2e_steps = max(3, min(args.steps, 10))
    for _ in range(2):
        e2e_step()
    R.barrier(world)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    R.barrier(world)
    torch.cuda.synchronize(dev)
    if attn.status() != 0:
        raise RuntimeError("device status after the e2e region")
    e2e_ms = R.max_over_ranks(e0.elapsed_time(e1), world, dev) / e2e_steps
    e2e_value = R.job_throughput(flops, world, e2e_ms * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    peak = 2.0 * peaks["bf16_tflops"]
    achieved = flops / (kern_ms_per * 1e-3) / 1e12
    cb = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cb = cpu_baseline_fp8(w, qkv_host, signs, args.cpu_budget_s)
    if rank == 0:
        print(json.dumps({
            "metric": METRIC_FP8, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
            "data": "synthetic (seeded Gaussian bf16 inputs; seeded rotation signs)",
            "config": {"workload": w.name, "pass": "fp8", "B": w.B, "H": w.H,
                       "N": w.N, "d": w.d, "causal": w.causal,
                       "l2": ("inputs larger than L2" if flush is None else
                              "L2 flushed between steps (outside the events)"),
                       "parallelism": f"{world} independent replicas"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_source": f"{peak_src} bf16 burst (cuBLAS) x 2, "
                                        "the nominal E4M3 / bf16 ratio",
                         "traffic": load_traffic(w.name, "traffic_fp8_"),
                         "kernel": "attn_fwd_sm100_kernel<128,*,FP8>",
                         "kernel_ms": kern_ms_per,
                         "quantize_ms": ms_per_step - kern_ms_per},
            "cpu_baseline": cb,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": 3 * qh.numel() * 2,
                    "d2h_bytes_per_step": oh.numel() * 2 + lh.numel() * 4,
                    "ms_per_step": e2e_ms, "steps": e2e_steps,
                    "api": "attn_fwd_fp8_host (pinned host buffers)"},
            "gpu_launches": 5 * args.steps, "clocks": clk}), flush=True)
    R.finish(world)
    return 0


METRIC_DECODE = ("attention decode: K/V bytes streamed per second (GB/s; "
                 "split-KV, HBM-bound)")


def cpu_baseline_decode(w, qkv, budget_s: float):
    """The fp64 oracle on query rows of the decode workload (every row of as
    many heads as the budget allows), all host cores; GB/s of K/V covered."""
    import numpy as np
    import oracle
    q, k, v = qkv
    bits = [oracle.bf16_bits(t) for t in (q, k, v)]
    threads = len(os.sched_getaffinity(0))
    rows_total = w.B * w.H * w.Nq
    done, elapsed, batch = 0, 0.0, max(1, min(threads, rows_total))
    while elapsed < budget_s and done < rows_total:
        rows = np.arange(done, min(rows_total, done + batch))
        t0 = time.perf_counter()
        oracle.attention_decode_rows_bf16(*bits, w.causal, w.scale, rows, threads)
        dt = time.perf_counter() - t0
        elapsed += dt
        done += rows.size
        if budget_s - elapsed < 0.5:
            break
    heads = done / w.Nq
    kv = heads * 2 * w.Nk * w.d * 2
    return {"value": kv / elapsed / 1e9, "unit": "GB/s", "cores": threads,
            "cpu_model": cpu_model(),
            "kind": "oracle",
            "sample": f"{done} of {rows_total} query rows of {w.name} "
                      f"(fp64 oracle, {elapsed:.1f} s)"}


def run_decode(args):
    """Time attn_decode on a decode workload (Nq new queries against an
    Nk-long key/value sequence per head); one launch per step."""
    import torch
    from exact_io_aware_73_b200 import attn
    name = args.workload if args.workload in W.DECODE_WORKLOADS else W.DECODE_HEADLINE
    w = W.DECODE_WORKLOADS[name]
    world, rank, local = R.env_ranks()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    R.init("nccl", world, device=dev)
    qkv_host = W.make_decode_qkv(w, seed=R.rank_seed(w.seed, rank))
    q, k, v = (t.to(dev) for t in qkv_host)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    ws = torch.empty(attn.decode_workspace_bytes(w.B, w.H, w.Nq, w.Nk, w.d),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    flush = None if w.kv_bytes() > L2_BYTES else torch.empty(
        2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def step():
        rc = attn.attn_decode_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                  o.data_ptr(), lse.data_ptr(), w.B, w.H, w.Nq,
                                  w.Nk, w.d, w.causal, w.scale, ws.data_ptr(),
                                  ws.numel(), sh)
        if rc != 0:
            raise attn.AttnError(rc, "attn_decode")

    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        step()
    if attn.status() != 0:
        raise RuntimeError("device status after warm-up")
    R.barrier(world)
    torch.cuda.synchronize(dev)
    clocks.begin()
    evs = []
    for _ in range(args.steps):
        if flush is not None:
            flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        evs.append((a, b))
    R.barrier(world)
    torch.cuda.synchronize(dev)
    clocks.end()
    clk = clocks.stop()
    if attn.status() != 0:
        raise RuntimeError("device status after the timed region")
    ms = R.max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, dev)
    ms_per_step = ms / args.steps
    kv = w.kv_bytes()
    value = R.job_throughput(kv, world, ms_per_step * 1e-3) / 1e9
    # end to end: the step's new queries copied in from pinned host memory,
    # O and lse copied out; the key/value cache stays resident on the device
    qh = qkv_host[0].pin_memory()
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32).pin_memory()

    def e2e_step():
        q.copy_(qh, non_blocking=True)
        step()
        oh.copy_(o, non_blocking=True)
        lh.copy_(lse, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 20))
    for _ in range(2):
        e2e_step()
    R.barrier(world)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    R.barrier(world)
    torch.cuda.synchronize(dev)
    if attn.status() != 0:
        raise RuntimeError("device status after the e2e region")
    e2e_ms = R.max_over_ranks(e0.elapsed_time(e1), world, dev) / e2e_steps
    peaks, peak_src = load_peaks()
    achieved = kv / (ms_per_step * 1e-3) / 1e9
    algo_bytes = kv + 2 * q.numel() * 2 + lse.numel() * 4
    # the library's choice: one tensor-core launch for all queries, or one
    # CUDA-core launch per group of 4
    mma = attn.decode_kernel_for(w.Nq, w.d) == attn.DECODE_TENSOR_CORES
    launches = 1 if mma else -(-w.Nq // attn.DECODE_GROUP_Q)
    kernel = f"attn_decode_mma_kernel<{w.d}>" if mma else f"attn_decode_kernel<{w.d}>"
    cb = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cb = cpu_baseline_decode(w, qkv_host, args.cpu_budget_s)
    if rank == 0:
        print(json.dumps({
            "metric": METRIC_DECODE, "value": value, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Gaussian bf16 inputs)",
            "config": {"workload": w.name, "pass": "decode", "B": w.B, "H": w.H,
                       "Nq": w.Nq, "Nk": w.Nk, "d": w.d, "causal": w.causal,
                       "l2": ("K/V larger than L2" if flush is None else
                              "L2 flushed between steps (outside the events)"),
                       "parallelism": f"{world} independent replicas"},
            "tflops": w.flops() / (ms_per_step * 1e-3) / 1e12,
            "roofline": {"bound": "hbm", "achieved": achieved,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"],
                         "peak_source": f"{peak_src} HBM copy bandwidth",
                         "traffic": load_traffic(w.name, "traffic_decode_",
                                                 DECODE_MMA_SOURCES if mma
                                                 else DECODE_SOURCES),
                         "algorithmic_bytes_per_launch": algo_bytes,
                         "kernel": kernel},
            "cpu_baseline": cb,
            "e2e": {"value": kv / (e2e_ms * 1e-3) / 1e9 * world, "unit": "GB/s",
                    "h2d_bytes_per_step": qh.numel() * 2,
                    "d2h_bytes_per_step": oh.numel() * 2 + lh.numel() * 4,
                    "ms_per_step": e2e_ms, "steps": e2e_steps,
                    "api": "attn.attn_decode with the new queries copied in and "
                           "O / lse copied out; the K/V cache stays on the device"},
            "gpu_launches": launches * args.steps, "clocks": clk}), flush=True)
    R.finish(world)
    return 0


METRIC_SEQPAR = ("attention fwd TFLOP/s, one sequence sharded over ranks "
                 "(ring of K/V shards + exact lse merge)")


def run_seqpar(args, w):
    """Sequence-sharded forward: the workload's sequence split into P
    contiguous shards.  Under torchrun each rank holds one shard and the K/V
    shards go around the ring (NCCL point-to-point); with one process and
    --shards P > 1 the P ranks run emulated on the one GPU, one after
    another (the same blocks and merges, no exchange)."""
    import torch
    from exact_io_aware_73_b200 import attn, seqpar
    world, rank, local = R.env_ranks()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    R.init("nccl", world, device=dev)
    shards = world if world > 1 else max(1, args.shards)
    if w.N % shards:
        raise SystemExit(f"N = {w.N} is not a multiple of {shards} shards")
    q, k, v = (t.to(dev) for t in W.make_qkv(w))
    n = w.N // shards
    if world > 1:
        sl = slice(rank * n, (rank + 1) * n)
        q, k, v = (t[:, :, sl].contiguous() for t in (q, k, v))

        def step():
            return seqpar.ring_attention(q, k, v, w.causal, w.scale)
    else:
        qs, ks, vs = (seqpar.shard(t, shards) for t in (q, k, v))
        del q, k, v

        def step():
            return seqpar.ring_attention_emulated(qs, ks, vs, w.causal, w.scale)
    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        step()
    if attn.status() != 0:
        raise RuntimeError("device status after warm-up")
    R.barrier(world)
    torch.cuda.synchronize(dev)
    clocks.begin()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    R.barrier(world)
    torch.cuda.synchronize(dev)
    clocks.end()
    clk = clocks.stop()
    if attn.status() != 0:
        raise RuntimeError("device status after the timed region")
    ms_per_step = R.max_over_ranks(a.elapsed_time(b), world, dev) / args.steps
    flops = w.flops()
    value = flops / (ms_per_step * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    cb = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cb = cpu_baseline(w, W.make_qkv(w), args.cpu_budget_s)
        cb["sample"] = ("sharding does not change the result: the fp64 oracle "
                        "on " + cb["sample"])
    if rank == 0:
        print(json.dumps({
            "metric": METRIC_SEQPAR, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Gaussian bf16 inputs)",
            "config": {"workload": w.name, "pass": "seqpar", "shards": shards,
                       "emulated": world == 1 and shards > 1, "B": w.B, "H": w.H,
                       "N": w.N, "d": w.d, "causal": w.causal,
                       "l2": "inputs larger than L2" if 3 * w.B * w.H * w.N * w.d * 2 > L2_BYTES
                             else "inputs may stay in L2",
                       "parallelism": (f"sequence sharded over {world} ranks" if world > 1
                                       else f"{shards} shards emulated on one GPU")},
            "roofline": {"bound": "tensor", "achieved": value,
                         "peak": peaks["bf16_tflops"] * world, "unit": "TFLOP/s",
                         "frac": value / (peaks["bf16_tflops"] * world),
                         "peak_source": f"{peak_src} bf16 burst (cuBLAS) x ranks",
                         "traffic": None},
            "cpu_baseline": cb, "e2e": None,
            "gpu_launches": None, "clocks": clk}), flush=True)
    R.finish(world)
    return 0


METRIC_SPARSE = "block-sparse attention fwd TFLOP/s (bf16; FLOPs of the computed blocks)"


def cpu_baseline_sparse(w, qkv, mask, budget_s: float, seed: int = 17):
    """The block-sparse fp64 oracle on random rows of the workload, all host
    cores; TFLOP/s over the FLOPs those rows' kept keys take."""
    import numpy as np
    import oracle
    bits = [oracle.bf16_bits(t) for t in qkv]
    m = mask.numpy()
    threads = len(os.sched_getaffinity(0))
    rng = np.random.default_rng(seed)
    T = (w.N + 127) // 128
    keep = m.reshape(-1, T, T)[0].astype(np.int64)

    def row_flops(rows):
        i = rows % w.N
        kept = np.zeros(len(rows))
        for a, r in enumerate(i):
            js = np.arange((r + 1) if w.causal else w.N)
            kept[a] = keep[r // 128][js // 128].sum()
        return float(np.sum(4.0 * kept * w.d))

    done, flops, elapsed, batch = 0, 0.0, 0.0, max(threads, 8)
    while elapsed < budget_s:
        rows = rng.integers(0, w.B * w.H * w.N, size=batch)
        t0 = time.perf_counter()
        oracle.attention_block_sparse_rows_bf16(*bits, w.causal, w.scale, m, rows,
                                                threads)
        dt = time.perf_counter() - t0
        elapsed += dt
        done += batch
        flops += row_flops(rows)
        batch = int(min(max(threads, batch / max(dt, 1e-6) * (budget_s - elapsed) * 0.9),
                        w.B * w.H * w.N))
        if budget_s - elapsed < 0.5:
            break
    return {"value": flops / elapsed / 1e12, "unit": "TFLOP/s", "cores": threads,
            "cpu_model": cpu_model(), "kind": "oracle",
            "sample": f"{done} random query rows of {w.name} with its block mask, "
                      f"fp64 block-sparse oracle, {elapsed:.1f} s"}


def run_sparse(args):
    """Block-sparse forward: the named workload's shape with its seeded block
    mask (a sliding window of key tiles plus random ones, one mask for every
    head).  A step is one attn_fwd_block_sparse launch; FLOPs count the
    computed blocks only."""
    import torch
    from exact_io_aware_73_b200 import attn
    name = args.workload if args.workload in W.SPARSE_WORKLOADS else \
        "sparse_long_b1h32n16384d128"
    w, density, local = W.SPARSE_WORKLOADS[name]
    world, rank, local_rank = R.env_ranks()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    R.init("nccl", world, device=dev)
    qkv_host = W.make_qkv(w, seed=R.rank_seed(w.seed, rank))
    mask = W.block_mask_for(name)
    q, k, v = (t.to(dev) for t in qkv_host)
    md = mask.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    flops = W.sparse_flops(w, mask)
    kept = float(mask.float().mean())
    in_bytes = 3 * q.numel() * 2
    flush = None if in_bytes > L2_BYTES else torch.empty(2 * L2_BYTES, dtype=torch.uint8,
                                                         device=dev)

    def step():
        rc = attn.attn_fwd_block_sparse_raw(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
            w.B, w.H, w.N, w.d, w.causal, w.scale, md.data_ptr(), False, sh)
        if rc != 0:
            raise attn.AttnError(rc, "attn_fwd_block_sparse")

    clocks = ClockSampler(local_rank)
    clocks.start()
    for _ in range(args.warmup):
        step()
    if attn.status() != 0:
        raise RuntimeError("device status after warm-up")
    R.barrier(world)
    torch.cuda.synchronize(dev)
    clocks.begin()
    evs = []
    for _ in range(args.steps):
        if flush is not None:
            flush.zero_()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        evs.append((a, b))
    R.barrier(world)
    torch.cuda.synchronize(dev)
    clocks.end()
    clk = clocks.stop()
    if attn.status() != 0:
        raise RuntimeError("device status after the timed region")
    ms = R.max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world, dev)
    ms_per_step = ms / args.steps
    value = world * flops / (ms_per_step * 1e-3) / 1e12
    # end to end: inputs from pinned host memory, the call, outputs back
    qh, kh, vh = (t.pin_memory() for t in qkv_host)
    mh = mask.pin_memory()
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()

    def e2e_step():
        for src, dst in ((qh, q), (kh, k), (vh, v), (mh, md)):
            dst.copy_(src, non_blocking=True)
        step()
        oh.copy_(o, non_blocking=True)
        lh.copy_(lse, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, min(args.steps, 10))
    e0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if attn.status() != 0:
        raise RuntimeError("device status after the e2e region")
    e2e_ms = R.max_over_ranks(e0.elapsed_time(e1), world, dev) / n_e2e
    peaks, peak_src = load_peaks()
    achieved = flops / (ms_per_step * 1e-3) / 1e12
    cb = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cb = cpu_baseline_sparse(w, qkv_host, mask, args.cpu_budget_s)
    if rank == 0:
        print(json.dumps({
            "metric": METRIC_SPARSE, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded Gaussian bf16 inputs, seeded block mask)",
            "config": {"workload": name, "pass": "sparse", "B": w.B, "H": w.H,
                       "N": w.N, "d": w.d, "causal": w.causal,
                       "blocks_kept": round(kept, 4), "window_tiles": local,
                       "random_density": density,
                       "l2": "inputs larger than L2" if flush is None else
                             "L2 flushed between steps (outside the events)",
                       "parallelism": f"{world} independent replicas"},
            "roofline": {"bound": "tensor", "achieved": achieved,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"],
                         "peak_source": f"{peak_src} bf16 burst (cuBLAS)",
                         "traffic": load_traffic(name),
                         "algorithmic_flops_per_launch": flops,
                         "kernel": KERNEL_NAME},
            "cpu_baseline": cb,
            "e2e": {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": in_bytes + mask.numel(),
                    "d2h_bytes_per_step": o.numel() * 2 + lse.numel() * 4,
                    "ms_per_step": e2e_ms, "steps": n_e2e,
                    "api": "attn_fwd_block_sparse with torch copies from pinned host memory"},
            "gpu_launches": args.steps, "clocks": clk}), flush=True)
    R.finish(world)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=W.HEADLINE,
                    choices=sorted(W.WORKLOADS) + sorted(W.DECODE_WORKLOADS) +
                    sorted(W.SPARSE_WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--pass", dest="pass_", default="fwd",
                    choices=["fwd", "bwd", "fp8", "decode", "seqpar", "sparse"],
                    help="fwd (default): the forward hot path; bwd: attn_bwd; "
                         "fp8: the FP8 forward with incoherent processing; "
                         "decode: split-KV decode (decode_* workloads); "
                         "seqpar: one sequence sharded over ranks; "
                         "sparse: block-sparse forward (sparse_* workloads)")
    ap.add_argument("--split", default="replicas", choices=["replicas", "heads"],
                    help="forward on N GPUs: replicas (default: every rank "
                         "its own seeded problem, weak scaling) or heads (the "
                         "B*H heads of one problem split into contiguous "
                         "ranges over the ranks, strong scaling)")
    ap.add_argument("--shards", type=int, default=1,
                    help="seqpar on one process: shards emulated on one GPU")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=15.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.pass_ == "decode":
        if args.impl == "reference":
            ap.error("the reference arm times the forward oracle")
        return run_decode(args)
    if args.pass_ == "sparse":
        if args.impl == "reference":
            ap.error("the reference arm times the forward oracle")
        return run_sparse(args)
    if args.workload not in W.WORKLOADS:
        ap.error(f"{args.workload} is a decode or block-sparse workload: use "
                 "--pass decode or --pass sparse")
    w = W.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.pass_ == "bwd":
        return run_backward(args, w)
    if args.pass_ == "fp8":
        return run_fp8(args, w)
    if args.pass_ == "seqpar":
        return run_seqpar(args, w)

    import torch
    from exact_io_aware_73_b200 import attn

    world, rank, local = R.env_ranks()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    R.init("nccl", world, device=dev)

    def barrier():
        R.barrier(world)

    # ---- inputs, resident in HBM before timing: a problem of its own per
    # rank (seeded per rank), or this rank's range of the heads of one problem
    heads = args.split == "heads"
    seed = w.seed if heads else R.rank_seed(w.seed, rank)
    qkv_host = W.make_qkv(w, seed=seed)
    Bs, Hs = w.B, w.H
    if heads:
        h0, nh = R.head_shard(w.B * w.H, world, rank)
        qkv_host = tuple(t.reshape(w.B * w.H, w.N, w.d)[h0:h0 + nh]
                         .reshape(1, nh, w.N, w.d).contiguous() for t in qkv_host)
        Bs, Hs = 1, nh
    q, k, v = (t.to(dev) for t in qkv_host)
    o = torch.empty_like(q)
    lse = torch.empty((Bs, Hs, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    in_bytes = 3 * q.numel() * 2
    flush = None if in_bytes > L2_BYTES else torch.empty(
        2 * L2_BYTES, dtype=torch.uint8, device=dev)

    def step():
        rc = attn.attn_fwd_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(),
                               o.data_ptr(), lse.data_ptr(), Bs, Hs, w.N,
                               w.d, w.causal, w.scale, sh)
        if rc != 0:
            raise attn.AttnError(rc, "attn_fwd")

    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        step()
    rc = attn.status()
    if rc != 0:
        raise attn.AttnError(rc, "warm-up")

    # ---- device-timed region
    barrier()
    torch.cuda.synchronize(dev)
    clocks.begin()
    if flush is None:
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        barrier()
        torch.cuda.synchronize(dev)
        kernel_ms = ev0.elapsed_time(ev1)
        l2_note = (f"inputs larger than L2 ({in_bytes / 2**20:.0f} MiB of Q/K/V "
                   f"vs 126 MiB); back-to-back launches")
    else:
        evs = [(torch.cuda.Event(enable_timing=True),
                torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            step()
            b.record(stream)
        barrier()
        torch.cuda.synchronize(dev)
        kernel_ms = sum(a.elapsed_time(b) for a, b in evs)
        l2_note = "L2 flushed between steps (252 MiB write outside the events)"
    clocks.end()
    clk = clocks.stop()
    rc = attn.status()
    if rc != 0:
        raise attn.AttnError(rc, "timed region")

    max_ms = R.max_over_ranks(kernel_ms, world, dev)
    ms_per_step = max_ms / args.steps
    # FLOPs of this rank's launch; the job's are every rank's (replicas) or
    # the one problem's (heads)
    flops = w.flops() * (Bs * Hs) / (w.B * w.H)
    job_flops = w.flops() if heads else world * w.flops()
    value = job_flops / (ms_per_step * 1e-3) / 1e12

    # ---- end to end through the host-buffer C entry point
    qh, kh, vh = (x.pin_memory() for x in qkv_host)
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((Bs, Hs, w.N), dtype=torch.float32).pin_memory()
    ws = torch.empty(attn.host_workspace_bytes(Bs, Hs, w.N, w.d),
                     dtype=torch.uint8, device=dev)
    del q, k, v, o, lse
    e2e_steps = max(3, min(args.steps, 10))
    for _ in range(2):
        attn.attn_fwd_host(qh, kh, vh, oh, lh, w.causal, w.scale, ws, stream=sh)
    barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        attn.attn_fwd_host(qh, kh, vh, oh, lh, w.causal, w.scale, ws, stream=sh)
    e1.record(stream)
    barrier()
    torch.cuda.synchronize(dev)
    rc = attn.status()
    if rc != 0:
        raise attn.AttnError(rc, "e2e region")
    e2e_ms = R.max_over_ranks(e0.elapsed_time(e1), world, dev) / e2e_steps
    e2e_value = job_flops / (e2e_ms * 1e-3) / 1e12
    h2d = 3 * qh.numel() * 2
    d2h = oh.numel() * 2 + lh.numel() * 4

    # ---- roofline of the one kernel (the whole step is one launch)
    peaks, peak_src = load_peaks()
    achieved = flops / (ms_per_step * 1e-3) / 1e12
    roofline = {
        "bound": "tensor", "achieved": achieved,
        "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
        "frac": achieved / peaks["bf16_tflops"],
        "peak_source": f"{peak_src} bf16 burst (cuBLAS)",
        "frac_of_sustained_peak": achieved / peaks["bf16_tflops_sustained"],
        "traffic": load_traffic(w.name),
        "algorithmic_flops_per_launch": flops,
        "kernel": KERNEL_NAME,
    }

    cb = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        cb = cpu_baseline(w, qkv_host, args.cpu_budget_s)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if heads else "weak", "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded Gaussian/uniform bf16 inputs)",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N,
                       "d": w.d, "causal": w.causal, "scale": w.scale,
                       "l2": l2_note,
                       "parallelism": (
                           f"the {w.B * w.H} heads of one problem split over "
                           f"{world} GPUs (contiguous ranges, no collective)"
                           if heads else f"{world} independent replicas (one "
                           "workload per GPU, no collective)")},
            "roofline": roofline,
            "exp_roof": exp_roof(flops, w.d, ms_per_step,
                                 torch.cuda.get_device_properties(dev).multi_processor_count,
                                 (clk or {}).get("sm_mhz")),
            "cpu_baseline": cb,
            "e2e": {"value": e2e_value, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "steps": e2e_steps,
                    "api": "attn_fwd_host (pinned host buffers)"},
            "context": pages_context(w),
            "gpu_launches": args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    R.finish(world)
    return 0


if __name__ == "__main__":
    sys.exit(main())
