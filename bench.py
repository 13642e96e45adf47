"""Benchmark of the exact attention forward (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--splits S|auto] [--skip-cpu-baseline]
                    [--skip-e2e]

A step is one forward (one fa_fwd launch) over the whole workload; the
default workload is the non-causal B=4, H=48, L=8192, D=128 fp16 forward.
The metric is forward TFLOPS with the pages' convention 4*B*H*L_q*L_k*D
(halved when causal).  Timing: W untimed warm-up steps, then K steps timed
with CUDA events on the launching stream, bracketed by a barrier and a
device synchronise; the slowest rank's time counts.  The inputs (1.2 GB) are
larger than the 126 MB L2, so no flush is needed between steps; a workload
whose inputs and outputs are smaller than twice the L2 gets 256 MiB written
between its steps (outside the steps' events, whose times are summed).
Clocks and throttle reasons are sampled through NVML every 10 ms during the
timed steps.  `roofline.traffic` is read from the machine-written summary
profiles/fa_fwd_kernel_roofline_b4h48l8192d128_dram.txt (an ncu capture of
the DRAM byte counters on this workload, ingested with --ingest-ncu) while
the kernel's code is unchanged since the capture.

N > 1 (torchrun, one process per GPU, NCCL for the barrier and the max):
every rank runs the same-sized problem on its own inputs (weak scaling; the
path has no exchange step), and the value is all ranks' FLOPs over the
slowest rank's time.

--pass bwd times fa_bwd (the backward, after one untimed forward for O and
lse): a step is its three launches (delta / lse prep, the gradient kernel,
the dQ conversion); the metric counts 2.5x the forward's FLOPs.

--fp8 times fa_fwd_fp8 on the workload's inputs converted to E4M3 (bf16
output); its roofline peak is the measured bf16 rate x 2 (the nominal
fp8 / bf16 ratio of the tensor cores).  With --splits it times
fa_fwd_fp8_splitkv (an fp8 key/value cache; HBM-bound decodes count the
inputs at one byte per element).

--sweep prints one line per named workload (tiny, GPT-2, memory-table,
the B4 H48 sequence sweep, the GQA window, the roofline point; the decoding
shapes through fa_fwd_splitkv): % of the tensor peak, of the exp bound and,
for the memory-bound ones, of HBM.  Not the driver's single-line run.

--splits S (or auto) times fa_fwd_splitkv instead: one split-KV launch plus
one merge launch per step, for the decoding workloads (a few query rows, a
long key/value cache), whose roofline is HBM bandwidth rather than the
tensor pipe.

--impl reference runs the fp64 CPU oracle (the only other implementation
this path has) on the host cores, over a bounded sample of query rows of the
same workload per step, and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from exact_attention_113_b200 import inputs as W  # noqa: E402

METRIC = "attention fwd TFLOPS (and % of B200 fp16 tensor peak) vs seq len"
METRIC_BWD = "attention bwd TFLOPS (five GEMMs: 2.5x the forward's FLOPs)"
UNIT = "TFLOPS"
BWD_FLOP_FACTOR = 2.5      # backward: S, dP, dV, dK, dQ = 5 GEMMs vs the forward's 2
# MUFU ex2 rate per SM and clock: 8 clk per warp instruction per sub-partition
# (measured with a one-CTA microbenchmark on this GPU), 4 sub-partitions
MUFU_EX2_PER_CLK_SM = 16.0
SM_COUNT = 148
DEFAULT_WORKLOAD = W.ROOFLINE.name
# DRAM traffic of the forward kernel on the default workload: written by
# `bench.py --ingest-ncu` from an ncu capture of that workload
TRAFFIC_SUMMARY = os.path.join(ROOT, "profiles", "fa_fwd_kernel_roofline_b4h48l8192d128_dram.txt")
TRAFFIC_METRICS = ("dram__bytes_read.sum", "dram__bytes_write.sum")
# the forward kernel's device code (the ncu summary is valid while it is
# unchanged; the host-side launch code lives in fa_api.cu)
KERNEL_SOURCES = [os.path.join(ROOT, "exact_attention_113_b200", "csrc", f)
                  for f in ("fa_fwd_kernel.cuh", "sm100.cuh")]
L2_BYTES = 126 * 1024 * 1024
L2_FLUSH_BELOW = 2 * L2_BYTES         # workloads smaller than this get an L2 flush
L2_FLUSH_BYTES = 256 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ FLOPs
def visible_pairs_per_head(w: W.Workload) -> int:
    """(query, key) pairs that pass the mask in one head."""
    wr = 0 if w.causal else w.window_right
    i = np.arange(w.L_q, dtype=np.int64)
    lo = np.zeros_like(i) if w.window_left < 0 else np.maximum(i - w.window_left, 0)
    hi = np.full_like(i, w.L_k - 1) if wr < 0 else np.minimum(i + wr, w.L_k - 1)
    return int(np.clip(hi - lo + 1, 0, None).sum())


def metric_flops(w: W.Workload) -> float:
    """The pages' convention: 4*B*H*L_q*L_k*D, halved when causal."""
    f = 4.0 * w.B * w.H * w.L_q * w.L_k * w.D
    return f / 2 if w.causal else f


def algorithmic_flops(w: W.Workload) -> float:
    """Two length-D dot products (4*D FLOP) per visible (query, key) pair."""
    return 4.0 * w.D * w.B * w.H * visible_pairs_per_head(w)


def row_flops(w: W.Workload, rows: np.ndarray) -> float:
    """Algorithmic FLOPs of the given flattened query rows."""
    i = rows % w.L_q
    wr = 0 if w.causal else w.window_right
    lo = np.zeros_like(i) if w.window_left < 0 else np.maximum(i - w.window_left, 0)
    hi = np.full_like(i, w.L_k - 1) if wr < 0 else np.minimum(i + wr, w.L_k - 1)
    return float(4.0 * w.D * np.clip(hi - lo + 1, 0, None).sum())


# ------------------------------------------------------------------ ranks
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest value of x over all ranks (identity for one rank)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def whole_job_value(flops_per_rank_step: float, world: int, steps: int,
                    max_seconds: float) -> float:
    """All ranks' FLOPs over the slowest rank's time, in TFLOPS."""
    return flops_per_rank_step * world * steps / max_seconds / 1e12


# ------------------------------------------------------------------ peaks
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def code_hash(texts) -> str:
    """sha256 (16 hex digits) of source texts with // comments, trailing
    blanks and empty lines removed: a comment edit keeps the hash, any code
    edit changes it."""
    h = hashlib.sha256()
    for text in texts:
        for line in text.splitlines():
            code = line.split("//", 1)[0].rstrip()
            if code:
                h.update(code.encode("utf-8") + b"\n")
    return h.hexdigest()[:16]


def kernel_source_hash() -> str:
    """code_hash of the forward kernel's device code (the committed ncu
    summary records the value its counters were taken on)."""
    texts = []
    for p in KERNEL_SOURCES:
        with open(p, encoding="utf-8") as f:
            texts.append(f.read())
    return code_hash(texts)


def profiled_traffic(path: str = TRAFFIC_SUMMARY):
    """DRAM bytes per launch from the machine-written traffic summary, if it
    was taken on the kernel sources as they are now (else None)."""
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"^kernel_source_hash:\s*([0-9a-f]+)", text, re.M)
    m_bytes = re.search(r"^dram_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
    if not m_hash or not m_bytes or m_hash.group(1) != kernel_source_hash():
        return None
    return float(m_bytes.group(1))


_UNITS = {"byte": 1.0, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "tbyte": 1e12,
          "kibyte": 1024.0, "mibyte": 1024.0 ** 2, "gibyte": 1024.0 ** 3}


def parse_ncu_metrics_csv(text: str, kernel_regex: str = "fa_fwd_kernel") -> dict:
    """{launch id: {"kernel": name, metric: bytes}} from `ncu --csv
    --metrics ...` output (one row per launch and metric)."""
    import csv
    import io
    lines = [ln for ln in text.splitlines() if ln.startswith('"')]
    rows = list(csv.reader(io.StringIO("\n".join(lines))))
    if not rows:
        return {}
    head = rows[0]
    col = {name: head.index(name) for name in ("ID", "Kernel Name", "Metric Name",
                                               "Metric Unit", "Metric Value")}
    out = {}
    for r in rows[1:]:
        if len(r) < len(head) or not re.search(kernel_regex, r[col["Kernel Name"]]):
            continue
        unit = r[col["Metric Unit"]].strip().lower()
        val = float(r[col["Metric Value"]].replace(",", "")) * _UNITS.get(unit, 1.0)
        d = out.setdefault(r[col["ID"]], {"kernel": r[col["Kernel Name"]]})
        d[r[col["Metric Name"]]] = val
    return out


def ingest_ncu(csv_path: str, command: str, w: W.Workload, out_path: str = TRAFFIC_SUMMARY):
    """Write the traffic summary that `roofline.traffic` reads from an ncu
    capture of `TRAFFIC_METRICS` on workload ``w``."""
    launches = parse_ncu_metrics_csv(open(csv_path, errors="replace").read())
    launches = {k: v for k, v in launches.items() if all(m in v for m in TRAFFIC_METRICS)}
    if not launches:
        raise SystemExit(f"no fa_fwd_kernel launch with {TRAFFIC_METRICS} in {csv_path}")
    rd = statistics.mean(v[TRAFFIC_METRICS[0]] for v in launches.values())
    wr = statistics.mean(v[TRAFFIC_METRICS[1]] for v in launches.values())
    kernels = sorted({v["kernel"] for v in launches.values()})
    alg = min_hbm_bytes(w)
    text = (f"# DRAM traffic of the forward kernel on the workload {w.name}\n"
            f"# (machine-written by: python bench.py --ingest-ncu <csv> --workload {w.name})\n"
            f"command: {command}\n"
            f"kernel: {'; '.join(kernels)}\n"
            f"kernel_source_hash: {kernel_source_hash()}\n"
            f"launches_captured: {len(launches)}\n"
            f"dram_bytes_read_per_launch: {rd:.6g}\n"
            f"dram_bytes_write_per_launch: {wr:.6g}\n"
            f"dram_bytes_per_launch: {rd + wr:.6g}\n"
            f"algorithmic_bytes_per_launch: {alg:.6g}\n"
            f"traffic_over_algorithmic: {(rd + wr) / alg:.4f}\n")
    with open(out_path, "w") as f:
        f.write(text)
    print(text, end="")


# ------------------------------------------------------------------ clocks
def physical_gpu_index(cuda_index: int) -> int:
    """nvidia-smi's index of torch's cuda:<cuda_index>."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").strip()
    if vis:
        ids = [t.strip() for t in vis.split(",") if t.strip()]
        if cuda_index < len(ids) and ids[cuda_index].isdigit():
            return int(ids[cuda_index])
    return cuda_index


class ClockSampler:
    """SM clock, power and throttle reasons sampled during the timed region.

    Reads NVML (read-only queries, every 10 ms from a thread), so that even a
    timed region of ~0.1 s gets several samples; falls back to `nvidia-smi
    -lms 200` without NVML.  ``summary()`` counts only samples taken between
    mark_start() and mark_end()."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: int, pci_bus_id: str | None = None, period_s: float = 0.01):
        self.gpu = gpu_index
        self.pci = pci_bus_id
        self.period = period_s
        self.proc = None
        self.thread = None
        self.stop = threading.Event()
        self.samples = []          # (time, sm_mhz, max_mhz, reasons set)
        self.source = None
        self.t0, self.t1 = -1e30, 1e30

    # -- NVML
    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.pci:
            try:
                return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(self.pci)
            except pynvml.NVMLError:
                pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll_nvml(self, nv, h):
        bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
        while not self.stop.is_set():
            ts = time.perf_counter()
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            except nv.NVMLError:
                break
            self.samples.append((ts, sm, mx, {n for n, b in bits.items() if rs & b}))
            self.stop.wait(self.period)

    # -- nvidia-smi fallback
    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm, mx = float(parts[0]), float(parts[1])
            except ValueError:
                continue
            rs = {n for n, v in zip(self.REASONS, parts[4:8]) if v.lower() == "active"}
            self.samples.append((time.perf_counter(), sm, mx, rs))

    def __enter__(self):
        try:
            nv, h = self._nvml_handle()
            self.thread = threading.Thread(target=self._poll_nvml, args=(nv, h), daemon=True)
            self.source = "nvml, every %g ms" % (self.period * 1e3)
            self.thread.start()
            return self
        except Exception:  # no NVML: sample with nvidia-smi instead
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.source = "nvidia-smi -lms 200"
            self.thread.start()
        except (OSError, ValueError):
            self.proc = None
        return self

    def mark_start(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def __exit__(self, *exc):
        self.stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self):
        """Median SM clock and active throttle reasons over the samples taken
        inside the marked (timed) window."""
        inside = [s for s in self.samples if self.t0 <= s[0] <= self.t1]
        sm = [s[1] for s in inside]
        reasons = set()
        for s in inside:
            reasons |= s[3]
        mx = inside[-1][2] if inside else (self.samples[-1][2] if self.samples else None)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "sm_mhz_min": min(sm) if sm else None, "reasons": sorted(reasons),
                "samples": len(sm), "source": self.source}


# ------------------------------------------------------------------ CPU oracle
def cpu_oracle_sample(w: W.Workload, q, k, v, target_seconds: float, seed: int = 0):
    """Time the oracle on a seeded sample of query rows sized to about
    ``target_seconds`` of CPU work.  Returns (TFLOPS, threads, description)."""
    import oracle
    from exact_attention_113_b200.inputs import to_bits
    qb, kb, vb = to_bits(q), to_bits(k), to_bits(v)
    rng = np.random.default_rng(seed)
    n_total = w.B * w.H * w.L_q
    # calibrate on a few rows, then size the sample
    probe = rng.integers(0, n_total, size=64)
    t0 = time.perf_counter()
    oracle.attention_rows(qb, kb, vb, w.dtype, w.softmax_scale, w.causal, w.window_left,
                          w.window_right, rows=probe)
    dt = max(time.perf_counter() - t0, 1e-6)
    n = int(min(n_total, max(64, 64 * target_seconds / dt)))
    rows = np.sort(rng.choice(n_total, size=n, replace=False))
    t0 = time.perf_counter()
    _, _, used = oracle.attention_rows(qb, kb, vb, w.dtype, w.softmax_scale, w.causal,
                                       w.window_left, w.window_right, rows=rows)
    dt = time.perf_counter() - t0
    tflops = row_flops(w, rows) / dt / 1e12
    desc = (f"{n} of {n_total} query rows ({n / n_total:.3%}), seeded uniform sample, "
            f"fp64 oracle, {dt:.1f} s")
    return tflops, used, desc


# ------------------------------------------------------------------ our arm
def run_ours(args, w: W.Workload):
    import torch
    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import exact_attention_113_b200 as fa

    # per-rank problem: same shape, its own seed (weak scaling)
    w_rank = W.Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank})
    fp8 = getattr(args, "fp8", False)
    q_cpu, k_cpu, v_cpu = W.make_qkv_fp8(w_rank) if fp8 else W.make_qkv(w_rank)
    q, k, v = (t.to(dev) for t in (q_cpu, k_cpu, v_cpu))
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev) if fp8 else torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.L_q), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    bwd = args.pass_ == "bwd"
    n_splits = 0 if bwd else resolve_splits(args.splits, w, fp8)
    ws = None
    if n_splits:
        ws = torch.empty(fa.fa_splitkv_workspace_bytes(w.B, w.H, w.L_q, w.D, n_splits),
                         dtype=torch.uint8, device=dev)
    launches_per_step = 3 if bwd else (2 if n_splits else 1)
    fm = BWD_FLOP_FACTOR if bwd else 1.0

    if bwd:
        do_cpu = W.make_dout(w_rank)
        dout = do_cpu.to(dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        bws = torch.empty(fa.fa_bwd_workspace_bytes(w.B, w.H, w.L_q, w.D), dtype=torch.uint8,
                          device=dev)
        with torch.cuda.stream(stream):
            fa.flash_fwd(q, k, v, scale=w.softmax_scale, causal=w.causal,
                         window_left=w.window_left, window_right=w.window_right,
                         out=out, lse=lse, stream=stream)

        def step():
            fa.flash_bwd(q, k, v, out, dout, lse, scale=w.softmax_scale, causal=w.causal,
                         window_left=w.window_left, window_right=w.window_right, dq=dq, dk=dk,
                         dv=dv, workspace=bws, stream=stream)
    elif fp8:
        def step():
            fa.flash_fwd_fp8(q, k, v, scale=w.softmax_scale, causal=w.causal,
                             window_left=w.window_left, window_right=w.window_right,
                             out=out, lse=lse, stream=stream, n_splits=n_splits, workspace=ws)
    else:
        def step():
            fa.flash_fwd(q, k, v, scale=w.softmax_scale, causal=w.causal,
                         window_left=w.window_left, window_right=w.window_right,
                         out=out, lse=lse, stream=stream, n_splits=n_splits, workspace=ws)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    if fa.fa_get_device_status(stream.cuda_stream) != 0:
        raise RuntimeError("device watchdog fired during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    # inputs and outputs that fit in L2 twice over: write a buffer larger than
    # L2 between timed steps (outside their events); the step time is then the
    # sum of the steps' own times
    flush = None
    if min_hbm_bytes(w, 1 if fp8 else 2) < L2_FLUSH_BELOW:
        flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    props = torch.cuda.get_device_properties(dev)
    pci = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
    with ClockSampler(physical_gpu_index(dev.index), pci) as clk:
        time.sleep(0.3)                    # let the sampler start
        # the GPU idled during that pause: one more untimed step right before
        # the timed ones (the same sequence as a timed step, flush included),
        # or the first of them pays for the wake-up
        with torch.cuda.stream(stream):
            if flush is not None:
                flush.fill_(0.0)
            step()
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        clk.mark_start()
        with torch.cuda.stream(stream):
            for s in range(args.steps):
                if flush is not None:
                    flush.fill_(float(s))
                starts[s].record(stream)
                step()
                ends[s].record(stream)
        torch.cuda.synchronize(dev)
        clk.mark_end()
        barrier(world, dev)
    launch_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    if flush is None:
        total_s = starts[0].elapsed_time(ends[-1]) / 1e3
    else:
        total_s = sum(launch_ms) / 1e3
    if fa.fa_get_device_status(stream.cuda_stream) != 0:
        raise RuntimeError("device watchdog fired during the timed steps")
    max_total = max_over_ranks(total_s, world, dev)
    value = whole_job_value(fm * metric_flops(w), world, args.steps, max_total)
    avg_launch_s = sum(launch_ms) / len(launch_ms) / 1e3

    # ---- roofline of the (only) kernel
    peaks, peak_kind = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    if fp8:
        peak *= 2.0                 # nominal fp8 / bf16 dense ratio
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    in_bytes = 1 if fp8 else 2
    if bwd or roofline_bound(w, peak, hbm, in_bytes) == "tensor":
        achieved = fm * algorithmic_flops(w) / avg_launch_s / 1e12
        sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        if fp8:
            sustained *= 2.0
        roofline = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                    "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                    # the same against the power-capped rate of a seconds-long
                    # cuBLAS loop (this bench's steps also run back to back)
                    "peak_sustained": sustained,
                    "frac_of_sustained": round(achieved / sustained, 4),
                    "traffic": profiled_traffic() if w.name == W.ROOFLINE.name else None,
                    "traffic_source": (os.path.relpath(TRAFFIC_SUMMARY, ROOT)
                                       if w.name == W.ROOFLINE.name else None),
                    "peak_source": (f"{peak_kind} cuBLAS bf16 burst x 2 (nominal fp8 ratio)" if fp8
                                    else f"{peak_kind} cuBLAS bf16 burst (fp16 dense rate is the same)")}
    else:
        achieved = min_hbm_bytes(w, in_bytes) / avg_launch_s / 1e9
        roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm,
                    "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": None,
                    "peak_source": f"{peak_kind} HBM copy bandwidth"}
    roofline.update({"algorithmic_flop_per_launch": fm * algorithmic_flops(w),
                     "min_hbm_bytes_per_launch": min_hbm_bytes(w, in_bytes)})
    if bwd:
        roofline["traffic"] = None
        roofline["timed"] = "whole step: prep, gradient kernel and dQ conversion launches"
    if n_splits:
        roofline["timed"] = (f"whole step: split-KV launch ({n_splits} key slices) "
                             "plus merge launch")
    clocks = clk.summary()
    if clocks.get("sm_mhz"):
        clocks["ms_x_mhz"] = round(avg_launch_s * 1e3 * clocks["sm_mhz"], 1)
    exp_bound = exp_roof(w, avg_launch_s, clocks.get("sm_mhz") or clocks.get("sm_max_mhz"),
                         bwd)
    exp_bound["clock"] = ("median SM clock sampled in the timed region" if clocks.get("sm_mhz")
                          else "no sample in the timed region: the maximum SM clock")

    # ---- end to end through host buffers (pinned), rank-local
    e2e = None
    if not args.skip_e2e:
        hq, hk, hv = (t.pin_memory() for t in (q_cpu, k_cpu, v_cpu))
        if bwd:
            # inputs: q, k, v, out, dout, lse; results: dq, dk, dv
            h_in = [hq, hk, hv, out.cpu().pin_memory(), do_cpu.pin_memory(),
                    lse.cpu().pin_memory()]
            d_in = [q, k, v, out, dout, lse]
            d_out = [dq, dk, dv]
        else:
            h_in = [hq, hk, hv]
            d_in = [q, k, v]
            d_out = [out, lse]
        h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in d_out]
        host_api = not bwd and not fp8 and not n_splits
        if host_api:
            # the forward through fa_fwd_host: chunked copies in and out on
            # their own streams, overlapped with the kernels
            hws = torch.empty(fa.fa_fwd_host_workspace_bytes(w.B, w.H, w.H_kv, w.L_q, w.L_k,
                                                             w.D, args.host_chunks),
                              dtype=torch.uint8, device=dev)

        def e2e_step():
            if host_api:
                fa.flash_fwd_host(hq, hk, hv, scale=w.softmax_scale, causal=w.causal,
                                  window_left=w.window_left, window_right=w.window_right,
                                  out=h_out[0], lse=h_out[1], n_chunks=args.host_chunks,
                                  workspace=hws, device=dev, stream=stream)
                return
            for d, h in zip(d_in, h_in):
                d.copy_(h, non_blocking=True)
            step()
            for h, d in zip(h_out, d_out):
                h.copy_(d, non_blocking=True)

        n_e2e = max(3, min(args.steps, 10))
        with torch.cuda.stream(stream):
            e2e_step()
            torch.cuda.synchronize(dev)
            barrier(world, dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n_e2e):
                e2e_step()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)
        h2d = sum(t.numel() * t.element_size() for t in h_in)
        d2h = sum(t.numel() * t.element_size() for t in h_out)
        e2e = {"value": round(whole_job_value(fm * metric_flops(w), world, n_e2e, e2e_s), 2),
               "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "path": (f"fa_fwd_host, {args.host_chunks} chunks, copies overlapped" if host_api
                        else "copies in, step, copies out on one stream"),
               "steps": n_e2e, "ms_per_step": round(e2e_s / n_e2e * 1e3, 3)}

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline and not bwd and not fp8:
        tf, cores, desc = cpu_oracle_sample(w, q_cpu, k_cpu, v_cpu, args.cpu_seconds)
        cpu = {"value": round(tf, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": desc, "host_nproc": os.cpu_count()}

    line = {
        "metric": METRIC_BWD if bwd else METRIC, "value": round(value, 2), "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(max_total / args.steps * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if fp8 else ("f16" if w.dtype == W.F16 else "bf16"),
        "data": "synthetic (seeded N(0,%g) inputs, per-rank seeds)" % w.std,
        "config": workload_config(w, world, flush is not None),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "clocks": clocks, "gpu_launches": args.steps * launches_per_step,
        "exp_bound": exp_bound,
        "pct_of_tensor_peak": round(100.0 * value / world / peak, 2),
        "launch_ms": {"min": round(min(launch_ms), 4), "median": round(statistics.median(launch_ms), 4),
                      "max": round(max(launch_ms), 4)},
    }
    if n_splits:
        line["config"]["entry"] = "fa_fwd_splitkv"
        line["config"]["n_splits"] = n_splits
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def exp_roof(w: W.Workload, launch_s: float, sm_mhz, bwd: bool = False) -> dict:
    """The third roof: one exponential per visible (query, key) pair (the
    backward recomputes them once more) against MUFU's ex2 rate at the
    sampled SM clock."""
    mhz = float(sm_mhz) if sm_mhz else 1965.0
    exps = float(w.B * w.H * visible_pairs_per_head(w))
    per_clk_sm = exps / (launch_s * mhz * 1e6 * SM_COUNT)
    return {"exps_per_launch": exps, "achieved_per_clk_per_sm": round(per_clk_sm, 3),
            "peak_per_clk_per_sm": MUFU_EX2_PER_CLK_SM,
            "frac": round(per_clk_sm / MUFU_EX2_PER_CLK_SM, 4), "sm_mhz_used": mhz,
            "note": "backward: P recomputed once" if bwd else "forward"}


def resolve_splits(arg: str, w: W.Workload, fp8: bool = False) -> int:
    """--splits: 0 (fa_fwd), an explicit slice count, or auto."""
    if arg == "auto":
        from exact_attention_113_b200.binding import choose_splits
        return choose_splits(w.B, w.H, w.L_q, w.L_k, H_kv=w.H_kv, D=w.D,
                             dtype=2 if fp8 else w.dtype)
    return int(arg)


def roofline_bound(w: W.Workload, tflops: float, gbs: float, in_bytes: int = 2) -> str:
    """Whichever of the tensor pipe and HBM takes longer for the workload's
    algorithmic FLOPs and minimum bytes."""
    t_tensor = algorithmic_flops(w) / (tflops * 1e12)
    t_hbm = min_hbm_bytes(w, in_bytes) / (gbs * 1e9)
    return "tensor" if t_tensor >= t_hbm else "hbm"


def min_hbm_bytes(w: W.Workload, in_bytes: int = 2) -> int:
    """Q, K, V read once (in_bytes per element: 2, or 1 for E4M3 codes), O
    written once (2 B/elem: fp16 / bf16), lse written (4 B/row)."""
    q = w.B * w.H * w.L_q * w.D
    kv = 2 * w.B * w.H_kv * w.L_k * w.D
    return (q + kv) * in_bytes + q * 2 + 4 * w.B * w.H * w.L_q


def workload_config(w: W.Workload, world: int, flushed: bool = False) -> dict:
    return {"workload": w.name, "B": w.B, "H": w.H, "H_kv": w.H_kv, "L_q": w.L_q,
            "L_k": w.L_k, "D": w.D, "causal": w.causal, "window_left": w.window_left,
            "window_right": w.window_right, "scale": w.softmax_scale,
            "input_dtype": W.DTYPE_NAME[w.dtype], "accumulate": "fp32",
            "l2": (f"L2 flushed between steps ({L2_FLUSH_BYTES >> 20} MiB written outside "
                   "the steps' events)" if flushed
                   else "inputs larger than L2 (no flush between steps)"),
            "parallelism": f"{world} independent replica(s), one per GPU"}


# ------------------------------------------------------------------ reference arm
def run_reference(args, w: W.Workload):
    world, rank, _ = dist_env()
    if rank != 0:
        return                       # rank 0 alone runs the CPU oracle
    q, k, v = W.make_qkv(w)
    import oracle
    from exact_attention_113_b200.inputs import to_bits
    qb, kb, vb = to_bits(q), to_bits(k), to_bits(v)
    n_total = w.B * w.H * w.L_q
    rng = np.random.default_rng(1)
    # size one step to ~target seconds of CPU work from a short calibration
    probe = rng.integers(0, n_total, size=32)
    t0 = time.perf_counter()
    oracle.attention_rows(qb, kb, vb, w.dtype, w.softmax_scale, w.causal, w.window_left,
                          w.window_right, rows=probe)
    per_row = max(time.perf_counter() - t0, 1e-6) / 32
    n = int(max(32, min(n_total, args.ref_step_seconds / per_row)))
    times, flops, used = [], 0.0, 0
    for s in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(n_total, size=n, replace=False))
        t0 = time.perf_counter()
        _, _, used = oracle.attention_rows(qb, kb, vb, w.dtype, w.softmax_scale, w.causal,
                                           w.window_left, w.window_right, rows=rows)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
            flops += row_flops(w, rows)
    total = sum(times)
    value = flops / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded N(0,%g) inputs)" % w.std,
        "config": workload_config(w, world),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": used,
                         "kind": "oracle",
                         "sample": f"{n} of {n_total} query rows per step, seeded uniform "
                                   f"samples, fp64 oracle on the host cores"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.ALL))
    ap.add_argument("--pass", dest="pass_", choices=("fwd", "bwd"), default="fwd",
                    help="time the forward (default) or the backward")
    ap.add_argument("--host-chunks", type=int, default=16,
                    help="chunks of the host-buffer forward in the e2e leg")
    ap.add_argument("--fp8", action="store_true",
                    help="time fa_fwd_fp8 on the inputs converted to E4M3")
    ap.add_argument("--splits", default="0",
                    help="key slices for fa_fwd_splitkv (0: plain fa_fwd; auto)")
    ap.add_argument("--sweep", action="store_true",
                    help="one line per named workload (kernel timing only)")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU work in the cpu_baseline sample")
    ap.add_argument("--ref-step-seconds", type=float, default=4.0,
                    help="CPU work per step of --impl reference")
    ap.add_argument("--ingest-ncu", metavar="CSV",
                    help="write the DRAM traffic summary of the workload from an ncu "
                         "--csv capture of dram__bytes_read.sum and dram__bytes_write.sum")
    ap.add_argument("--ncu-command", default="",
                    help="with --ingest-ncu: the command line that made the capture")
    args = ap.parse_args(argv)
    if args.ingest_ncu:
        ingest_ncu(args.ingest_ncu, args.ncu_command, W.ALL[args.workload])
        return
    args.warmup = max(3, args.warmup)      # at least 3 untimed warm-up steps
    args.steps = max(1, args.steps)
    if args.sweep and args.impl == "ours":
        import gc
        named = W.TINY + [W.GPT2] + W.MEMTABLE + W.SWEEP + [W.GQA_WINDOW, W.ROOFLINE]
        for wk in named + W.DECODE:
            sub = argparse.Namespace(**vars(args))
            sub.skip_cpu_baseline = True
            sub.skip_e2e = True
            sub.splits = "auto" if wk in W.DECODE else "0"
            run_ours(sub, wk)
            gc.collect()
        return
    w = W.ALL[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
