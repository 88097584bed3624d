"""Benchmark of the MoE FFN layer forward on B200 (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one moe_layer_forward over the whole workload (route, permute, gate/up GEMM
with SwiGLU, down GEMM, shared expert if any, combine) with inputs resident in HBM.
L2 is flushed (a 512 MiB write) before every timed step, outside the timed events.
With N > 1 (torchrun, one process per GPU) every rank runs an independent replica of
the layer on its own inputs (the layer has no cross-GPU exchange on one node's data
path): the reported value is all ranks' tokens over the slowest rank's time.

The headline workload is the DeepSeek-V3-shaped prefill layer (T=8192, H=7168, I=2048,
256 routed experts, top-8, plus a shared expert), the largest of the five workloads.
On one GPU the line also carries, under "configs", the same record for each of the
other four workloads (tiny, Mixtral-shaped prefill, DeepSeek-V3-shaped decode, skewed
FP8) and for the decode layer with e2m1 expert weights, each timed over enough steps to
fill a few hundred ms, and under "micro" the GroupedTopK kernel alone (83 tokens, 256
experts) in us per call.

Each record has `value` (tokens/s), the grouped-GEMM TFLOP/s and each GEMM kernel's
fraction of the measured bf16 burst peak, an end-to-end number through
moe_layer_forward_host_batches (each batch's host activations copied in and its output
copied back inside the timed region, overlapping the neighbouring batches' layers), the
roofline of the dominant kernel from CUDA events recorded around
its launches, the SM clocks sampled (NVML, every 5 ms) during the timed region, and the
fp64 CPU oracle timed on a bounded sample of the same workload.  `--impl reference`
times that oracle alone, per step, on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mixture_experts_ffn_08_b200 import binding as B  # noqa: E402
from mixture_experts_ffn_08_b200 import inputs, workloads as W  # noqa: E402

METRIC = "MoE layer tokens/s and grouped-GEMM TFLOP/s (or HBM GB/s) vs B200 roofline"
FLUSH_BYTES = 512 << 20


GEMM_SOURCES = ("csrc/tc_gemm.cuh", "csrc/common.cuh", "csrc/gemm.cu")
DUAL_GEMM_SOURCES = ("csrc/tc_gemm_dual.cuh", "csrc/tc_gemm.cuh", "csrc/common.cuh", "csrc/gemm.cu")
FP8_GEMM_SOURCES = ("csrc/tc_gemm_fp8.cuh", "csrc/tc_gemm.cuh", "csrc/common.cuh", "csrc/gemm_fp8.cu")


def gateup_sources(wl):
    """Source files of the gate/up kernel the library runs for this workload: the
    block-scaled GEMM for e4m3 activations; for bf16, the two-M-tile GEMM when the
    average expert holds two 128-row M-tiles (T*K >= 256*E), else the one-tile GEMM."""
    if wl.dtype in (W.DTYPE_FP8, W.DTYPE_FP8_FP4):
        return FP8_GEMM_SOURCES
    return DUAL_GEMM_SOURCES if wl.T * wl.K >= 256 * wl.E else GEMM_SOURCES


def sources_sha256(files):
    """sha256 over the given source files of the package, in order."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "mixture_experts_ffn_08_b200", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _profiled_traffic(workload, sources=GEMM_SOURCES, algorithmic_bytes=None):
    """(DRAM bytes per launch of the gate/up kernel, where the figure comes from), from the
    committed ncu summary of this workload; (None, reason) if there is none, it covers
    another kernel than `sources` (the files of the kernel that runs now), or those
    sources changed since it was taken.  A summary gives either the bytes of a full-size
    capture (traffic_bytes_per_launch:) or, for a workload too large to capture, the
    ratio of DRAM bytes to algorithmic bytes measured on a smaller case of the same
    kernel (traffic_per_algorithmic_byte:, scaled_from:), which is applied to this run's
    algorithmic bytes.  The summary names the sources it covers (kernel_sources:,
    default the bf16 GEMM)."""
    import re
    path = os.path.join(ROOT, "profiles", f"gateup_swiglu_{workload}.md")
    if not os.path.exists(path):
        return None, "no ncu summary for this workload"
    txt = open(path, encoding="utf-8").read()
    m_t = re.search(r"^traffic_bytes_per_launch:\s*(\d+)", txt, re.M)
    m_r = re.search(r"^traffic_per_algorithmic_byte:\s*([0-9.]+)", txt, re.M)
    m_f = re.search(r"^scaled_from:\s*(.+)$", txt, re.M)
    m_h = re.search(r"^kernel_source_sha256:\s*([0-9a-f]+)", txt, re.M)
    m_s = re.search(r"^kernel_sources:\s*(.+)$", txt, re.M)
    if not ((m_t or m_r) and m_h):
        return None, "ncu summary without a traffic figure"
    files = [f.strip() for f in m_s.group(1).split(",")] if m_s else list(GEMM_SOURCES)
    if files != list(sources):
        return None, "ncu summary covers another kernel"
    if sources_sha256(files) != m_h.group(1):
        return None, "kernel sources changed since the ncu capture"
    if m_t:
        return int(m_t.group(1)), f"ncu capture of {workload} (profiles/gateup_swiglu_{workload}.md)"
    if algorithmic_bytes is None:
        return None, "scaled figure needs the algorithmic bytes"
    ratio = float(m_r.group(1))
    return int(ratio * algorithmic_bytes), (f"DRAM/algorithmic bytes {ratio:.4f} measured on "
                                            f"{m_f.group(1).strip() if m_f else 'a smaller case'}, "
                                            f"times this launch's algorithmic bytes")


def _peaks():
    """(bf16 burst TFLOP/s, bf16 sustained TFLOP/s, HBM GB/s, kind)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), d["hbm_gbs"], "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


REFERENCE_BUDGET_S = 90.0   # oracle seconds for a whole --impl reference run
# nominal dense peaks of one B200, for the spec-relative fractions beside the measured ones
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0    # the "~8 TB/s" the decode target is stated against
FP8_OVER_BF16 = 2.0   # nominal dense e4m3 / bf16 tensor throughput (4.5 / 2.25 PFLOP/s)


def power_capped(clk) -> bool:
    """Whether the clock record says the power cap held the SM clock (sw_power_cap in at
    least a fifth of the in-window samples, or a median under load below 90 % of the
    maximum).  Reported beside the roofline; the fraction itself is always taken
    against the burst peak."""
    if not clk:
        return False
    n = clk.get("samples_in_window") or clk.get("samples") or 0
    capped_samples = clk.get("sw_power_cap_samples")
    if capped_samples is None:
        by_reason = "sw_power_cap" in clk.get("reasons", [])
    else:
        by_reason = n > 0 and capped_samples >= 0.2 * n
    low = bool(clk.get("sm_mhz") and clk.get("sm_max_mhz") and clk["sm_mhz"] < 0.9 * clk["sm_max_mhz"])
    return bool(by_reason or low)


def roofline_record(flops, nbytes, launch_ms, clk, fp8, peaks):
    """Roofline of one kernel from its algorithmic FLOPs and bytes per launch and its
    launch times (ms): tensor-bound when flops/bytes reaches the ridge of the peaks,
    else HBM-bound.  `frac` is taken against the measured burst tensor peak (these
    kernels run for milliseconds inside steps of milliseconds); frac_of_sustained is
    the same figure against the seconds-long power-capped loop, frac_of_nominal against
    the nominal dense peak (2.25 PFLOP/s bf16, ~8 TB/s HBM).  e4m3 takes twice the bf16
    figure (the nominal dense ratio).  peaks = (bf16 burst TFLOP/s, bf16 sustained
    TFLOP/s, HBM GB/s, kind)."""
    burst, sustained, hbm_peak, peak_kind = peaks
    ratio = FP8_OVER_BF16 if fp8 else 1.0
    tensor_peak = burst * ratio
    avg = statistics.mean(launch_ms) if launch_ms else None
    ridge = tensor_peak * 1e12 / (hbm_peak * 1e9)
    if flops / nbytes >= ridge:
        achieved = flops / (avg / 1e3) / 1e12 if avg else None
        rec = {"bound": "tensor", "achieved": achieved, "peak": tensor_peak, "unit": "TFLOP/s",
               "peak_kind": f"{peak_kind} bf16 burst" + (" x2 (e4m3/bf16 nominal ratio)" if fp8 else ""),
               "frac_of_sustained": achieved / (sustained * ratio) if achieved else None}
    else:
        achieved = nbytes / (avg / 1e3) / 1e9 if avg else None
        rec = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
               "peak_kind": f"{peak_kind} HBM copy"}
    nominal = NOMINAL_BF16_TFLOPS * ratio if rec["bound"] == "tensor" else NOMINAL_HBM_GBS
    rec.update({"frac": achieved / rec["peak"] if achieved else None,
                "frac_of_nominal": achieved / nominal if achieved else None, "nominal_peak": nominal,
                "launches_timed": len(launch_ms),
                "avg_ms": avg, "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": nbytes,
                "tflops": flops / (avg / 1e3) / 1e12 if avg else None,
                "gbs": nbytes / (avg / 1e3) / 1e9 if avg else None,
                "power_capped": power_capped(clk)})
    return rec


def _describe(wl):
    s = (f"T={wl.T} H={wl.H} I={wl.I} E={wl.E} K={wl.K} "
         f"{'softmax' if wl.score_fn == 0 else 'sigmoid'}")
    if wl.n_group > 1:
        s += f" groups={wl.n_group}/keep{wl.topk_group}/top{wl.group_topn}"
    if wl.has_bias:
        s += " bias"
    s += f" renorm x{wl.routed_scale:g}" if wl.renormalize else f" x{wl.routed_scale:g}"
    if wl.I_shared:
        s += f" +shared I={wl.I_shared}"
    if wl.fused_combine:
        s += " fused-combine"
    if wl.block_m:
        s += f" block_m={wl.block_m}"
    if wl.masked_cap:
        s += f" masked-layout cap={wl.masked_cap}"
    return s + {W.DTYPE_BF16: " bf16", W.DTYPE_FP8: " fp8", W.DTYPE_FP8_FP4: " fp8 x fp4 weights"}[wl.dtype]


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest value over all ranks (the slowest rank's time); the value itself on one
    rank.  Every rank must call it at the same point."""
    if world <= 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank: int, world: int, ms_step: float) -> float:
    """Whole-job tokens/s of `world` independent replicas, each processing tokens_per_rank
    tokens per step, timed by the slowest rank's ms per step."""
    return tokens_per_rank * world / (ms_step / 1e3)


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ------------------------------------------------------------------ clocks
def _is_num(v):
    return v.replace(".", "", 1).isdigit()


def summarize_clock_rows(lines, window=None):
    """Summary of nvidia-smi samples (ClockSampler.FIELDS, csv, noheader, nounits): median SM
    clock under load, maximum SM clock, and the throttle reasons seen.  It is taken over the
    samples whose timestamps fall inside window = (t0, t1), host time.time() values around
    the timed region, or over all samples when none does (a region shorter than the
    sampling interval); samples_in_window says which."""
    from datetime import datetime
    rows = []
    for line in lines:
        r = [c.strip() for c in line.split(",")]
        if len(r) < 10:
            continue
        try:
            ts = datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            ts = None
        rows.append((ts, r))
    inside = [r for ts, r in rows if window and ts is not None and window[0] <= ts <= window[1]]
    use = inside or [r for _, r in rows]
    sm = [float(r[2]) for r in use if _is_num(r[2])]
    smax = [float(r[3]) for _, r in rows if _is_num(r[3])]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in use for i in range(4) if r[6 + i] == "Active"})
    loaded = [v for v in sm if smax and v > 0.5 * max(smax)] or sm
    pw = [float(r[4]) for r in use if _is_num(r[4])]
    return {"sm_mhz": statistics.median(loaded) if loaded else None,
            "power_w_median": statistics.median(pw) if pw else None,
            "sm_mhz_min": min(loaded) if loaded else None,
            "sm_max_mhz": max(smax) if smax else None, "reasons": reasons,
            "sw_power_cap_samples": sum(1 for r in use if r[9] == "Active"),
            "samples": len(rows), "samples_in_window": len(inside)}


class NvmlClockSampler:
    """Samples the SM clock, power and throttle reasons through NVML every 5 ms on a host
    thread (reading only), producing rows in ClockSampler's csv format."""
    INTERVAL_S = 0.005
    # NVML clocks-event reason bits: sw power cap, hw slowdown, sw thermal, hw thermal
    _CAP, _HW, _SWT, _HWT = 0x4, 0x8, 0x20, 0x40

    def __init__(self, device):
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(device).uuid)
        if not uuid.startswith("GPU-"):
            uuid = "GPU-" + uuid
        self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
        self.rows, self.thread, self.stop_flag = [], None, False

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(fn(self.h))

    def _loop(self):
        from datetime import datetime
        nv = self.nv
        smax = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        act = lambda bits, b: "Active" if bits & b else "Not Active"  # noqa: E731
        while not self.stop_flag:
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                r = self._reasons()
            except Exception:  # noqa: BLE001 - a failed read ends the sampling
                break
            ts = datetime.fromtimestamp(time.time()).strftime("%Y/%m/%d %H:%M:%S.%f")
            self.rows.append(f"{ts}, 0, {sm}, {smax}, {pw:.1f}, {r:#x}, {act(r, self._HW)}, "
                             f"{act(r, self._HWT)}, {act(r, self._SWT)}, {act(r, self._CAP)}")
            time.sleep(self.INTERVAL_S)

    def start(self):
        import threading
        self.thread = threading.Thread(target=self._loop, daemon=True)
        self.thread.start()
        time.sleep(0.05)

    def stop(self, window=None):
        time.sleep(0.05)
        self.stop_flag = True
        self.thread.join(timeout=5)
        rec = summarize_clock_rows(self.rows, window)
        rec["sampler"] = f"nvml every {self.INTERVAL_S * 1e3:g} ms"
        return rec


def clock_sampler(device):
    """NVML sampler where pynvml works, else nvidia-smi."""
    try:
        return NvmlClockSampler(device)
    except Exception:  # noqa: BLE001
        return ClockSampler(device)


class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 50

    def __init__(self, device):
        self.proc = None
        self.uuid = str(torch.cuda.get_device_properties(device).uuid)
        if not self.uuid.startswith("GPU-"):
            self.uuid = "GPU-" + self.uuid

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self, window=None):
        """window: (t0, t1) host time.time() values around the timed region."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.3)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        return summarize_clock_rows(out.strip().splitlines(), window)


# ------------------------------------------------------------------ CPU oracle leg
def _expert_f64_bytes(wl):
    return 3 * wl.H * wl.I * 8


def _host_cache_bytes():
    """fp64 expert weights the oracle leg may keep on the host: half the available RAM,
    at most 120 GiB."""
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:  # noqa: BLE001
        avail = 32 << 30
    return int(min(avail // 2, 120 << 30))


class HostWeights:
    """Expert weights for the oracle leg as exact fp64 values (bf16 widened, e4m3 codes
    times their block scales, e2m1 through the oracle's decoder), loaded when the oracle
    first asks for an expert and kept up to a host-memory cap, oldest first out.  Loading
    is reading the layer's inputs, not layer work: its time is accumulated in load_s and
    taken out of the oracle's measured time."""

    def __init__(self, wl, d, cap_bytes=None):
        self.wl, self.d, self.cache, self.load_s = wl, d, {}, 0.0
        cap = _host_cache_bytes() if cap_bytes is None else cap_bytes
        self.cap = max(1, cap // _expert_f64_bytes(wl))
        self.shared = None
        if wl.I_shared:
            self.shared = tuple(d[n].to(torch.float64).cpu().numpy() for n in ("ws_gate", "ws_up", "ws_down"))

    def _load(self, e):
        from oracle import moe_oracle as o
        wl, d = self.wl, self.d
        if wl.dtype == W.DTYPE_FP8:
            def deq(n):
                q = d[n + "_q"][e].view(torch.float8_e4m3fn).to(torch.float64)
                s = d[n + "_s"][e].to(torch.float64).repeat_interleave(128, 0).repeat_interleave(128, 1)
                return (q * s).cpu().numpy()
            return tuple(deq(n) for n in ("w_gate", "w_up", "w_down"))
        if wl.dtype == W.DTYPE_FP8_FP4:
            return tuple(o.dequant_fp4(d[n + "_q"][e].cpu().numpy(), d[n + "_s"][e].cpu().numpy())
                         for n in ("w_gate", "w_up", "w_down"))
        return tuple(d[n][e].to(torch.float64).cpu().numpy() for n in ("w_gate", "w_up", "w_down"))

    def __call__(self, e):
        e = int(e)
        if e not in self.cache:
            t0 = time.perf_counter()
            while self.cache and len(self.cache) >= self.cap:
                self.cache.pop(next(iter(self.cache)))
            self.cache[e] = self._load(e)
            self.load_s += time.perf_counter() - t0
        return self.cache[e]


def _oracle_sample(wl, d, n_tokens, seed=0, host_w=None):
    """Oracle forward (route + experts + combine) of a seeded token sample; returns
    (tokens, seconds, threads).  Host copies of the sampled activations are made before
    the clock starts; the time spent loading expert weights on first use (host_w, a
    HostWeights, which keeps them across calls) is taken out."""
    from oracle import moe_oracle as o
    from threadpoolctl import threadpool_info
    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(wl.T, size=min(n_tokens, wl.T), replace=False))
    idx = torch.as_tensor(toks, device=d["w_r"].device)
    if wl.dtype in (W.DTYPE_FP8, W.DTYPE_FP8_FP4):
        xq, xs = d["x_q"][idx].cpu().numpy(), d["x_scale"][idx].cpu().numpy()
        x_of = lambda: o.dequant_blocks(xq, xs, 1)  # noqa: E731
    else:
        xh = d["x"][idx].cpu().to(torch.float64).numpy()
        x_of = lambda: xh  # noqa: E731
    w_r = d["w_r"].cpu().to(torch.float64).numpy()
    bias = d["bias"].cpu().to(torch.float64).numpy() if d["bias"] is not None else None
    if host_w is None:
        host_w = HostWeights(wl, d)
    load0 = host_w.load_s
    t0 = time.perf_counter()
    o.layer_forward(x_of(), w_r, bias, host_w, wl, host_w.shared)
    dt = time.perf_counter() - t0 - (host_w.load_s - load0)
    threads = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    return len(toks), dt, threads


def _cpu_sample_tokens(wl):
    """Tokens in one oracle sample: about 2e12 fp64 FLOP of expert work (a few seconds on
    the host cores), at least 4, at most the batch."""
    per_token_flops = 6 * wl.K * wl.H * wl.I + 6 * wl.H * wl.I_shared
    return int(max(4, min(wl.T, 2.0e12 / max(per_token_flops, 1))))


CPU_MIN_SECONDS = 2.0   # a sample shorter than this is repeated (same tokens) until it is not


def host_cpu():
    """(CPU model name, logical CPUs) of the host, from /proc/cpuinfo and os.cpu_count()."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo", encoding="utf-8", errors="replace") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return model, os.cpu_count()


def oracle_flops_per_token(wl) -> float:
    """Multiply-add work of one token through the layer as the oracle computes it: router
    logits, K routed SwiGLU FFNs, the shared expert (2 FLOP per multiply-add)."""
    return 2.0 * wl.H * wl.E + wl.K * 6.0 * wl.H * wl.I + 6.0 * wl.H * wl.I_shared


def cpu_baseline_record(wl, d):
    host_w = HostWeights(wl, d)
    n, dt, threads = _oracle_sample(wl, d, _cpu_sample_tokens(wl), host_w=host_w)
    reps = 1
    while dt < CPU_MIN_SECONDS and reps < 10000:
        _, t, _ = _oracle_sample(wl, d, n, host_w=host_w)
        dt += t
        reps += 1
    what = f"{n} seeded tokens" + (f", {reps} times" if reps > 1 else "")
    model, ncpu = host_cpu()
    return {"value": n * reps / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "gflops": n * reps / dt * oracle_flops_per_token(wl) / 1e9,
            "cpu_model": model, "host_logical_cpus": ncpu,
            "sample": f"{what}, of {wl.name} through the fp64 oracle (route, experts, combine; the time "
                      f"to load expert weights as fp64 is not counted); {dt:.2f} s"}


# ------------------------------------------------------------------ our arm
def _steps_for(ms_one, min_steps, target_ms=300.0, max_steps=1000):
    """Steps that fill about target_ms of device time, at least min_steps."""
    return int(min(max(min_steps, -(-target_ms // max(ms_one, 1e-3))), max(max_steps, min_steps)))


def _gemm_peak(wl):
    burst = _peaks()[0]
    return burst * (FP8_OVER_BF16 if wl.dtype in (W.DTYPE_FP8, W.DTYPE_FP8_FP4) else 1.0)


def measure(wl, steps, warmup, world=1, rank=0, local=0, cpu=True, adapt_steps=False):
    """One workload: W warm-up steps, then the timed steps (L2 flushed before each),
    the per-kernel breakdown, the end-to-end run through the host entry point, and
    (rank 0, one GPU) the oracle's CPU baseline.  Returns the record (rank 0) or None."""
    p = B.params(wl)
    d = inputs.make_inputs(wl, seed=rank, device="cuda")
    fp8 = wl.dtype in (W.DTYPE_FP8, W.DTYPE_FP8_FP4)     # e4m3 activations
    w4 = wl.dtype == W.DTYPE_FP8_FP4                    # e2m1 expert weights
    a = dict(x=d["x_q"] if fp8 else d["x"], x_scale=d.get("x_scale"))
    scales = [d.get("w_gate_s"), d.get("w_up_s"), d.get("w_down_s")]
    if w4:  # weight-load step, once: UE8M0 scale bytes -> tensor-core scale atoms
        scales = []
        for n, rows, K in (("w_gate", wl.E * wl.I, wl.H), ("w_up", wl.E * wl.I, wl.H),
                           ("w_down", wl.E * wl.H, wl.I)):
            atoms = torch.empty(rows * K // 32, dtype=torch.uint8, device="cuda")
            B.check(B.moe_prepare_fp4_scales(d[n + "_s"], rows, K, atoms), "moe_prepare_fp4_scales")
            scales.append(atoms)
    wts = [d["w_gate_q"] if fp8 else d["w_gate"], d["w_up_q"] if fp8 else d["w_up"],
           d["w_down_q"] if fp8 else d["w_down"], *scales,
           d.get("ws_gate"), d.get("ws_up"), d.get("ws_down")]
    ws_bytes = B.moe_workspace_size_host(p)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    ids = torch.empty((wl.T, wl.K), dtype=torch.int32, device="cuda")
    wgt = torch.empty((wl.T, wl.K), dtype=torch.float32, device="cuda")
    counts = torch.empty((wl.E,), dtype=torch.int32, device="cuda")
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    B.check(B.moe_clear_device_status(ws))

    def step():
        B.check(B.moe_layer_forward(p, a["x"], a["x_scale"], d["w_r"], d["bias"], *wts, out, ids, wgt,
                                    counts, ws, ws_bytes), "moe_layer_forward")

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if adapt_steps:  # fill a few hundred ms, so the clock record has many in-window samples
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        step()
        s1.record(stream)
        torch.cuda.synchronize()
        steps = _steps_for(s0.elapsed_time(s1), steps)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    # ---------------- timed region: device-resident inputs
    clocks = clock_sampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
    dominant = B.K_GATEUP
    B.check(B.moe_trace_enable(1 << dominant, 4 * steps))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier()
    t_region = time.time()
    for i in range(steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    barrier()
    t_region = (t_region, time.time())
    step_ms = [s.elapsed_time(e) for s, e in ev]
    traced = B.moe_trace_collect()
    B.moe_trace_disable()
    clk = clocks.stop(t_region) if clocks else None
    status = B.moe_get_device_status(ws)
    if status != 0:
        raise B.MoEError(f"device status {status:#x} after the timed steps of {wl.name}")

    # per-kernel breakdown: a few more steps, every kernel of the library bracketed by
    # events (outside the timed region, so the events do not perturb the headline)
    B.check(B.moe_trace_enable((1 << 13) - 1, 64 * 8))
    for _ in range(3):
        flush.fill_(0)
        step()
    breakdown = {}
    for k, ms in B.moe_trace_collect():
        breakdown.setdefault(B.KERNEL_NAMES[k], []).append(ms)
    B.moe_trace_disable()
    kernel_ms = {k: round(sum(v) / 3, 4) for k, v in breakdown.items()}

    counts_h = counts.cpu().numpy()
    P = wl.T * wl.K
    ms_total = max_over_ranks(float(sum(step_ms)), world, "cuda")
    ms_step = ms_total / steps
    tokens_per_s = replica_throughput(wl.T, world, ms_step)

    # algorithmic work (unpadded rows; weights of experts that received tokens)
    abytes = 1 if fp8 else 2                       # activation bytes per element
    wbytes = (0.5 + 1 / 32) if w4 else abytes       # weight bytes per element (e2m1: + one scale byte per 32)
    active = int((counts_h > 0).sum())
    flops = {"gateup_swiglu": 4.0 * P * wl.H * wl.I, "down": 2.0 * P * wl.I * wl.H,
             "shared_gateup": 4.0 * wl.T * wl.H * wl.I_shared, "shared_down": 2.0 * wl.T * wl.H * wl.I_shared}
    gemm_flops = sum(flops.values())
    bytes_gateup = (active * 2 * wl.I * wl.H * wbytes + P * wl.H * abytes + P * wl.I * abytes)
    # at prefill sizes the shared expert is one more group of the routed two-tile launches
    # (no launches of its own in the trace): its work then counts toward theirs
    shared_in_routed = wl.I_shared > 0 and "shared_gateup" not in kernel_ms
    if shared_in_routed:
        flops["gateup_swiglu"] += flops.pop("shared_gateup")
        flops["down"] += flops.pop("shared_down")
        bytes_gateup += 2 * wl.I_shared * wl.H * 2 + wl.T * wl.H * 2 + wl.T * wl.I_shared * 2
    layer_bytes = (active * 3 * wl.I * wl.H * wbytes + 3 * wl.I_shared * wl.H * 2 + wl.E * wl.H * 2
                   + wl.T * wl.H * (abytes + 2))
    dt_name = "e4m3 x e2m1" if w4 else ("e4m3" if fp8 else "bf16")
    dom_ms = [ms for k, ms in traced if k == dominant]
    roofline = roofline_record(flops["gateup_swiglu"], bytes_gateup, dom_ms, clk, fp8, _peaks())
    traffic, traffic_src = _profiled_traffic(wl.name, gateup_sources(wl), bytes_gateup)
    roofline.update({"kernel": f"gateup_swiglu (grouped GEMM, fused SwiGLU, {dt_name})",
                     "traffic": traffic, "traffic_source": traffic_src})
    peak_t = _gemm_peak(wl)
    hbm_peak = _peaks()[2]
    gemm_ms = sum(kernel_ms.get(k, 0.0) for k in flops)
    bm = B.moe_effective_block_m(p)
    mma_rows = int(sum(-(-int(c) // bm) * bm for c in counts_h))   # bucket rows the routed GEMMs compute

    # ---------------- end to end: host activations in, host output out.  One call runs all
    # K batches through moe_layer_forward_host_batches: every batch's activations are
    # copied in from pinned host memory and its output copied back, the copies overlapping
    # the neighbouring batches' layers; timed as a whole (no L2 flush between batches).
    x_host = (d["x_q"] if fp8 else d["x"]).cpu().pin_memory()
    xs_host = d["x_scale"].cpu().pin_memory() if fp8 else None
    out_host = [torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]

    def e2e_run(n):
        B.check(B.moe_layer_forward_host_batches(p, [x_host] * n, [xs_host] * n if fp8 else None, d["w_r"],
                                                 d["bias"], *wts, [out_host[i % 2] for i in range(n)], ws,
                                                 ws_bytes), "moe_layer_forward_host_batches")
    e2e_run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    e2e_run(steps)
    e1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, "cuda") / steps
    xbytes = wl.T * wl.H * (1 if fp8 else 2) + (wl.T * (wl.H // 128) * 4 if fp8 else 0)

    base = cpu_baseline_record(wl, d) if (cpu and rank == 0 and world == 1) else None
    del d, ws, flush
    torch.cuda.empty_cache()
    if rank != 0:
        return None
    return {
        "workload": f"{wl.name}: {_describe(wl)}",
        "value": tokens_per_s, "unit": "tokens/s", "ms_per_step": ms_step, "steps": steps,
        "ms_per_step_median_rank0": statistics.median(step_ms),
        "dtype": "fp8xfp4" if w4 else ("fp8" if fp8 else "bf16"),
        "grouped_gemm_tflops": gemm_flops / (ms_step / 1e3) / 1e12 * world,
        "gemm_kernel_tflops": {k: f / (kernel_ms[k] / 1e3) / 1e12 for k, f in flops.items() if kernel_ms.get(k)},
        "gemm_kernel_frac_of_burst": {k: f / (kernel_ms[k] / 1e3) / 1e12 / peak_t
                                      for k, f in flops.items() if kernel_ms.get(k)},
        "gemm_kernels_frac_of_burst": (gemm_flops / (gemm_ms / 1e3) / 1e12 / peak_t) if gemm_ms else None,
        "layer_hbm_gbs": layer_bytes / (ms_step / 1e3) / 1e9 * world,
        "layer_hbm_frac": layer_bytes / (ms_step / 1e3) / 1e9 / hbm_peak,
        "layer_algorithmic_bytes": layer_bytes,
        "active_experts": active,
        "shared_expert_in_routed_launches": shared_in_routed,
        "routed_gemm_rows": {"real": P, "computed": mma_rows,
                             "pad_frac": (mma_rows - P) / mma_rows if mma_rows else 0.0},
        "e2e": {"value": wl.T * world / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": xbytes, "d2h_bytes_per_step": wl.T * wl.H * 2,
                "ms_per_step": e2e_ms,
                "how": "moe_layer_forward_host_batches over the K steps: each batch copied in from pinned "
                       "host memory and its output copied back, copies overlapping neighbouring batches; "
                       "no L2 flush between batches"},
        "roofline": roofline,
        "clocks": clk,
        "gpu_launches": B.moe_layer_launch_count(p) * steps,
        "cpu_baseline": base,
        "kernel_ms_per_step": kernel_ms,
        "expert_load": {"max": int(counts_h.max()), "min": int(counts_h.min()), "mean": P / wl.E},
    }


SUB_CONFIGS = ("tiny", "mixtral_prefill", "dsv3_decode", "skewed_fp8", "dsv3_prefill")
# beyond the five workloads: the DeepSeek-V3 decode layer with e2m1 expert weights
EXTRA_CONFIGS = ("dsv3_decode_fp4",)


def run_ours(args):
    world, rank, local = _dist()
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    wl = {**W.ALL, **W.PROFILE, **W.FP4}[args.workload]
    if args.fused_combine:
        wl = wl.with_(fused_combine=True)
    if args.block_m:
        wl = wl.with_(block_m=args.block_m)
    if args.masked_cap:
        wl = wl.with_(masked_cap=args.masked_cap)
    rec = measure(wl, args.steps, args.warmup, world, rank, local, cpu=not args.no_cpu_baseline)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    configs = None
    if world == 1 and not args.no_configs:
        configs = {}
        for name in SUB_CONFIGS + EXTRA_CONFIGS:
            if name == wl.name:
                continue
            # (the e2m1 record carries no CPU baseline: its oracle would first widen ~50 GB of
            # expert weights to fp64, a minute of the run for a figure the other records give)
            configs[name] = measure((W.ALL | W.FP4)[name], args.steps, args.warmup,
                                    cpu=not args.no_cpu_baseline and name not in EXTRA_CONFIGS, adapt_steps=True)
        micro = {"grouped_topk": micro_grouped_topk_record(1000, args.warmup)}
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": rec["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": rec["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": rec["dtype"],
        "data": "synthetic (seeded Gaussian activations and random-init weights)",
        "config": {"workload": rec["workload"], "global_batch": wl.T * world,
                   "seq_len": 1, "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "flushed before every timed step (512 MiB write, outside the events)"},
    }
    line.update({k: v for k, v in rec.items() if k not in ("workload", "value", "unit", "ms_per_step",
                                                           "steps", "dtype")})
    if configs is not None:
        line["configs"] = configs
        line["micro"] = micro
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    world, rank, _ = _dist()
    if rank != 0:
        return
    wl = {**W.ALL, **W.PROFILE, **W.FP4}[args.workload]
    d = inputs.make_inputs(wl, seed=0, device="cpu" if not torch.cuda.is_available() else "cuda")
    host_w = HostWeights(wl, d)
    # Every step runs the same seeded token sample (as the GPU arm re-runs one batch);
    # expert weights are loaded as fp64 on first use, kept while host memory allows, and
    # their load time is not counted.  The sample makes all warm-up and timed steps
    # together take about REFERENCE_BUDGET_S of oracle time, at most the cpu sample.
    cap = min(wl.T, _cpu_sample_tokens(wl))
    k0, t0, _ = _oracle_sample(wl, d, min(cap, 64), seed=0, host_w=host_w)
    c1 = max(t0 / k0, 1e-6)
    per_step = REFERENCE_BUDGET_S / (args.warmup + args.steps)
    n = int(max(1, min(cap, per_step / c1)))
    times, toks, threads = [], 0, 1
    for i in range(args.warmup + args.steps):
        k, dt, threads = _oracle_sample(wl, d, n, seed=0, host_w=host_w)
        if i >= args.warmup:
            times.append(dt)
            toks += k
    value = toks / sum(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded Gaussian activations and random-init weights)",
        "config": {"workload": f"{wl.name}: {_describe(wl)}", "global_batch": wl.T, "seq_len": 1,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "gflops": value * oracle_flops_per_token(wl) / 1e9,
                         "cpu_model": host_cpu()[0], "host_logical_cpus": host_cpu()[1],
                         "sample": f"the same {n} seeded tokens every step through the fp64 oracle "
                                   f"(route, experts, combine; the time to load expert weights as "
                                   f"fp64 is not counted)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def micro_grouped_topk_record(steps, warmup):
    """GroupedTopK alone at the routing primer's KernelSwift shape (§十): 83 tokens, 256
    experts in 8 groups of 32, keep 4 groups, top-8, softmax, renormalised."""
    wl = W.Workload("grouped_topk_kernelswift", T=83, H=7168, I=128, E=256, K=8, n_group=8,
                    topk_group=4, group_topn=1)
    p = B.params(wl)
    g = torch.Generator(device="cuda").manual_seed(0)
    logits = torch.randn((wl.T, wl.E), generator=g, device="cuda")
    ids = torch.empty((wl.T, wl.K), dtype=torch.int32, device="cuda")
    w = torch.empty((wl.T, wl.K), dtype=torch.float32, device="cuda")
    for _ in range(warmup):
        B.check(B.moe_grouped_topk(p, logits, None, ids, w))
    # the launches go into a CUDA graph so the host's per-call cost does not set the pace
    per_graph = 50
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for _ in range(per_graph):
                B.check(B.moe_grouped_topk(p, logits, None, ids, w))
    torch.cuda.current_stream().wait_stream(side)
    graph.replay()
    reps = max(steps // per_graph, 4)
    n = reps * per_graph
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record()
    for _ in range(reps):
        graph.replay()
    e.record()
    torch.cuda.synchronize()
    us = s.elapsed_time(e) * 1e3 / n
    del graph
    return {"metric": "GroupedTopK latency (83 tokens, 256 experts, 8x32 groups, keep 4, top-8)",
            "value": us, "unit": "us/call", "higher_is_better": False, "steps": n,
            "warmup": warmup, "n_gpus": 1, "dtype": "f32",
            "config": {"workload": wl.name}, "gpu_launches": n}


def run_micro_grouped_topk(args):
    print(json.dumps(micro_grouped_topk_record(args.steps, args.warmup)), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="dsv3_prefill", choices=sorted(W.ALL) + sorted(W.PROFILE) + sorted(W.FP4))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="time only --workload (no per-config records of the other workloads)")
    ap.add_argument("--fused-combine", action="store_true",
                    help="down projection adds into the output with fp32 atomics (non-deterministic)")
    ap.add_argument("--block-m", type=int, default=0, choices=[0, 128, 256],
                    help="bucket alignment: 256 selects the two-SM (cta_group::2) GEMM tiles")
    ap.add_argument("--masked-cap", type=int, default=0,
                    help="masked bucket layout: expert e owns rows [e*cap, (e+1)*cap) (multiple of 128)")
    ap.add_argument("--micro", choices=["grouped_topk"], default=None,
                    help="time one stage alone instead of the layer")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.micro == "grouped_topk":
        run_micro_grouped_topk(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
