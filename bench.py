"""Benchmark: tiled attention forward + backward on B200 (one JSON line).

A step is one pass of the whole hot path over one batch: fa_fwd then fa_bwd
(preprocess, main kernel, dQ convert) on the long-sequence workload
B=2, Hq=Hkv=32, N=8192, D=128, causal, bf16 (inputs of 128 MiB each, larger
than the 126 MB L2, so no L2 flush is needed between steps).  FLOPs follow
the matmul convention: fwd 4*B*H*N^2*D, bwd 10*B*H*N^2*D, causal halved.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long]
  python bench.py --impl reference ...   # the fp64 CPU oracle as the reference arm

Multi-GPU (torchrun, one rank per GPU): each rank solves its own independent
problem of the same size (weak scaling, no data-path collective); the timed
region is bracketed by barriers and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd/bwd TFLOP/s on 1 B200 and % of dense BF16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.window = None   # host wall-clock (start, end) of the timed region

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            if self.window is not None:
                try:   # keep only the samples taken inside the timed region
                    ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    ts = None
                if ts is not None and not self.window[0] <= ts <= self.window[1]:
                    continue
            try:
                sm.append(float(f[2]))
                mx = float(f[3])
            except ValueError:
                continue
            for n, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


class NvmlClockSampler:
    """SM clock and clock-event reasons read through NVML every `period_s` from a
    background thread (read-only queries; nothing on the GPU is changed).  A
    20-step timed region lasts about 0.1 s, too short for nvidia-smi's
    100 ms loop, so this is the sampler the bench uses where NVML loads;
    ClockSampler (nvidia-smi) is the fallback.  `nvml` may be a stand-in
    module (tests)."""
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}

    def __init__(self, pci_bus_id: str | None = None, index: int = 0, period_s: float = 0.005, nvml=None):
        self.bus, self.index, self.period = pci_bus_id, index, period_s
        self.nv = nvml
        self.samples = []    # (host time, SM MHz, reason bits)
        self.window = None
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def start(self) -> bool:
        try:
            if self.nv is None:
                import pynvml
                self.nv = pynvml
            nv = self.nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByPciBusId(self.bus) if self.bus else nv.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:   # no NVML, no device: the caller falls back to nvidia-smi
            return False

        def run():
            while not self._stop.is_set():
                try:
                    self.samples.append((time.time(), float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                         int(reasons(h))))
                except Exception:
                    return
                self._stop.wait(self.period)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()
        return True

    def stop(self):
        if self._thread is None:
            return None
        self._stop.set()
        self._thread.join(timeout=5)
        try:
            self.nv.nvmlShutdown()
        except Exception:
            pass
        got = [s for s in self.samples if self.window is None or self.window[0] <= s[0] <= self.window[1]]
        if not got:
            return None
        bits = 0
        for s in got:
            bits |= s[2]
        return {"sm_mhz": statistics.median(s[1] for s in got), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(n for n, b in self.REASON_BITS.items() if bits & b), "samples": len(got),
                "source": f"nvml every {self.period * 1e3:.0f} ms"}


# ----------------------------------------------------------------------------- traffic record
# Sources that decide what each kernel reads and writes: its own file plus
# the launch configuration (API layer) and the shared headers.
COMMON_SOURCES = ("fa_api.cu", "sm100.cuh", "fa_internal.h")
KERNEL_FILES = {
    "fa_fwd_kernel": ("fa_fwd.cu",),
    "fa_fwd_pair_kernel": ("fa_fwd_pair.cu",),
    "fa_fwd_fp8_kernel": ("fa_fwd_fp8.cu",),
    "fa_bwd_dkdv_kernel": ("fa_bwd_split.cu", "fa_bwd.cu"),
    "fa_bwd_dkdv_pair_kernel": ("fa_bwd_pair.cu", "fa_bwd.cu"),
    "fa_bwd_dq_pair_kernel": ("fa_bwd_pair.cu", "fa_bwd.cu"),
    "fa_bwd_dq_kernel": ("fa_bwd_split.cu", "fa_bwd.cu"),
    "fa_bwd_kernel": ("fa_bwd.cu",),
    "fa_bwd_fused_kernel": ("fa_bwd_fused.cu", "fa_bwd.cu"),
    "fa_bwd_preprocess": ("fa_bwd.cu",),
    "fa_decode_split_kernel": ("fa_decode.cu",),
    "fa_decode_combine_kernel": ("fa_decode.cu",),
}
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "dram_traffic.json")


def kernel_source_hash(kernel: str) -> str:
    """sha256 prefix over the sources of `kernel` (its file and the common ones)."""
    h = hashlib.sha256()
    for f in KERNEL_FILES.get(kernel, ()) + COMMON_SOURCES:
        with open(os.path.join(ROOT, "tiled_attention_16_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch from the committed ncu record
    (profiles/dram_traffic.json), or None when there is none for this kernel
    and workload or it was taken on other kernel sources."""
    try:
        with open(TRAFFIC_RECORD) as f:
            entries = json.load(f)["entries"]
    except (OSError, ValueError, KeyError):
        return None
    src = kernel_source_hash(kernel)
    for e in entries:
        if e.get("kernel") == kernel and e.get("workload") == workload and e.get("source_hash") == src:
            return int(e["read_bytes"]) + int(e["write_bytes"])
    return None


# ----------------------------------------------------------------------------- CPU oracle
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"] or [1])
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


def oracle_sample(wl, heads: int):
    """fp64 oracle forward + backward on `heads` (b, h) heads of the workload.
    Returns (seconds, flops counted with the same convention, threads)."""
    import oracle
    from tiled_attention_16_b200.workloads import make_inputs
    q, k, v, do = make_inputs(wl.with_(B=1, Hq=heads, Hkv=heads))
    sc = wl.softmax_scale
    t0 = time.perf_counter()
    oracle.attention_forward(q, k, v, sc, wl.causal)
    oracle.attention_backward(q, k, v, do, sc, wl.causal)
    dt = time.perf_counter() - t0
    per_head = (wl.flops_fwd() + wl.flops_bwd()) / (wl.B * wl.Hq)
    return dt, per_head * heads, blas_threads()


def reference_step_sample(wl, q, k, v, do, rows):
    """One reference step: the oracle's forward and backward terms of a
    strided sample of query rows of one head (rows spread evenly over the
    sequence, so their causal cost averages like the whole head's)."""
    import oracle
    t0 = time.perf_counter()
    oracle.attention_rows_fwd_bwd(q, k, v, do, wl.softmax_scale, wl.causal, 0, 0, rows)
    return time.perf_counter() - t0


def run_reference(args, wl):
    import numpy as np
    from tiled_attention_16_b200.workloads import make_inputs
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    R = min(wl.N, 512)
    stride = wl.N // R
    rows = np.arange(stride // 2, wl.N, stride)[:R]
    q, k, v, do = make_inputs(wl.with_(B=1, Hq=1, Hkv=1))
    for _ in range(args.warmup):
        reference_step_sample(wl, q, k, v, do, rows)
    times = [reference_step_sample(wl, q, k, v, do, rows) for _ in range(args.steps)]
    ms = 1e3 * sum(times) / len(times)
    per_head = (wl.flops_fwd() + wl.flops_bwd()) / (wl.B * wl.Hq)
    flops = per_head * len(rows) / wl.N
    value = flops / (ms * 1e-3) / 1e12
    sample = (f"{len(rows)} of {wl.N} query rows (stride {stride}) of 1 of {wl.B * wl.Hq} heads per step, "
              f"fwd+bwd terms in fp64 (numpy/OpenBLAS)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, ws),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(wl, ws):
    return {"workload": f"{wl.name}: B={wl.B} Hq={wl.Hq} Hkv={wl.Hkv} N={wl.N} D={wl.D} "
                        f"{'causal' if wl.causal else 'non-causal'} bf16 fwd+bwd",
            "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "N": wl.N, "D": wl.D, "causal": wl.causal,
            "scale": wl.softmax_scale, "seed": wl.seed,
            "l2": "inputs larger than L2 (128 MiB per tensor); no flush",
            "parallelism": f"{ws} independent replica(s), one per GPU"}


# ----------------------------------------------------------------------------- ranks
def rank_workload(wl, rank: int):
    """Each rank solves its own independent problem of the same size."""
    return wl.with_(seed=wl.seed + rank)


def max_over_ranks(ms: float, ws: int, device) -> float:
    """Slowest rank's elapsed time (the job time of independent replicas)."""
    if ws <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_step: float, ws: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank's flops over the max-over-ranks step time."""
    return flops_per_step * ws / (ms_per_step * 1e-3) / 1e12


# ----------------------------------------------------------------------------- GPU arm
def run_gpu(args, wl):
    import torch
    import torch.distributed as dist
    from tiled_attention_16_b200 import attention as A
    from tiled_attention_16_b200.build import build
    from tiled_attention_16_b200.workloads import WORKLOADS, make_inputs

    ws, rank, local = dist_env()
    if ws > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    if rank == 0:
        build()
    if ws > 1:
        dist.barrier()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    # inputs resident in HBM (rank r draws its own problem: seed + r)
    q, k, v, do = (x.to(dev) for x in make_inputs(rank_workload(wl, rank)))
    o = torch.empty_like(q)
    lse = torch.empty((wl.B, wl.Hq, wl.N), device=dev, dtype=torch.float32)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsb = torch.empty(A.workspace_bytes(wl.B, wl.Hq, wl.Hkv, wl.N, wl.D), device=dev, dtype=torch.uint8)

    def step():
        A.fwd(q, k, v, causal=wl.causal, out=o, lse=lse)
        A.bwd(q, k, v, o, do, lse, causal=wl.causal, dq=dq, dk=dk, dv=dv, workspace=wsb)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if A.device_status(dev) != A.FA_OK:
        raise RuntimeError(f"device status not OK after warm-up (sites {A.timeout_sites():#x})")

    props = torch.cuda.get_device_properties(dev)
    sampler = NvmlClockSampler(f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0")
    if not sampler.start():
        sampler = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else 0)
        sampler.start()
        time.sleep(0.3)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    A.profile_begin()
    t_start = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    sampler.mark(t_start, time.time())
    per_kernel = A.profile_end()
    if ws > 1:
        dist.barrier()
    clocks = sampler.stop()
    if A.device_status(dev) != A.FA_OK:
        raise RuntimeError(f"device status not OK after timing (sites {A.timeout_sites():#x})")
    ms_total = max_over_ranks(e0.elapsed_time(e1), ws, dev)
    ms = ms_total / args.steps
    flops_step = wl.flops_fwd() + wl.flops_bwd()
    value = job_tflops(flops_step, ws, ms)

    # kernel-level numbers from the live events
    kms = {k: (t / n if n else None) for k, (t, n) in per_kernel.items()}
    fwd_kinds = ("fa_fwd_kernel", "fa_fwd_pair_kernel")
    fwd_kernel = max(fwd_kinds, key=lambda k: kms[k] or 0.0)   # the forward kernel the step ran
    fwd_ms = kms[fwd_kernel]
    bwd_ms = sum(x for k, x in kms.items() if k not in fwd_kinds and x)
    peaks, peak_src = load_peaks()
    peak_tf = peaks["bf16_tflops"]
    # GEMM flops each tensor kernel executes (one "GEMM" over a head = 2*N^2*D,
    # halved when causal): fused backward 5, dK/dV kernel 4 (S, dP, dV, dK),
    # dQ kernel 3 (S and dP recomputed, dQ).
    gemm = wl.flops_fwd() / 2
    kernel_flops = {"fa_fwd_kernel": 2 * gemm, "fa_fwd_pair_kernel": 2 * gemm, "fa_bwd_kernel": 5 * gemm,
                    "fa_bwd_fused_kernel": 5 * gemm,
                    "fa_bwd_dkdv_kernel": 4 * gemm, "fa_bwd_dkdv_pair_kernel": 4 * gemm, "fa_bwd_dq_kernel": 3 * gemm,
                    "fa_bwd_dq_pair_kernel": 3 * gemm}
    tensor_k = {k: v for k, v in kms.items() if v and k in kernel_flops}
    dominant = max(tensor_k, key=lambda k: tensor_k[k])
    achieved = kernel_flops[dominant] / (tensor_k[dominant] * 1e-3) / 1e12
    roofline = {"kernel": dominant, "bound": "tensor", "achieved": achieved, "peak": peak_tf,
                "unit": "TFLOP/s", "frac": achieved / peak_tf, "traffic": recorded_traffic(dominant, wl.name),
                "peak_source": f"{peak_src} bf16_tflops (burst)", "per_launch_ms": tensor_k[dominant],
                "frac_of_sustained_peak": (achieved / peaks["bf16_tflops_sustained"]
                                           if peaks.get("bf16_tflops_sustained") else None),
                "flops_per_launch": kernel_flops[dominant]}
    fwd_tf = wl.flops_fwd() / (fwd_ms * 1e-3) / 1e12
    bwd_tf = wl.flops_bwd() / (bwd_ms * 1e-3) / 1e12
    pre_zero = wl.B * wl.Hq * wl.N * wl.D * 4 if (kms.get("fa_bwd_kernel") or kms.get("fa_bwd_fused_kernel")) else 0
    pre_bytes = wl.B * wl.Hq * wl.N * (2 * wl.D * 2 + 4 + 8) + pre_zero
    conv_bytes = wl.B * wl.Hq * wl.N * wl.D * (4 + 2)
    breakdown = {
        "fwd_ms": fwd_ms, "fwd_tflops": fwd_tf, "fwd_frac_of_peak": fwd_tf / peak_tf,
        "bwd_ms": bwd_ms, "bwd_tflops": bwd_tf, "bwd_frac_of_peak": bwd_tf / peak_tf,
        "bwd_mode": ("separate dQ pass" if (kms.get("fa_bwd_dq_kernel") or kms.get("fa_bwd_dq_pair_kernel"))
                     else "fused (fp32 dQ reductions)"),
        "fwd_kernel": fwd_kernel,
        "bwd_kernels_ms": {k: v for k, v in kms.items() if v and k not in fwd_kinds},
        "bwd_preprocess_gbs": pre_bytes / (kms["fa_bwd_preprocess"] * 1e-3) / 1e9 if kms["fa_bwd_preprocess"] else None,
        "bwd_dq_convert_gbs": conv_bytes / (kms["fa_bwd_dq_convert"] * 1e-3) / 1e9 if kms["fa_bwd_dq_convert"] else None,
        "hbm_peak_gbs": peaks["hbm_gbs"],
    }
    launches = sum(n for _, n in per_kernel.values())

    # FP8 (e4m3) forward on the same workload, timed separately (not part of
    # the step): tensor peak for e4m3 = measured bf16 peak x the nominal 2x ratio
    if not args.no_fp8 and wl.D == 128:
        from tiled_attention_16_b200.workloads import make_fp8_inputs
        q8, k8, v8, qs, ks, vs = make_fp8_inputs(rank_workload(wl, rank))
        q8, k8, v8 = q8.to(dev), k8.to(dev), v8.to(dev)
        o8 = torch.empty_like(o)
        for _ in range(3):
            A.fwd_fp8(q8, k8, v8, qs, ks, vs, causal=wl.causal, out=o8, lse=lse)
        torch.cuda.synchronize()
        A.profile_begin()
        for _ in range(20):
            A.fwd_fp8(q8, k8, v8, qs, ks, vs, causal=wl.causal, out=o8, lse=lse)
        t8, n8 = A.profile_end()["fa_fwd_fp8_kernel"]
        if A.device_status(dev) != A.FA_OK:
            raise RuntimeError("device status not OK after the FP8 forward")
        f8_ms = t8 / n8
        f8_tf = wl.flops_fwd() / (f8_ms * 1e-3) / 1e12
        breakdown["fp8_fwd"] = {"ms": f8_ms, "tflops": f8_tf, "peak": 2 * peak_tf,
                                "frac_of_peak": f8_tf / (2 * peak_tf),
                                "peak_source": f"{peak_src} bf16_tflops (burst) x 2 (nominal e4m3/bf16 ratio)",
                                "launches": n8, "timed_alone": True,
                                "traffic": recorded_traffic("fa_fwd_fp8_kernel", wl.name)}
        del q8, k8, v8, o8

    # decode (split-KV) on its own workload: bound by reading the K/V history
    if not args.no_decode:
        from tiled_attention_16_b200.workloads import KV_WORKLOADS, make_kv_inputs
        kwl = KV_WORKLOADS[args.decode_workload]
        dq_, dk_, dv_ = (x.to(dev) for x in make_kv_inputs(kwl))
        dws = torch.empty(A.decode_workspace_bytes(kwl.B, kwl.Hq, kwl.Hkv, kwl.Nq, kwl.Nk, kwl.D, kwl.causal),
                          device=dev, dtype=torch.uint8)
        do_ = torch.empty_like(dq_)
        dlse = torch.empty((kwl.B, kwl.Hq, kwl.Nq), device=dev, dtype=torch.float32)
        # the whole cache (1 GiB) exceeds L2, so consecutive launches read it from HBM
        for _ in range(3):
            A.decode(dq_, dk_, dv_, causal=kwl.causal, out=do_, lse=dlse, workspace=dws)
        torch.cuda.synchronize()
        A.profile_begin()
        for _ in range(20):
            A.decode(dq_, dk_, dv_, causal=kwl.causal, out=do_, lse=dlse, workspace=dws)
        td, nd = A.profile_end()["fa_decode"]
        if A.device_status(dev) != A.FA_OK:
            raise RuntimeError("device status not OK after decode")
        d_ms = td / nd
        gbs = kwl.kv_bytes() / (d_ms * 1e-3) / 1e9
        breakdown["decode"] = {
            "workload": f"{kwl.name}: B={kwl.B} Hq={kwl.Hq} Hkv={kwl.Hkv} Nq={kwl.Nq} Nk={kwl.Nk} D={kwl.D} causal",
            "ms": d_ms, "bound": "hbm", "algorithmic_bytes": kwl.kv_bytes(), "achieved_gbs": gbs,
            "traffic": recorded_traffic("fa_decode_split_kernel", kwl.name),
            "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"],
            "peak_source": f"{peak_src} hbm_gbs", "launches": nd, "timed_alone": True}
        del dq_, dk_, dv_, dws, do_, dlse

    # context parallel: a ring of --cp-ranks ranks over a long sequence
    # (--cp-workload, zigzag chunks), every rank's pairs run on this one GPU
    # in ring order; the exchange is not timed (it needs more GPUs).  The
    # single-kernel path is timed on the same inputs, so the ratio of the two
    # rates is what chunking, merging and accumulating cost.
    cwl = WORKLOADS[args.cp_workload]
    if not args.no_cp and cwl.N % (2 * args.cp_ranks) == 0:
        from tiled_attention_16_b200 import context_parallel as cp
        R = args.cp_ranks
        cq, ck, cv, cdo = (x.to(dev) for x in make_inputs(rank_workload(cwl, rank)))
        sh = lambda x: [cp.shard_sequence(x, r, R) for r in range(R)]  # noqa: E731
        sq, sk, sv, sdo = sh(cq), sh(ck), sh(cv), sh(cdo)

        def ring_step():
            fw = cp.virtual_ring_fwd(sq, sk, sv, cwl.causal, cwl.softmax_scale)
            cp.virtual_ring_bwd(sq, sk, sv, [f[0] for f in fw], sdo, [f[1] for f in fw], cwl.causal,
                                cwl.softmax_scale)

        cws = torch.empty(A.workspace_bytes(cwl.B, cwl.Hq, cwl.Hkv, cwl.N, cwl.D), device=dev, dtype=torch.uint8)

        def mono_step():
            co, clse = A.fwd(cq, ck, cv, causal=cwl.causal)
            A.bwd(cq, ck, cv, co, cdo, clse, causal=cwl.causal, workspace=cws)

        def timed_once(fn):
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record()
            fn()
            t1.record()
            torch.cuda.synchronize()
            return t0.elapsed_time(t1)

        # Each leg runs ~70 ms, long enough for the power cap to move the SM
        # clock between runs, so the two legs are timed interleaved, in
        # alternating order, and compared by their medians: both see the same
        # power state.
        n_cp = 5
        for _ in range(2):
            mono_step()
            ring_step()
        torch.cuda.synchronize()
        mono_runs, cp_runs = [], []
        for i in range(n_cp):
            legs = [(mono_runs, mono_step), (cp_runs, ring_step)]
            for runs, fn in (legs if i % 2 == 0 else legs[::-1]):
                runs.append(timed_once(fn))
        mono_ms, cp_ms = statistics.median(mono_runs), statistics.median(cp_runs)
        # one more ring step under the per-kernel profiler (launch count, merge
        # and accumulate time), outside the timed runs
        A.profile_begin()
        ring_step()
        cp_kernels = A.profile_end()
        if A.device_status(dev) != A.FA_OK:
            raise RuntimeError("device status not OK after the context-parallel ring")
        cflops = cwl.flops_fwd() + cwl.flops_bwd()
        cp_tf = cflops / (cp_ms * 1e-3) / 1e12
        mono_tf = cflops / (mono_ms * 1e-3) / 1e12
        n_all = 1
        breakdown["context_parallel"] = {
            "workload": f"{cwl.name}: B={cwl.B} Hq={cwl.Hq} Hkv={cwl.Hkv} N={cwl.N} D={cwl.D}"
                        f"{' causal' if cwl.causal else ''}",
            "ranks": R, "chunk_rows": cwl.N // (2 * R), "layout": "zigzag",
            "ms_per_step": cp_ms, "tflops": cp_tf, "single_kernel_ms": mono_ms, "single_kernel_tflops": mono_tf,
            "vs_single_kernel": cp_tf / mono_tf, "timing": f"{n_cp} runs of each leg interleaved in alternating order; medians",
            "runs_ms": {"ring": cp_runs, "single_kernel": mono_runs},
            "merge_ms": cp_kernels["fa_lse_merge_kernel"][0] / n_all,
            "accumulate_ms": cp_kernels["fa_accumulate_kernel"][0] / n_all,
            "launches_per_step": sum(nn for _, nn in cp_kernels.values()) / n_all,
            "exchange": "not timed (one GPU): the ranks run one after another on it", "timed_alone": True}
        del cq, ck, cv, cdo, sq, sk, sv, sdo, cws

    # end to end through the public API with host buffers (pinned), copies timed.
    # Every step copies its inputs host->device and its results device->host;
    # steps are pipelined the way a caller streams batches: two device buffer
    # sets, the input copies on one stream, the attention on another and the
    # result copies on a third, so step i's copies overlap steps i-1 / i+1.
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hdo = (x.pin_memory() for x in make_inputs(rank_workload(wl, rank)))
        ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
        hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
        hdq = torch.empty(dq.shape, dtype=dq.dtype, pin_memory=True)
        hdk = torch.empty(dk.shape, dtype=dk.dtype, pin_memory=True)
        hdv = torch.empty(dv.shape, dtype=dv.dtype, pin_memory=True)
        h_in, h_out = (hq, hk, hv, hdo), (ho, hl, hdq, hdk, hdv)
        h2d = sum(x.numel() * x.element_size() for x in h_in)
        d2h = sum(x.numel() * x.element_size() for x in h_out)
        sets = [((q, k, v, do), (o, lse, dq, dk, dv))]
        sets.append((tuple(torch.empty_like(x) for x in sets[0][0]), tuple(torch.empty_like(x) for x in sets[0][1])))
        s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        computed = [torch.cuda.Event() for _ in range(2)]   # set b's inputs consumed, outputs written
        copied_in = [torch.cuda.Event() for _ in range(2)]
        copied_out = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def e2e_step(i):
            b = i % 2
            (xq, xk, xv, xdo), (xo, xl, xdq, xdk, xdv) = sets[b]
            with torch.cuda.stream(s_in):
                if used[b]:
                    s_in.wait_event(computed[b])
                for d, h in zip((xq, xk, xv, xdo), h_in):
                    d.copy_(h, non_blocking=True)
                copied_in[b].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(copied_in[b])
                if used[b]:
                    s_comp.wait_event(copied_out[b])
                A.fwd(xq, xk, xv, causal=wl.causal, out=xo, lse=xl)
                A.bwd(xq, xk, xv, xo, xdo, xl, causal=wl.causal, dq=xdq, dk=xdk, dv=xdv, workspace=wsb)
                computed[b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(computed[b])
                for h, d in zip(h_out, (xo, xl, xdq, xdk, xdv)):
                    h.copy_(d, non_blocking=True)
                copied_out[b].record(s_out)
            used[b] = True

        e2e_steps = max(3, min(args.steps, 20))
        torch.cuda.synchronize()   # earlier work on the default stream still reads set 0
        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(s_in)
        for i in range(e2e_steps):
            e2e_step(i)
        for st in (s_in, s_comp):
            s_out.wait_stream(st)
        a1.record(s_out)
        torch.cuda.synchronize()
        if A.device_status(dev) != A.FA_OK:
            raise RuntimeError("device status not OK after the end-to-end steps")
        e_ms = max_over_ranks(a0.elapsed_time(a1), ws, dev)
        e2e = {"value": job_tflops(flops_step, ws, e_ms / e2e_steps), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "pipelined": "2 buffer sets; H2D, compute, D2H on separate streams"}
        del sets

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        heads = 4
        dt, fl, threads = oracle_sample(wl, heads)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{heads} of {wl.B * wl.Hq} (b,h) heads, full fwd+bwd in fp64 ({dt:.1f} s)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_of(wl, ws),
            "frac_of_peak": value / ws / peak_tf, "breakdown": breakdown, "roofline": roofline,
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "gpu_launches": launches,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the separate FP8 forward measurement")
    ap.add_argument("--no-decode", action="store_true", help="skip the separate decode (split-KV) measurement")
    ap.add_argument("--no-cp", action="store_true", help="skip the context-parallel (ring) measurement")
    ap.add_argument("--cp-ranks", type=int, default=4, help="ranks of the context-parallel ring measurement")
    ap.add_argument("--cp-workload", default="stress", help="sequence of the context-parallel ring measurement")
    ap.add_argument("--decode-workload", default="decode70b", help="KV-history workload of the decode measurement")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from tiled_attention_16_b200.workloads import WORKLOADS
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_gpu(args, wl)


if __name__ == "__main__":
    sys.exit(main())
