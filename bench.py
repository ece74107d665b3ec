#!/usr/bin/env python
"""Benchmark of the TT-gather training step on B200 (one process per GPU).

A step is the whole hot path over one batch: index validation and key
extraction, radix sort, unique + prefix grouping, the fused gather with
in-kernel pooling, the backward into the cores and the SGD update.  The
default workload is the 26-table, rank-64 training step at batch 32768
(pooling Poisson(20)+1, Zipf(1.1) indices); ``--config`` picks another of the
five workloads.  Inputs (indices 143 MB, upstream gradient 436 MB, cores
221 MB) are larger than the 126 MB L2, so no flush is needed between steps.

Prints ONE JSON line on rank 0.  ``--impl reference`` times the fp64 CPU
oracle instead, on a bounded sample of the same workload.
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
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "pooled TT lookups/sec fwd and fwd+bwd at batch 32768; % of roofline"
# FP32 FFMA peak, derived from the unit counts and the maximum SM clock (148 SMs x 128 FP32
# lanes x 2 flops x 1.965 GHz): the kernels are bound by plain FP32 arithmetic, for which no
# measured peak is recorded.
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# used only when MEASURED_PEAKS.json (written per machine next to this file) is absent
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def _find_number(obj, names):
    """First numeric value stored under one of `names` anywhere in a nested JSON object."""
    if isinstance(obj, dict):
        for n in names:
            v = obj.get(n)
            if isinstance(v, (int, float)) and not isinstance(v, bool):
                return float(v)
        for v in obj.values():
            x = _find_number(v, names)
            if x is not None:
                return x
    elif isinstance(obj, list):
        for v in obj:
            x = _find_number(v, names)
            if x is not None:
                return x
    return None


def measured_peaks():
    """HBM copy bandwidth (GB/s) and dense bf16 GEMM throughput (TF/s, burst) of this machine's
    B200, from MEASURED_PEAKS.json when present; otherwise the fallback figures."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    data = None
    if os.path.exists(path):
        try:
            data = json.load(open(path))
        except (OSError, ValueError):
            data = None
    hbm = _find_number(data, ("hbm_gbs",)) if data is not None else None
    bf16 = _find_number(data, ("bf16_tflops",)) if data is not None else None
    return {"hbm_gbs": hbm if hbm else FALLBACK_HBM_GBS,
            "hbm_source": "of measured (MEASURED_PEAKS.json hbm_gbs)" if hbm else "of fallback",
            "bf16_tflops": bf16 if bf16 else FALLBACK_BF16_TFLOPS,
            "bf16_source": "of measured (MEASURED_PEAKS.json bf16_tflops, burst)" if bf16 else "of fallback"}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--config", type=int, default=4)
    p.add_argument("--batch", type=int, default=None, help="smaller batch (profiling runs)")
    p.add_argument("--tables", type=int, default=None, help="fewer tables (profiling runs)")
    p.add_argument("--sched", choices=["static", "steal", "steal_l2"], default="steal_l2",
                   help="work distribution of the fused kernels (ablation)")
    p.add_argument("--grouping", choices=["prefix", "unique"], default="prefix",
                   help="prefix reuse, or one unit per unique row (ablation)")
    p.add_argument("--precision", choices=["auto", "fp32", "split", "bf16"], default="auto",
                   help="prefix-level products: fp32 on the FP32 pipes; split = fp32-accurate on the "
                        "tcgen05 tensor cores (two bf16 terms per value, three products); bf16 on the "
                        "tensor cores; auto = split where the shape has tensor-core kernels, else fp32")
    p.add_argument("--generic", action="store_true",
                   help="force the shape-generic kernels (comparison and profiling runs)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra-fwd", action="store_true",
                   help="skip the forward of the 26-table rank-32 workload that the default run adds")
    p.add_argument("--cpu-seconds", type=float, default=15.0,
                   help="target CPU time of the oracle sample")
    return p.parse_args()


# ---------------------------------------------------------------------------
# workload arithmetic (counts only; the TT arithmetic runs in the kernels)
# ---------------------------------------------------------------------------
def macs_per_prefix(d, r):
    """MACs of the shared prefix chain of one group (first k-1 slices)."""
    k, rows, m = len(d), d[0], 0
    for j in range(1, k - 1):
        m += rows * r[j] * d[j] * r[j + 1]
        rows *= d[j]
    return m


def macs_per_suffix(d, r):
    k = len(d)
    return int(np.prod(d[:-1])) * r[k - 1] * d[k - 1]


def algorithmic(w, U, G):
    """Algorithmic FLOPs (the method's own work, recomputation not counted) and compulsory bytes.

    Three cores: each prefix group contracts its shared slices once (M_p MACs)
    and each distinct row its last slice (M_s).  Four cores run on the merged
    first core G_12 = G_1 . G_2, built once for every (i_1, i_2): the shared
    work is then n_1 n_2 d_1 r_1 d_2 r_2 MACs per table plus the remaining
    prefix step per group (multi-level prefix reuse)."""
    d, r = w.d, w.r
    L, D, T, B = w.num_lookups, w.dim, w.num_tables, w.batch
    Ms = macs_per_suffix(d, r)
    if len(d) == 4:
        pairs = sum(n[0] * n[1] for n in w.n)
        m12 = pairs * d[0] * r[1] * d[1] * r[2]
        Mp = d[0] * d[1] * r[2] * d[2] * r[3]
        shared = m12 + G * Mp
    else:
        Mp = macs_per_prefix(d, r)
        shared = G * Mp
    f_fwd = 2.0 * (shared + U * Ms) + L * D
    f_bwd_kernel = 2.0 * (2 * U * Ms + 2 * shared)
    f_bwd = f_bwd_kernel + L * D
    core_bytes = 4.0 * sum(c.size for tab in w.cores for c in tab)
    io = 8.0 * L + 8.0 * (T * B + 1)
    out_bytes = 4.0 * B * T * D
    b_fwd = io + out_bytes + core_bytes
    b_train = b_fwd + out_bytes + core_bytes + 3 * core_bytes
    return {"f_fwd": f_fwd, "f_bwd": f_bwd, "f_bwd_kernel": f_bwd_kernel, "f_sgd": 2.0 * core_bytes / 4,
            "f_fwd_prefix": 2.0 * shared,
            "b_fwd": b_fwd, "b_train": b_train, "b_rowsum": out_bytes + 4.0 * U * D, "Mp": Mp, "Ms": Ms}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and throttle reasons sampled during the timed region.

    NVML is polled from a thread every 10 ms (the timed region of a default run lasts well
    under a second, too short for nvidia-smi's 200 ms period); nvidia-smi is the fallback."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None
        self.thread = None
        self.samples = []
        self.stop_flag = threading.Event()
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            p = torch.cuda.get_device_properties(self.idx)
            bus = "%08x:%02x:%02x.0" % (p.pci_domain_id, p.pci_bus_id, p.pci_device_id)
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.idx)

    def _poll(self, nv, h):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop_flag.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), smax, int(get_reasons(h))))
            except Exception:
                break
            time.sleep(0.01)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            self.thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
            self.thread.start()
            self.source = "nvml, 10 ms"
            time.sleep(0.05)
            return
        except Exception:
            self.thread = None
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi, 50 ms"
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            rows = self.samples
            if not rows:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
            reasons = sorted({name for _, _, bits in rows for b, name in self.REASONS.items() if bits & b})
            return {"sm_mhz": statistics.median(float(r[0]) for r in rows),
                    "sm_max_mhz": float(max(r[1] for r in rows)), "reasons": reasons,
                    "samples": len(rows), "source": self.source}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": self.source}
        sm = [float(x[0]) for x in rows if x[0].replace(".", "").isdigit()]
        mx = [float(x[1]) for x in rows if x[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for x in rows for i in range(4) if x[4 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "source": self.source}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_init(n, backend=None):
    """Joins the process group of a torchrun launch (NCCL on GPUs; gloo when torch has no
    CUDA device, which the CPU tests use).  Returns (world, rank, local rank)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cuda = torch.cuda.is_available()
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or ("nccl" if cuda else "gloo")
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300), **kw)
    elif cuda:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, x):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_teardown(world):
    """Last collective step of every rank: a barrier, then the process group is destroyed once."""
    if world > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.barrier()
            dist.destroy_process_group()


def kernel_traffic(name, precision, config, lookups):
    """Per-launch DRAM bytes of a fused kernel from a committed single-kernel ncu capture
    (profiles/ncu_traffic.json), taken on a smaller batch of the same workload and the same
    kernel variant (precision mode) with the current kernel source, scaled to this launch by
    the number of lookups it processes; None when no such capture exists."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    try:
        rec = json.load(open(path)).get(name)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("precision", "fp32") != precision or rec.get("config") != config:
        return None
    src = os.path.join(ROOT, "tensor_train_compressed_mixed_b200", "csrc", rec["source"])
    if not os.path.exists(src):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if sha != rec.get("source_sha") or not rec.get("lookups"):
        return None
    return rec["dram_bytes_per_launch"] * lookups / rec["lookups"]


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample (the reported CPU baseline / reference arm)
# ---------------------------------------------------------------------------
def oracle_step(w_sample, threads):
    import oracle
    t0 = time.perf_counter()
    oracle.workload_forward(w_sample, threads=threads)
    grads = oracle.workload_backward(w_sample, threads=threads) if w_sample.grad_out is not None else None
    if grads is not None:
        oracle.sgd(w_sample.cores, grads, w_sample.lr)
    return time.perf_counter() - t0


def cpu_sample(w, target_s, threads):
    """Pick the number of samples whose oracle step takes about target_s seconds.

    Small probes underuse the thread pool, so the probe grows geometrically until
    it takes a quarter of the target, and the last probe's rate is extrapolated."""
    from workloads import sub_batch
    S = 1
    while True:
        t = oracle_step(sub_batch(w, np.arange(S)), threads)
        if t >= 0.25 * target_s or S >= w.batch:
            break
        S = min(w.batch, int(S * min(16.0, max(2.0, 0.3 * target_s / max(t, 1e-3)))))
    S = int(max(1, min(w.batch, S * target_s / max(t, 1e-6))))
    return sub_batch(w, np.arange(S)), S


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from workloads import config_workload
    w = config_workload(args.config, batch=args.batch, tables=args.tables, with_grad=True)
    threads = len(os.sched_getaffinity(0))
    per_step = max(0.5, min(6.0, 150.0 / max(args.steps + args.warmup, 1)))
    sample, S = cpu_sample(w, per_step, threads)
    for _ in range(args.warmup):
        oracle_step(sample, threads)
    total = 0.0
    for _ in range(args.steps):
        total += oracle_step(sample, threads)
    v = sample.num_lookups * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "lookups/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "tables": w.num_tables,
                   "sample_samples": S, "step": "fwd+bwd+sgd" if w.grad_out is not None else "fwd"},
        "cpu_baseline": {"value": v, "unit": "lookups/s", "cores": threads, "kind": "oracle",
                         "sample": f"first {S} of {w.batch} samples, all {w.num_tables} tables "
                                   f"({sample.num_lookups} lookups) per step"},
        "e2e": {"value": v, "unit": "lookups/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------


def kernel_roofline(kernel, ms, alg, precision, w, peaks, config):
    """Roofline record of one fused kernel from its per-launch device time `ms`.

    The fused kernels are bound by arithmetic.  Where part of a kernel's algorithmic work
    runs on the tensor cores (the prefix-level products in the bf16 and split modes), the
    peak is the work-weighted combination of the two pipes: ideal time = F_tc x products /
    P_bf16 + F_fp32 / P_fp32, three tensor-core products per algorithmic one in split mode."""
    flops = {"fwd_fused": alg["f_fwd"], "bwd_fused": alg["f_bwd_kernel"]}
    tc_work = {}
    if precision in ("bf16", "split"):
        tc_work["fwd_fused"] = alg["f_fwd_prefix"]
        if len(w.d) == 3 and w.r[1] == 64:
            tc_work["bwd_fused"] = 2.0 * alg["f_fwd_prefix"]
    traffic = kernel_traffic(kernel, precision, config, w.num_lookups)
    p_bf16 = peaks["bf16_tflops"]
    if kernel in tc_work:
        f_all = flops[kernel]
        f_tc = tc_work[kernel]
        f_rest = f_all - f_tc
        products = 3 if precision == "split" else 1
        t_ideal = products * f_tc / (p_bf16 * 1e12) + f_rest / (FP32_PEAK_TFLOPS * 1e12)
        peak = f_all / t_ideal / 1e12
        achieved = f_all / (ms / 1e3) / 1e12
        return {"bound": "alu", "kernel": kernel, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic,
                "peak_source": f"work-weighted: {f_tc / 1e9:.1f} GFLOP of prefix-level products as {products} "
                               f"bf16 tensor-core product(s) each at the bf16 peak {p_bf16:.0f} TF/s "
                               f"{peaks['bf16_source']}, {f_rest / 1e9:.1f} GFLOP at the FP32 peak "
                               f"{FP32_PEAK_TFLOPS:.1f} TF/s derived from 148 SM x 128 lanes x 2 x 1.965 GHz"}
    if kernel in flops:
        achieved = flops[kernel] / (ms / 1e3) / 1e12
        return {"bound": "alu", "kernel": kernel, "achieved": achieved, "peak": FP32_PEAK_TFLOPS,
                "unit": "TFLOP/s", "frac": achieved / FP32_PEAK_TFLOPS, "traffic": traffic,
                "peak_source": "derived: 148 SM x 128 FP32 lanes x 2 x 1.965 GHz"}
    byts = {"bwd_rowsum": alg["b_rowsum"], "sgd": alg["b_train"] - alg["b_fwd"]}.get(kernel)
    ach = byts / (ms / 1e3) / 1e9 if byts else None
    hbm = peaks["hbm_gbs"]
    return {"bound": "hbm", "kernel": kernel, "achieved": ach, "peak": hbm, "unit": "GB/s",
            "frac": ach / hbm if ach else None, "traffic": traffic,
            "peak_source": f"HBM copy bandwidth {peaks['hbm_source']}"}


def balance_report(records, cap):
    """Per fused kernel: busy time per SM (block start to end, minus time in bounded waits),
    its max and mean over SMs, and the kernel span, from the probe records of one step."""
    import numpy as np
    r = records.view(2, cap, 4).cpu().numpy().astype(np.int64)
    out = {}
    for slot, name in ((0, "fwd_fused"), (1, "bwd_fused")):
        rec = r[slot]
        rec = rec[rec[:, 1] > 0]
        if rec.size == 0:
            continue
        sm = rec[:, 0] & 0xffff
        ckpt = (rec[:, 0] >> 16) & 0xffff
        tasks = rec[:, 0] >> 32
        busy = rec[:, 2] - rec[:, 1] - rec[:, 3]
        per_sm = {}
        for s_, b_ in zip(sm.tolist(), busy.tolist()):
            per_sm[s_] = per_sm.get(s_, 0) + b_
        v = np.array(list(per_sm.values()), dtype=np.float64) / 1e6
        out[name] = {"blocks": int(rec.shape[0]), "sms": int(len(per_sm)),
                     "span_ms": float(rec[:, 2].max() - rec[:, 1].min()) / 1e6,
                     "busy_max_ms": float(v.max()), "busy_mean_ms": float(v.mean()),
                     "max_over_mean": float(v.max() / v.mean()) if v.mean() > 0 else None,
                     "wait_mean_ms": float(rec[:, 3].mean()) / 1e6,
                     "tasks_max": int(tasks.max()), "tasks_mean": float(tasks.mean()),
                     "checkpoint_loads": int(ckpt.sum())}
    return out


def time_rank32_forward(args, world, rank, dev, peaks, barrier_fn, max_fn):
    """Forward pass of the 26-table, rank-32, batch-32768 workload on its own handle, timed
    like the main step (CUDA events, max over ranks), with the fused kernel's roofline."""
    import torch
    from tensor_train_compressed_mixed_b200 import abi, from_workload
    from workloads import config_workload
    w3 = config_workload(3, with_grad=False, shard=rank)
    opts = abi.tt_emb_default_options()
    opts.precision = abi.TT_PREC_FP32_SPLIT_TC
    emb3, cores3, idx3, off3 = from_workload(w3, device=dev, options=opts, with_grads=False)
    out3 = torch.empty(w3.batch, w3.num_tables * w3.dim, dtype=torch.float32, device=dev)
    emb3.reserve(w3.num_lookups, w3.batch)
    for _ in range(args.warmup):
        emb3.forward(idx3, off3, w3.batch, out3)
    emb3.sync()
    seg = emb3.segmentation()
    alg3 = algorithmic(w3, seg["num_unique"], seg["num_groups"])
    abi.tt_emb_enable_timing(emb3.handle, True)
    barrier_fn(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        emb3.forward(idx3, off3, w3.batch, out3)
    e1.record()
    torch.cuda.synchronize()
    emb3.sync()
    barrier_fn(world)
    ms = max_fn(world, e0.elapsed_time(e1)) / args.steps
    ph, _ = abi.tt_emb_phase_times(emb3.handle)
    abi.tt_emb_enable_timing(emb3.handle, False)
    fused_ms = ph["fwd_fused"] / args.steps
    t_roof = max(alg3["f_fwd"] / (FP32_PEAK_TFLOPS * 1e12), alg3["b_fwd"] / (peaks["hbm_gbs"] * 1e9))
    rec = {"workload": w3.name, "precision": "split", "lookups": w3.num_lookups,
           "value": world * w3.num_lookups / (ms / 1e3), "unit": "lookups/s", "ms": ms,
           "roofline_frac": t_roof / (ms / 1e3), "phases_ms": {k: v / args.steps for k, v in ph.items() if v},
           "fused_roofline": kernel_roofline("fwd_fused", fused_ms, alg3, "split", w3, peaks, 3)}
    emb3.close()
    del cores3, idx3, off3, out3
    torch.cuda.empty_cache()
    return rec


def run_ours(args):
    import torch
    from tensor_train_compressed_mixed_b200 import abi, dp, from_workload
    from workloads import config_workload

    world, rank, local = dist_init(args.gpus)
    dev = torch.device("cuda", local)
    peaks = measured_peaks()
    # every rank draws its own batch of the same workload (rank 0's is the single-GPU one)
    w = config_workload(args.config, batch=args.batch, tables=args.tables, with_grad=True, shard=rank)
    if args.precision == "auto":
        # the tensor-core kernels cover three cores with d = (4, 4, 8) and r = 32 or 64
        tc_shape = len(w.d) == 3 and tuple(w.d) == (4, 4, 8) and w.r[1] == w.r[2] and w.r[1] in (32, 64)
        args.precision = "split" if tc_shape else "fp32"
    train = w.grad_out is not None and args.config in (4, 5)
    opts = abi.tt_emb_default_options()
    opts.sched = {"static": abi.TT_SCHED_STATIC, "steal": abi.TT_SCHED_STEAL,
                  "steal_l2": abi.TT_SCHED_STEAL_L2}[args.sched]
    opts.grouping = abi.TT_GROUP_PREFIX if args.grouping == "prefix" else abi.TT_GROUP_UNIQUE_ONLY
    opts.precision = {"fp32": abi.TT_PREC_FP32, "split": abi.TT_PREC_FP32_SPLIT_TC,
                      "bf16": abi.TT_PREC_BF16_TC}[args.precision]
    if args.generic:
        opts.force_generic = 1
        opts.precision = abi.TT_PREC_FP32
        args.precision = "fp32"
    # data-parallel training: the core gradients of all ranks are summed (one NCCL
    # all-reduce over a flat buffer) before the SGD step
    dp_train = world > 1 and train
    emb, cores, idx, off = from_workload(w, device=dev, options=opts, with_grads=True, flat_grads=dp_train)
    g = torch.from_numpy(w.grad_out).to(dev)
    L, B, T, D = w.num_lookups, w.batch, w.num_tables, w.dim
    out = torch.empty(B, T * D, dtype=torch.float32, device=dev)
    emb.reserve(L, B)
    ws_bytes = abi.tt_emb_workspace_size(emb.handle, L, B)

    sgd = args.config == 4
    fused_sgd = sgd and not dp_train   # data parallel: the gradients are exchanged before SGD

    def step():
        emb.forward(idx, off, B, out)
        if fused_sgd:
            emb.backward_sgd(g, w.lr)
        elif train:
            emb.backward(g)
            if dp_train:
                dp.allreduce_grads(emb)
            if sgd:
                emb.sgd_update(w.lr)

    def timed(fn, K):
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(K):
            fn()
        e1.record()
        torch.cuda.synchronize()
        emb.sync()
        barrier(world)
        return max_over_ranks(world, e0.elapsed_time(e1))

    for _ in range(args.warmup):
        step()
    emb.sync()
    seg = emb.segmentation()
    U, G = seg["num_unique"], seg["num_groups"]
    alg = algorithmic(w, U, G)

    # --- the timed training steps (phase events on, clocks sampled) ---
    abi.tt_emb_enable_timing(emb.handle, True)
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    ms_total = timed(step, args.steps)
    clk = clocks.stop()
    ph, launches = abi.tt_emb_phase_times(emb.handle)
    abi.tt_emb_enable_timing(emb.handle, False)
    ms_step = ms_total / args.steps
    value = world * L * args.steps / (ms_total / 1e3)

    # --- forward only ---
    ms_fwd = timed(lambda: emb.forward(idx, off, B, out), args.steps) / args.steps

    # --- SM balance: one more step, untimed, with the scheduler probe on ---
    cap = 4096
    probe = torch.zeros(2 * cap * 4, dtype=torch.int64, device=dev)
    abi.tt_emb_set_probe(emb.handle, probe, cap)
    step()
    emb.sync()
    abi.tt_emb_set_probe(emb.handle, None, 0)
    balance = balance_report(probe, cap)

    # --- dominant kernel roofline (device times from the timed region) ---
    per_step = {k: v / args.steps for k, v in ph.items()}
    dom = max(per_step, key=per_step.get)
    roof = kernel_roofline(dom, per_step[dom], alg, args.precision, w, peaks, args.config)
    t_roof_step = max((alg["f_fwd"] + (alg["f_bwd"] if train else 0)) / (FP32_PEAK_TFLOPS * 1e12),
                      (alg["b_train"] if train else alg["b_fwd"]) / (peaks["hbm_gbs"] * 1e9))
    t_roof_fwd = max(alg["f_fwd"] / (FP32_PEAK_TFLOPS * 1e12), alg["b_fwd"] / (peaks["hbm_gbs"] * 1e9))

    # --- end to end through the public API with host buffers ---
    # Every step copies its inputs from pinned host memory and reads its pooled output
    # back.  The copies run on two copy streams, double-buffered, so step i+1's inputs
    # and step i's output cross the host link while the compute stream works.
    e2e = None
    if not args.no_e2e:
        h_idx = torch.from_numpy(w.indices).pin_memory()
        h_off = torch.from_numpy(w.offsets).pin_memory()
        h_g = torch.from_numpy(w.grad_out).pin_memory()
        h_out = [torch.empty(B, T * D, dtype=torch.float32).pin_memory() for _ in range(2)]
        d_idx = [torch.empty_like(idx) for _ in range(2)]
        d_off = [torch.empty_like(off) for _ in range(2)]
        d_g = [torch.empty_like(g) for _ in range(2)] if train else None
        d_out = [torch.empty_like(out) for _ in range(2)]
        comp = torch.cuda.current_stream(dev)
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]     # a slot's inputs are on the device
        ev_used = [torch.cuda.Event() for _ in range(2)]   # the step using a slot is done
        ev_fwd = [torch.cuda.Event() for _ in range(2)]    # a slot's pooled output is written
        ev_read = [torch.cuda.Event() for _ in range(2)]   # a slot's output is back on the host

        def upload(s):
            up.wait_event(ev_used[s])
            with torch.cuda.stream(up):
                d_idx[s].copy_(h_idx, non_blocking=True)
                d_off[s].copy_(h_off, non_blocking=True)
                if train:
                    d_g[s].copy_(h_g, non_blocking=True)
            ev_in[s].record(up)

        def run_steps(K):
            upload(0)
            for i in range(K):
                s = i % 2
                if i + 1 < K:
                    upload((i + 1) % 2)
                comp.wait_event(ev_in[s])
                comp.wait_event(ev_read[s])
                emb.forward(d_idx[s], d_off[s], B, d_out[s])
                ev_fwd[s].record(comp)
                down.wait_event(ev_fwd[s])
                with torch.cuda.stream(down):
                    h_out[s].copy_(d_out[s], non_blocking=True)
                ev_read[s].record(down)
                if fused_sgd:
                    emb.backward_sgd(d_g[s], w.lr)
                elif train:
                    emb.backward(d_g[s])
                    if dp_train:
                        dp.allreduce_grads(emb)
                    if sgd:
                        emb.sgd_update(w.lr)
                ev_used[s].record(comp)
            for s in range(2):
                comp.wait_event(ev_read[s])

        run_steps(2)
        torch.cuda.synchronize()
        K = max(4, args.steps // 2)
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        up.wait_event(e0)
        down.wait_event(e0)
        run_steps(K)
        e1.record(comp)
        torch.cuda.synchronize()
        emb.sync()
        barrier(world)
        ms_e2e = max_over_ranks(world, e0.elapsed_time(e1)) / K
        h2d = 8 * L + 8 * (T * B + 1) + (4 * B * T * D if train else 0)
        e2e = {"value": world * L / (ms_e2e / 1e3), "unit": "lookups/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": 4 * B * T * D, "ms_per_step": ms_e2e,
               "copies": "pinned host buffers, double-buffered on two copy streams, overlapped with compute"}

    # --- forward of the 26-table rank-32 workload (the forward-only configuration) ---
    extra = None
    if args.config == 4 and args.batch is None and args.tables is None and not args.no_extra_fwd:
        extra = time_rank32_forward(args, world, rank, dev, peaks, barrier, max_over_ranks)

    mem = {"workspace_bytes": ws_bytes,
           "core_bytes": int(sum(c.numel() for tab in cores for c in tab) * 4),
           "peak_allocated_bytes": int(torch.cuda.max_memory_allocated(dev)),
           "note": "workspace sized by tt_emb_workspace_size for this batch; peak over the whole run, "
                   "inputs, outputs, cores and gradients included"}

    # --- CPU oracle on a bounded sample (rank 0, one GPU only) ---
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        threads = len(os.sched_getaffinity(0))
        sample, S = cpu_sample(w, args.cpu_seconds, threads)
        sec = oracle_step(sample, threads)
        cpu = {"value": sample.num_lookups / sec, "unit": "lookups/s", "cores": threads,
               "kind": "oracle",
               "sample": f"first {S} of {B} samples, all {T} tables ({sample.num_lookups} lookups), "
                         f"fwd+bwd+sgd in fp64, {sec:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "lookups/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": {"fp32": "f32", "split": "f32 (prefix-level products as split bf16 on tensor cores)",
                      "bf16": "bf16 prefix-level products, f32 elsewhere"}[args.precision],
            "data": "synthetic",
            "config": {"workload": w.name, "batch": B, "tables": T, "lookups": L,
                       "unique_rows": U, "prefix_groups": G,
                       "step": ("fwd+bwd+sgd (fused sparse update of the middle cores)" if fused_sgd else
                                "fwd+bwd+sgd" if sgd else "fwd+bwd" if train else "fwd"),
                       "l2": "inputs larger than L2 (indices+grad+cores ~800 MB), no flush",
                       "parallelism": (f"dp{world}: own batch per GPU, NCCL all-reduce of the core gradients"
                                       if dp_train else (f"shards{world}: own batch per GPU, no exchange"
                                                         if world > 1 else "single")),
                       "sched": args.sched, "grouping": args.grouping,
                       "prefix_step": {"fp32": "fp32 FFMA",
                                       "split": "fp32-accurate: two bf16 terms per value, three tcgen05 "
                                                "products, fp32 accumulation",
                                       "bf16": "bf16 operands, fp32 accumulation, tcgen05"}[args.precision]},
            "fwd": {"value": world * L / (ms_fwd / 1e3), "unit": "lookups/s", "ms": ms_fwd,
                    "roofline_frac": t_roof_fwd / (ms_fwd / 1e3)},
            "step_roofline_frac": t_roof_step / (ms_step / 1e3),
            "phases_ms": per_step,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
            "memory": mem,
            "balance": balance,
            "peaks": {"hbm_gbs": peaks["hbm_gbs"], "hbm": peaks["hbm_source"],
                      "bf16_tflops": peaks["bf16_tflops"], "bf16": peaks["bf16_source"],
                      "fp32_tflops": FP32_PEAK_TFLOPS, "fp32": "derived from unit counts and the maximum SM clock"},
        }
        if extra is not None:
            line["fwd_rank32"] = extra
        print(json.dumps(line), flush=True)
    emb.close()
    dist_teardown(world)
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
