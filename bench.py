#!/usr/bin/env python
"""Benchmark of the block-wise microscaling FP4 hot path on B200.

One step = the whole hot path over one batch of synthetic input: for every
tensor of the workload, the per-tensor amax, the per-tensor scale, the fused
(rotate+)scale+round+pack quantize kernel that also measures the per-block /
per-tensor MSE with its three-term split, and dequantization.  Default workload: NVFP4 (block 16,
UE4M3 block scales, FP32 per-tensor scale amax/(6*448)) on the nine Qwen2.5-7B
MLP weights gate/up 18944x3584 and down 3584x18944 at sigma 0.005/0.02/0.05
(611M elements, 1.22 GB of bf16 per step: larger than L2).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fp4q|reference]

Prints one JSON line (rank 0).  Under torchrun each rank processes its own
copy of the workload (independent tensors, no data-path collective): weak
scaling, timed as the max over ranks of the device time.
"""
from __future__ import annotations

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

METRIC = "G elements/s and achieved HBM GB/s (% of B200 peak) for rotate+FP4 quantize"
SPEC_HBM_GBS = 8000.0
E8, U4, U5 = 0, 1, 2
NONE, COMP, GIVEN, FROM_AMAX = 0, 1, 2, 3


# --------------------------------------------------------------------------- args / dist
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["fp4q", "reference"], default="fp4q")
    ap.add_argument("--workload", default="nvfp4_qwen25_7b_mlp",
                    choices=["nvfp4_qwen25_7b_mlp", "rotated_activations_8192x5120", "mxfp4_gaussian_1024x1024"])
    ap.add_argument("--rot", type=int, default=128, help="rotation for the activation workload")
    ap.add_argument("--fmt", default="nvfp4", choices=["nvfp4", "mxfp4"], help="format for the activation workload")
    ap.add_argument("--e2e-steps", type=int, default=0, help="end-to-end steps (default: max(3, steps // 20))")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU work of the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--separate-mse", action="store_true",
                    help="measure the MSE with its own pass over x (fp4q_quantize + fp4q_block_mse + fp4q_dequantize)")
    ap.add_argument("--separate-dequant", action="store_true",
                    help="dequantize with its own pass over the codes (fp4q_quantize_mse + fp4q_dequantize)")
    ap.add_argument("--scale-search", default=None, metavar="BELOW,ABOVE",
                    help="MSE-optimised block scales: try BELOW codes below and ABOVE codes above the "
                         "max-rule code (fp4q_quantize_search + fp4q_block_mse + fp4q_dequantize)")
    ap.add_argument("--outlier-stats", type=float, default=None, metavar="P",
                    help="add the activation outlier statistics (max, nearest-rank P-quantile of |x|, channel "
                         "maxima: fp4q_outlier_stats) to every tensor of the step")
    args = ap.parse_args(argv)
    args.search = None
    if args.scale_search:
        below, above = (int(v) for v in args.scale_search.split(","))
        args.search = (below, above)
    return args


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def init_dist(world: int, backend: str, device=None):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        kw = dict(backend=backend, timeout=datetime.timedelta(seconds=120))
        if device is not None and backend == "nccl":
            kw["device_id"] = device
        dist.init_process_group(**kw)


def reduce_max(value: float, device) -> float:
    """Max over ranks (identity on one rank): the job is as slow as its slowest GPU."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own tensors (independent problems per GPU)."""
    return int(base) + 1_000_003 * int(rank)


# --------------------------------------------------------------------------- workload
def build_workload(name: str, device, rank: int, args):
    """[(label, x bf16 [rows, cols], fmt, block, rot, gmode)] on `device`."""
    import workloads as W
    out = []
    if name == "nvfp4_qwen25_7b_mlp":
        for si, sigma in enumerate(W.QWEN25_7B_SIGMAS):
            for ti, t in enumerate(W.QWEN25_7B_MLP):
                x = W.gaussian_bf16(t.rows, t.cols, sigma, rank_seed(1000 + 10 * si + ti, rank), device)
                out.append((f"{t.name}_s{sigma}", x, U4, 16, 0, COMP))
    elif name == "rotated_activations_8192x5120":
        x, _ = W.student_t_outliers_bf16(8192, 5120, rank_seed(77, rank), device=device)
        fmt, block = (U4, 16) if args.fmt == "nvfp4" else (E8, 32)
        out.append((f"act_rot{args.rot}", x, fmt, block, args.rot, COMP if fmt == U4 else NONE))
    else:
        x = W.gaussian_bf16(1024, 1024, 0.02, rank_seed(0, rank), device)
        out.append(("w1024", x, E8, 32, 0, NONE))
    return out


def bytes_per_element(block: int):
    """Algorithmic HBM bytes per element of each kernel (reads + writes)."""
    return {
        "amax": 2.0,
        "quantize": 2.0 + 0.5 + 1.0 / block,
        "quantize_search": 2.0 + 0.5 + 1.0 / block,
        "outlier_stats": 2.0,
        "quantize_mse": 2.0 + 0.5 + 1.0 / block + 4.0 / block,
        "quantize_mse_dequantize": 2.0 + 0.5 + 1.0 / block + 4.0 / block + 2.0,
        "dequantize": 0.5 + 1.0 / block + 2.0,
        "block_mse": 2.0 + 0.5 + 1.0 / block + 4.0 / block,
    }


class Pipeline:
    """Device buffers and the per-step launch sequence for a workload.

    The launches go straight to the C ABI with arguments marshalled once, so
    the host enqueues a step in a fraction of the step's device time.  Events
    sit between consecutive calls on the launching stream: the event after
    one kernel is the event before the next.
    """


    def __init__(self, fq, items, device, stream, separate_mse=False, separate_dequant=False, search=None,
                 outlier_p=None):
        import torch
        self.fq, self.items, self.device = fq, items, device
        L = fq.lib()
        sh = stream.cuda_stream
        self.bufs, self.calls = [], []
        # [amax, G] of every tensor in one buffer, cleared by one fill at the start of each step
        self.gs_all = torch.zeros((len(items), 2), dtype=torch.float32, device=device)
        self.any_comp = any(gm == COMP for *_, gm in items)
        separate_mse = separate_mse or search is not None     # the search has no fused MSE pass
        for ti, (label, x, fmt, block, rot, gmode) in enumerate(items):
            rows, cols = x.shape
            b = dict(
                codes=torch.empty((rows, cols // 2), dtype=torch.uint8, device=device),
                scales=torch.empty((rows, cols // block), dtype=torch.uint8, device=device),
                gscale=self.gs_all[ti],                                            # [amax, G]
                deq=torch.empty((rows, cols), dtype=torch.bfloat16, device=device),
                bm=torch.empty((rows, cols // block), dtype=torch.float32, device=device),
                terms=torch.empty((4,), dtype=torch.float64, device=device),
                ws=torch.zeros((fq.fp4q_block_mse_workspace_size(rows, cols, block),), dtype=torch.uint8,
                               device=device),
            )
            self.bufs.append(b)
            if outlier_p is not None:
                b["ostats"] = torch.empty((2,), dtype=torch.float32, device=device)
                b["ocols"] = torch.empty((cols,), dtype=torch.float32, device=device)
                b["ows"] = torch.empty((fq.lib().fp4q_outlier_stats_workspace_size(),), dtype=torch.uint8,
                                       device=device)
            p = {k: v.data_ptr() for k, v in b.items()}
            comp = gmode == COMP
            # per-tensor scale: the amax pass writes gscale[0]; the quantizer derives G from it
            # (FROM_AMAX) and writes it to gscale[1], where dequantize and block MSE read it
            gq = p["gscale"] if comp else None
            g = p["gscale"] + 4 if comp else None
            seq = []
            if outlier_p is not None:
                seq.append(("outlier_stats", L.fp4q_outlier_stats, (x.data_ptr(), rows, cols, float(outlier_p),
                                                                    p["ostats"], p["ocols"], p["ows"],
                                                                    b["ows"].numel(), sh)))
            if comp:
                seq.append(("amax", L.fp4q_tensor_amax_accumulate, (x.data_ptr(), rows, cols, rot, p["gscale"], sh)))
            gm = FROM_AMAX if comp else NONE
            if search is not None:
                seq.append(("quantize_search", L.fp4q_quantize_search,
                            (x.data_ptr(), rows, cols, fmt, block, rot, gm, search[0], search[1], p["codes"],
                             p["scales"], gq, sh)))
                seq.append(("block_mse", L.fp4q_block_mse, (x.data_ptr(), p["codes"], p["scales"], g, rows, cols,
                                                            fmt, block, rot, p["bm"], p["terms"], p["ws"],
                                                            b["ws"].numel(), sh)))
            elif separate_mse:
                seq.append(("quantize", L.fp4q_quantize, (x.data_ptr(), rows, cols, fmt, block, rot, gm,
                                                          p["codes"], p["scales"], gq, sh)))
                seq.append(("block_mse", L.fp4q_block_mse, (x.data_ptr(), p["codes"], p["scales"], g, rows, cols,
                                                            fmt, block, rot, p["bm"], p["terms"], p["ws"],
                                                            b["ws"].numel(), sh)))
            elif separate_dequant:
                seq.append(("quantize_mse", L.fp4q_quantize_mse,
                            (x.data_ptr(), rows, cols, fmt, block, rot, gm, p["codes"], p["scales"], gq, p["bm"],
                             p["terms"], p["ws"], b["ws"].numel(), sh)))
            else:
                # quantize, the MSE split and the dequantized bf16 tensor in one pass over x
                seq.append(("quantize_mse_dequantize", L.fp4q_quantize_mse_dequantize,
                            (x.data_ptr(), rows, cols, fmt, block, rot, gm, p["codes"], p["scales"], gq, p["deq"],
                             p["bm"], p["terms"], p["ws"], b["ws"].numel(), sh)))
            if separate_mse or separate_dequant:
                seq.append(("dequantize", L.fp4q_dequantize, (p["codes"], p["scales"], g, rows, cols, fmt, block, 0,
                                                              0, p["deq"], sh)))
            self.calls.append(seq)
        self.elements = sum(x.numel() for _, x, *_ in items)
        # kernels per step: amax (per-tensor scale), quantize (+MSE, reduced in-kernel, + dequantized output),
        # [block MSE], [dequantize]
        # outlier statistics: one histogram pass and a scan below 2^22 elements; above, a sampled
        # pass, the threshold scan, the main pass, a scan, and a pass and a scan that return at once
        # unless the threshold missed
        self.launches_per_step = sum(1 + (1 if gm == COMP else 0) + (2 if separate_mse else 0)
                                     + (1 if separate_dequant and not separate_mse else 0)
                                     + (0 if outlier_p is None else (6 if x.numel() >= (1 << 22) else 2))
                                     for _, x, *_, gm in items)
        self.events_per_step = 1 + sum(len(seq) for seq in self.calls)

    def step(self, stream, ev=None):
        """Enqueue one step; ev = events_per_step timing events or None."""
        bad = 0
        j = 0
        if ev is not None:
            ev[0].record(stream)
        if self.any_comp:
            self.gs_all.zero_()       # the maxima accumulate from 0
        for seq in self.calls:
            for stage, fn, args in seq:
                bad |= fn(*args)
                if ev is not None:
                    j += 1
                    ev[j].record(stream)
        if bad:
            raise RuntimeError(f"a C-ABI call returned an error status ({bad})")

    def new_events(self):
        import torch
        return [torch.cuda.Event(enable_timing=True) for _ in range(self.events_per_step)]

    def stage_times(self, ev):
        """[(tensor index, stage, ms)] of one step's events."""
        out, j = [], 0
        for i, seq in enumerate(self.calls):
            for stage, _, _ in seq:
                out.append((i, stage, ev[j].elapsed_time(ev[j + 1])))
                j += 1
        return out


# --------------------------------------------------------------------------- clocks
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    """Polls NVML (read-only) every few ms while the timed region runs."""

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nvml = pynvml
            props = torch.cuda.get_device_properties(device_index)
            try:
                bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:          # no NVML: report that instead of clocks
            self.nvml, self.error = None, f"{type(e).__name__}: {e}"

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                self.reasons |= int(self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self):
        if self.nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        reasons = [n for bit, n in _REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# --------------------------------------------------------------------------- measured peaks / traffic
def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def csrc_hash(files=None) -> str:
    """Hash of the named kernel sources (all of csrc/ when files is None)."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "microscaling_fp4_quantization_block_b200", "csrc")
    for f in sorted(files if files is not None else os.listdir(d)):
        with open(os.path.join(d, f), "rb") as fh:
            h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per element of `kernel` from the committed ncu summary, if the
    kernel sources have not changed since it was captured (else None)."""
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            t = json.load(f)
        e = t[workload][kernel]
        if e.get("csrc_sha") != csrc_hash(e.get("csrc_files")):
            return None
        return float(e["dram_bytes_per_element"])
    except Exception:
        return None


# --------------------------------------------------------------------------- CPU baseline (oracle)
def oracle_sample_step(items_cpu, search=None, outlier_p=None):
    """The oracle over host tensors: quantize (max rule, or the scale search),
    dequantize, block MSE."""
    import numpy as np
    import oracle
    n = 0
    for label, xb, fmt, block, rot, gmode in items_cpu:
        rows, cols = xb.shape
        if outlier_p is not None:
            oracle.outlier_stats(xb, outlier_p)
        if search is None:
            codes, scales, G = oracle.quantize(xb, fmt, block, rot, gmode)
        else:
            codes, scales, G = oracle.quantize_search(xb, fmt, block, rot, gmode, 1.0, search[0], search[1])
        oracle.dequantize(codes, scales, G, rows, cols, fmt, block, 0)
        oracle.block_mse(xb, codes, scales, G, fmt, block, rot)
        n += xb.size
    return n


def cpu_sample_items(name: str, args, elements_target: int):
    """A bounded sample of the workload, drawn on the host with the same recipe:
    the first rows of every tensor, about elements_target elements in all."""
    import numpy as np
    import torch
    import workloads as W
    out = []
    if name == "nvfp4_qwen25_7b_mlp":
        per = max(1, elements_target // 9)
        for si, sigma in enumerate(W.QWEN25_7B_SIGMAS):
            for ti, t in enumerate(W.QWEN25_7B_MLP):
                rows = max(1, min(t.rows, per // t.cols))
                x = W.gaussian_bf16(rows, t.cols, sigma, 1000 + 10 * si + ti)
                out.append((t.name, x.view(torch.int16).numpy().view(np.uint16), U4, 16, 0, COMP))
    elif name == "rotated_activations_8192x5120":
        rows = max(1, min(8192, elements_target // 5120))
        x, _ = W.student_t_outliers_bf16(rows, 5120, 77)
        fmt, block = (U4, 16) if args.fmt == "nvfp4" else (E8, 32)
        out.append(("act", x.view(torch.int16).numpy().view(np.uint16), fmt, block, args.rot,
                    COMP if fmt == U4 else NONE))
    else:
        x = W.gaussian_bf16(1024, 1024, 0.02, 0)
        out.append(("w1024", x.view(torch.int16).numpy().view(np.uint16), E8, 32, 0, NONE))
    return out


MAX_ORACLE_PROCS = 32


def _oracle_init():
    import oracle
    oracle.lib()


def _oracle_worker(payload):
    items, search, outlier_p = payload
    return oracle_sample_step(items, search, outlier_p)


def cpu_all_cores(items, args):
    """The same sample split into row ranges over independent oracle processes,
    one per host core (at most MAX_ORACLE_PROCS), started with spawn: wall-clock
    throughput of the oracle as it stands on the whole host."""
    import multiprocessing as mp
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    procs = max(1, min(cores, MAX_ORACLE_PROCS))
    parts = [[] for _ in range(procs)]
    for label, xb, fmt, block, rot, gmode in items:
        rows = xb.shape[0]
        for q in range(procs):
            lo, hi = rows * q // procs, rows * (q + 1) // procs
            if hi > lo:
                parts[q].append((label, xb[lo:hi].copy(), fmt, block, rot, gmode))
    payloads = [(part, args.search, args.outlier_stats) for part in parts]
    # every wait is bounded: a pool whose workers cannot start (for instance when
    # __main__ cannot be re-imported by spawn) raises here instead of hanging
    with mp.get_context("spawn").Pool(procs, initializer=_oracle_init) as pool:
        pool.map_async(_oracle_worker, [([], None, None)] * procs, chunksize=1).get(timeout=120)
        t0 = time.perf_counter()
        n = sum(pool.map_async(_oracle_worker, payloads, chunksize=1).get(timeout=120 + 20 * args.cpu_seconds))
        dt = time.perf_counter() - t0
    return {"value": n / dt / 1e9, "unit": "Gelem/s", "cores": procs, "host_cores": cores,
            "sample": f"the same {n} elements in {procs} row ranges, one oracle process each, {dt:.2f} s wall"}


def cpu_baseline(name, args):
    """Oracle throughput on ~args.cpu_seconds of single-threaded CPU work, and
    the same sample over all host cores in independent processes."""
    probe = cpu_sample_items(name, args, 1_000_000)
    t0 = time.perf_counter()
    n = oracle_sample_step(probe, args.search, args.outlier_stats)
    rate = n / max(time.perf_counter() - t0, 1e-9)
    target = int(min(rate * args.cpu_seconds, 2_000_000_000))
    items = cpu_sample_items(name, args, target)
    t0 = time.perf_counter()
    n = oracle_sample_step(items, args.search, args.outlier_stats)
    dt = time.perf_counter() - t0
    out = {"value": n / dt / 1e9, "unit": "Gelem/s", "cores": 1, "kind": "oracle",
           "sample": f"{n} elements: the first rows of each of the {len(items)} tensors, same recipe, "
                     f"drawn on the host; quantize + dequantize + block MSE, single-threaded C, {dt:.1f} s"}
    try:
        out["all_cores"] = cpu_all_cores(items, args)
    except Exception as e:                      # reported, never fatal to the GPU measurement
        out["all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"}
    return out


# --------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import numpy as np
    per_step = 6_000_000 if args.workload == "nvfp4_qwen25_7b_mlp" else 2_000_000
    items = cpu_sample_items(args.workload, args, per_step)
    for _ in range(args.warmup):
        oracle_sample_step(items, args.search, args.outlier_stats)
    t0 = time.perf_counter()
    n = 0
    for _ in range(args.steps):
        n += oracle_sample_step(items, args.search, args.outlier_stats)
    dt = time.perf_counter() - t0
    value = n / dt / 1e9
    line = {"metric": METRIC, "value": value, "unit": "Gelem/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": args.workload, "elements_per_step": int(n // args.steps),
                       "block_scales": "max rule" if args.search is None else
                                       f"MSE search: max-rule code, {args.search[1]} above, {args.search[0]} below",
                       "outlier_stats": None if args.outlier_stats is None else
                                        f"max, P{100 * args.outlier_stats:g} of |x| and channel maxima per tensor",
                       "note": "the CPU oracle (single-threaded C) on a bounded sample of the workload"},
            "cpu_baseline": {"value": value, "unit": "Gelem/s", "cores": 1, "kind": "oracle",
                             "sample": f"{n // args.steps} elements per step: the first rows of every tensor"},
            "e2e": {"value": value, "unit": "Gelem/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------------------- main (CUDA path)
def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    import torch
    import microscaling_fp4_quantization_block_b200 as fq

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl", device)
    import torch.distributed as dist

    items = build_workload(args.workload, device, rank, args)
    stream = torch.cuda.Stream(device)
    stream.wait_stream(torch.cuda.current_stream())
    pipe = Pipeline(fq, items, device, stream, separate_mse=args.separate_mse,
                    separate_dequant=args.separate_dequant, search=args.search, outlier_p=args.outlier_stats)
    in_l2 = sum(x.numel() * 2 for _, x, *_ in items) < 256 * 2 ** 20
    flush = torch.empty(512 * 2 ** 20, dtype=torch.uint8, device=device) if in_l2 else None

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            pipe.step(stream)
            if flush is not None:
                flush.zero_()
    torch.cuda.synchronize()

    # ---- timed region: K steps with events only at step boundaries (consecutive
    # kernels of a step overlap their launch latency; nothing is recorded between them)
    bounds = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    with sampler, torch.cuda.stream(stream):
        for k in range(args.steps):
            bounds[k][0].record(stream)
            pipe.step(stream)
            bounds[k][1].record(stream)
            if flush is not None:
                flush.zero_()         # between timed steps, outside the step's events
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        local_ms = sum(a.elapsed_time(b) for a, b in bounds)
        total_ms = reduce_max(local_ms, device)

        # ---- per-kernel pass (the same K steps, an event after every C-ABI call on the
        # launching stream): kernel shares and the dominant kernel's achieved bandwidth
        events = [pipe.new_events() for _ in range(args.steps)]
        for k in range(args.steps):
            pipe.step(stream, events[k])
            if flush is not None:
                flush.zero_()
        torch.cuda.synchronize()

    per_kernel = {}
    for k in range(args.steps):
        for i, stage, ms in pipe.stage_times(events[k]):
            per_kernel.setdefault(stage, []).append((i, ms))
    elements_step = pipe.elements
    value = world * elements_step * args.steps / (total_ms / 1e3) / 1e9

    # bytes per step and per-kernel roofline
    peak, peak_kind = measured_peaks()
    kernels = {}
    step_bytes = 0.0
    for stage, lst in per_kernel.items():
        tot_ms = sum(t for _, t in lst)
        byts = 0.0
        for i, t in lst:
            _, x, fmt, block, rot, gmode = items[i]
            byts += bytes_per_element(block).get(stage, 0.0) * x.numel()
        step_bytes += byts / args.steps
        kernels[stage] = {"ms_per_step": tot_ms / args.steps, "share": None,
                          "GB_per_s": (byts / 1e9) / (tot_ms / 1e3) if tot_ms > 0 else None}
    busy = sum(v["ms_per_step"] for v in kernels.values())
    for v in kernels.values():
        v["share"] = v["ms_per_step"] / busy if busy > 0 else None
        v["frac_of_peak"] = (v["GB_per_s"] / peak) if v["GB_per_s"] else None
    dominant = max(kernels, key=lambda s: kernels[s]["ms_per_step"])
    dk = kernels[dominant]
    launches = sum(1 for _ in per_kernel[dominant]) / args.steps
    _, x0, _, block0, _, _ = items[0]
    dom_bpe = bytes_per_element(block0).get(dominant, 0.0)
    tpe = ncu_traffic(dominant, args.workload)
    per_launch_elems = elements_step / max(launches, 1)
    roofline = {"bound": "hbm", "kernel": dominant, "achieved": dk["GB_per_s"], "peak": peak,
                "peak_kind": peak_kind, "unit": "GB/s", "frac": dk["GB_per_s"] / peak,
                "traffic": (tpe * per_launch_elems if tpe is not None else None),
                "algorithmic_bytes_per_launch": dom_bpe * per_launch_elems}

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(fq, pipe, items, stream, device, args, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, args)

    clocks = sampler.summary()
    step_ms = total_ms / args.steps
    line = {
        "metric": METRIC, "value": value, "unit": "Gelem/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": args.workload, "tensors": [f"{lbl}:{x.shape[0]}x{x.shape[1]}" for lbl, x, *_ in items],
                   "format": {U4: "NVFP4 b16 UE4M3", E8: "MXFP4 b32 E8M0"}[items[0][2]] +
                             (" + FP32 per-tensor scale" if items[0][5] == COMP else ""),
                   "rot": items[0][4], "elements_per_step": elements_step,
                   "block_scales": "max rule" if args.search is None else
                                   f"MSE search: max-rule code, {args.search[1]} above, {args.search[0]} below",
                   "outlier_stats": None if args.outlier_stats is None else
                                    f"max, P{100 * args.outlier_stats:g} of |x| and channel maxima per tensor",
                   "l2": "L2 flushed between steps (512 MiB write)" if in_l2 else
                         f"inputs larger than L2 ({elements_step * 2 / 1e9:.2f} GB bf16 per step)",
                   "parallelism": f"{world} independent replica(s), no data-path collective",
                   "timing": "CUDA events at step boundaries on the launching stream (value, ms_per_step); "
                             "kernel shares from a second pass of K steps with an event after every call",
                   "input": "bf16 written by torch's seeded generator on the device"},
        "hbm": {"GB_per_s": step_bytes / 1e9 / (step_ms / 1e3), "bytes_per_step": step_bytes,
                "frac_of_measured": step_bytes / 1e9 / (step_ms / 1e3) / peak,
                "frac_of_8TBs_spec": step_bytes / 1e9 / (step_ms / 1e3) / SPEC_HBM_GBS},
        "roofline": roofline,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": pipe.launches_per_step * args.steps,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(fq, pipe, items, stream, device, args, world):
    """Same step with the input in pinned host memory: H2D copy of every tensor,
    the hot path, and a D2H read of codes, scales, G and the MSE terms."""
    import torch
    steps = args.e2e_steps or max(3, args.steps // 20)
    host_in = [x.cpu().pin_memory() for _, x, *_ in items]
    host_out = [{k: torch.empty(b[k].shape, dtype=b[k].dtype, pin_memory=True)
                 for k in ("codes", "scales", "gscale", "terms")} for b in pipe.bufs]
    h2d = sum(h.numel() * 2 for h in host_in)
    d2h = sum(sum(o[k].numel() * o[k].element_size() for k in o) for o in host_out)

    def one():
        for (lbl, x, *_), h in zip(items, host_in):
            x.copy_(h, non_blocking=True)
        pipe.step(stream)
        for b, o in zip(pipe.bufs, host_out):
            for k in o:
                o[k].copy_(b[k], non_blocking=True)

    with torch.cuda.stream(stream):
        one()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            one()
        b.record(stream)
        torch.cuda.synchronize()
    ms = reduce_max(a.elapsed_time(b), device)
    return {"value": world * pipe.elements * steps / (ms / 1e3) / 1e9, "unit": "Gelem/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps}


if __name__ == "__main__":
    sys.exit(main())
