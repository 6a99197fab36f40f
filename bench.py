#!/usr/bin/env python
"""Throughput of the absorbed-MLA decode and verify path on B200.

One step = the whole hot path over one batch of a workload: query absorption
(q~ = W_UK^T q), split-L latent attention with the log-sum-exp combine, and the W_UV
up-projection (64 heads, 256-dim NoPE heads, latent 512, bf16).  The five workloads are
tiny dense decode (B=1, 256 rows), dense decode (B=32, 8,192 rows), MTP verify (B=16,
q_len=6, 32,768 + 6 rows), ragged paged decode (B=64, 1,024..131,072 rows in 64-row pages)
and indexed sparse decode (B=32, 2,048 listed rows of 131,072).  One JSON line reports
them all under "configs"; its headline fields are those of ragged paged decode, the
largest.  ``value`` is the effective HBM bandwidth of a step: the algorithmic bytes (every
visible cache row read once, 1,024 B, plus both weight matrices, q, and the output)
divided by the device time of a step; with N ranks every rank runs its own batch (weak
scaling, no collective on the data path) and value sums the bytes over ranks divided by
the slowest rank's time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME|all]

``--impl reference`` times the fp64 CPU oracle (test infrastructure) on a bounded sample
of the same workload instead; it is the reported CPU baseline.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "latent-cache attention: effective HBM GB/s & TFLOP/s vs B200 roofline, 1 GPU"
UNIT = "GB/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic of one attend launch (dram__bytes_read.sum + dram__bytes_write.sum) from the
# ncu capture summarised in profiles/, keyed by the hash of the kernel source it was taken on.
TRAFFIC = {
    ("tiny_dense_decode", "9b3bd05e2802578a"): 398_080,
    ("dense_decode", "9b3bd05e2802578a"): 277_927_936,
    ("mtp_verify", "9b3bd05e2802578a"): 556_837_376,
    ("ragged_paged_decode", "9b3bd05e2802578a"): 4_382_152_448,
    ("indexed_sparse_decode", "9b3bd05e2802578a"): 71_590_656,
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default="all",
                    help="one workload name, or 'all' (every configuration; the headline is ragged paged decode)")
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--cpu-seconds", type=float, default=20.0,
                    help="budget of the CPU-oracle samples, shared by the configurations")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--next-rows", action="store_true",
                    help="time the cache bookkeeping and k-pool producer entry points instead")
    ap.add_argument("--kpool-seqs", type=int, default=4, help="sequences of 131,072 rows for --next-rows")
    ap.add_argument("--prefill-lengths", default="1024,4096",
                    help="prefill lengths for the expanded-vs-absorbed comparison ('' to skip)")
    ap.add_argument("--batch", type=int, default=None,
                    help="profiling size: override the batch of the selected configuration")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="profiling size: every sequence gets this many rows (paged: instead of ragged lengths)")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- workload accounting

def step_bytes(wl) -> dict:
    """Algorithmic bytes of one step: each visible cache row once (1,024 B), both weights,
    q in, o_latent/q~ round trips excluded (intermediates), out written."""
    H, D, R = 64, 256, 512
    if wl.mode == "indexed":
        rows = wl.B * wl.Q * wl.indices.shape[2]
    elif wl.Q == 1:
        rows = int(sum(int(L) for L in wl.seq_lens))
    else:
        rows = int(sum(int(L) for L in wl.seq_lens))  # all Q queries share each row's single read
    visible_pairs = 0
    for L in wl.seq_lens:
        for i in range(wl.Q):
            visible_pairs += (wl.indices.shape[2] if wl.mode == "indexed" else int(L) - wl.Q + i + 1)
    cache = rows * R * 2
    weights = 2 * H * D * R * 2
    qio = 2 * wl.B * wl.Q * H * D * 2
    flops_attend = visible_pairs * H * 4 * R
    flops_proj = 2 * (2 * wl.B * wl.Q * H * D * R)
    return {"cache": cache, "total": cache + weights + qio, "flops_attend": flops_attend,
            "flops_total": flops_attend + flops_proj}


def index_list_sets(wl) -> int:
    """How many independently seeded index lists the indexed workload's steps cycle
    through, so that the rows they gather together exceed L2 (twice over)."""
    K = wl.indices.shape[2]
    return max(1, math.ceil(L2_BYTES * 2 / (wl.B * wl.Q * K * 1024)))


def arm_config(wl, name, world) -> dict:
    """The workload description of a bench line (the same for both arms)."""
    acc = step_bytes(wl)
    if wl.mode == "indexed":
        n = index_list_sets(wl)
        l2 = ("inputs larger than L2: steps cycle through %d seeded index lists, %.0f MB of gathered rows "
              "per cycle" % (n, n * acc["cache"] / 1e6))
    else:
        l2 = "inputs larger than L2 (cache %.0f MB per rank)" % (acc["cache"] / 1e6)
    return {"workload": name, "B": wl.B, "q_len": wl.Q, "mode": wl.mode,
            "cache_rows": int(sum(int(x) for x in wl.seq_lens)) if wl.mode != "indexed" else None,
            "heads": 64, "head_dim": 256, "latent": 512, "parallelism": f"dp{world} (independent batches)",
            "l2": l2}


def attend_roofline(acc, att_ms, peaks, peak_kind, traffic, kernel="attend_kernel + combine_kernel (mla_attend_*)"):
    """Roofline of the attend call (attend + split-L merge): bound by whichever of the cache
    bytes at the HBM peak and the attend FLOPs at the bf16 tensor peak takes longer;
    achieved = that quantity over the measured duration ``att_ms`` (milliseconds)."""
    t_mem = acc["cache"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = acc["flops_attend"] / (peaks["bf16_tflops"] * 1e12)
    common = {"traffic": traffic, "kernel": kernel, "peak_source": peak_kind}
    if t_tc > t_mem:
        ach = acc["flops_attend"] / (att_ms * 1e-3) / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": ach / peaks["bf16_tflops"], **common}
    ach = acc["cache"] / (att_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": ach / peaks["hbm_gbs"], **common}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash():
    """Hash of the attend kernel's code (comments and blank lines left out, so that a
    comment edit does not orphan the recorded traffic)."""
    import re
    h = hashlib.sha256()
    for fn in ("attend.cu", "sm100.cuh", "split.cuh", "internal.h"):
        with open(os.path.join(ROOT, "mla_absorbed_latent_mtp_b200", "csrc", fn)) as f:
            text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
        for line in text.splitlines():
            code = line.split("//", 1)[0].strip()
            if code:
                h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed loop runs.

    NVML is polled about once a millisecond from a thread (a timed region of a few tens
    of milliseconds still gets samples); without NVML, ``nvidia-smi -lms 50`` is read
    instead.  Only samples taken inside the timed window count: with none there, the
    summary says "unsampled" rather than reporting idle clocks."""
    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NVML_REASONS = ((0x4, "sw_power_cap"), (0x8, "hw_slowdown"), (0x20, "sw_thermal_slowdown"),
                    (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"))

    def __init__(self, index, pci_bus_id=None):
        self.index = index
        self.pci_bus_id = pci_bus_id
        self.proc = None
        self.rows = []  # (wall time, sm MHz, max sm MHz, [reason names])
        self.source = None
        self._stop = threading.Event()
        self.thread = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            if self.pci_bus_id:
                h = pynvml.nvmlDeviceGetHandleByPciBusId(self.pci_bus_id)
            else:
                h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.source = "nvml 1 ms"
            self.thread = threading.Thread(target=self._poll_nvml, args=(pynvml, h, max_mhz), daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi 50 ms"
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _poll_nvml(self, pynvml, h, max_mhz):
        while not self._stop.is_set():
            try:
                mhz = float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                bits = int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))
            except Exception:
                return
            row = (time.time(), mhz, max_mhz, [n for b, n in self.NVML_REASONS if bits & b])
            try:  # memory clock and board power, where NVML offers them
                row = row + (float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_MEM)),
                             pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0)
            except Exception:
                pass
            self.rows.append(row)
            time.sleep(0.001)

    def _read_smi(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.strip().split(",")]
            if len(parts) < 10:
                continue
            try:
                self.rows.append((time.time(), float(parts[2]), float(parts[3]),
                                  [names[k] for k, v in enumerate(parts[6:10]) if v.lower() == "active"]))
            except ValueError:
                continue

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        window = [r for r in self.rows if t0 <= r[0] <= t1]
        if not window:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0,
                    "source": self.source}
        reasons = sorted({n for r in window for n in r[3]})
        out = {"sm_mhz": statistics.median(r[1] for r in window), "sm_max_mhz": max(r[2] for r in window),
               "sm_mhz_min": min(r[1] for r in window), "reasons": reasons, "samples": len(window),
               "source": self.source}
        nv = [r for r in window if len(r) > 5]
        if nv:
            out["mem_mhz"] = statistics.median(r[4] for r in nv)
            out["mem_mhz_min"] = min(r[4] for r in nv)
            out["power_w_median"] = statistics.median(r[5] for r in nv)
            out["power_w_max"] = max(r[5] for r in nv)
        return out


# ----------------------------------------------------------------------------- distributed helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(values, device):
    """Element-wise max over ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def reduce_sum(values, device):
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.tolist()


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def aggregate(local_ms, local_bytes, device):
    """Whole-job throughput: bytes summed over ranks / slowest rank's time."""
    (ms,) = reduce_max([local_ms], device)
    (total_bytes,) = reduce_sum([float(local_bytes)], device)
    return ms, total_bytes / (ms * 1e-3) / 1e9


# ----------------------------------------------------------------------------- CPU oracle baseline

def cpu_baseline(wl, budget_s, got=None):
    """Time the fp64 oracle (expanded form, as it stands) on a bounded sample: heads of
    sequence 0, query 0, added until the budget is spent.  Reported in the metric's unit.

    ``got`` (the GPU step's output bits, [B, Q, 64, 256]) is compared with the oracle on the
    same sample: max-abs and mean-abs error (the parity gate's quantities) and max-abs over
    the RMS of the reference (a relative measure that does not shrink with the output)."""
    import numpy as np
    import oracle
    t_start = time.perf_counter()
    heads = 0
    outs = []
    while heads < 64:
        r = oracle.reference(wl, pairs=[(0, 0)], heads=[heads], row_source=None)
        outs.append(r[(0, 0)]["out"][0])
        heads += 1
        if time.perf_counter() - t_start > budget_s:
            break
    dt = time.perf_counter() - t_start
    L = int(wl.seq_lens[0]) if wl.mode != "indexed" else wl.indices.shape[2]
    bytes_attributed = L * 1024 * heads / 64.0
    cores = threads_used()
    res = {"value": bytes_attributed / dt / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
           "sample": f"sequence 0, query 0, {heads} of 64 heads, {L} cached rows, expanded fp64 form "
                     f"({dt:.1f} s)"}
    if got is not None:
        ref = np.stack(outs)
        g = (np.asarray(got, dtype=np.uint16)[0, 0, :heads].astype(np.uint32) << 16).view(np.float32)
        err = np.abs(g.astype(np.float64) - ref)
        rms = float(np.sqrt((ref ** 2).mean()))
        res["parity"] = {"max_abs": float(err.max()), "mean_abs": float(err.mean()),
                         "max_abs_over_rms": float(err.max()) / rms if rms > 0 else None,
                         "gate": "max-abs <= 2e-2 and mean-abs <= 2e-3",
                         "pass": bool(err.max() <= 2e-2 and err.mean() <= 2e-3)}
    return res


def threads_used():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("internal_api") in ("openblas", "mkl", "blis")]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def run_reference(args, wl_name):
    """The oracle on the host cores, each step a bounded sample (one head of one sequence)."""
    import synth
    world, rank, _ = dist_env()
    if rank != 0:
        return
    wl = synth.make_workload(wl_name, with_data=False)
    import oracle

    L = int(wl.seq_lens[0]) if wl.mode != "indexed" else wl.indices.shape[2]
    rows_fn = lambda b, pos: synth.cache_rows(wl, b, pos)  # noqa: E731
    budget_total = 150.0
    # calibrate the rows per step so that warmup + steps fit the budget
    rows = L
    t = time.perf_counter()
    sub = _truncated(wl, rows)
    oracle.reference(sub, pairs=[(0, sub.Q - 1)], heads=[0], row_source=rows_fn)
    one = time.perf_counter() - t
    per_step = budget_total / max(args.steps + args.warmup, 1)
    if one > per_step:
        rows = max(64, int(L * per_step / one))
        sub = _truncated(wl, rows)
    for _ in range(args.warmup):
        oracle.reference(sub, pairs=[(0, sub.Q - 1)], heads=[0], row_source=rows_fn)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.reference(sub, pairs=[(0, sub.Q - 1)], heads=[0], row_source=rows_fn)
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    value = rows * 1024 / 64.0 / dt / 1e9
    sample = f"one head of sequence 0 (last query), {rows} cached rows per step, expanded fp64 form"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": arm_config(wl, wl_name, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads_used(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def _truncated(wl, rows):
    """Same workload restricted to its first `rows` cache rows of sequence 0."""
    import copy
    sub = copy.copy(wl)
    import numpy as np
    lens = wl.seq_lens.copy()
    if wl.mode != "indexed":
        lens[0] = min(int(lens[0]), rows)
    else:
        sub.indices = wl.indices[:, :, :rows]
    sub.seq_lens = lens
    return sub


# ----------------------------------------------------------------------------- our arm

def run_next_rows(args):
    """Event timing (median) of the latent-cache bookkeeping and the k-pool index producer:
    append / truncate on the verify shape (B=16, q_len=6, 32,768-row prefix), pooled keys and
    selection on --kpool-seqs sequences of 131,072 rows (pools of 64, topk 2,048 + tail)."""
    import numpy as np
    import torch

    import mla_absorbed_latent_mtp_b200 as m
    import synth
    from mla_absorbed_latent_mtp_b200 import _build

    _build.build()
    torch.cuda.set_device(0)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)

    B, Q, L0 = 16, 6, 32768
    cache = torch.zeros(B, L0 + 64, 512, dtype=torch.bfloat16, device="cuda")
    lens = torch.full((B,), L0, dtype=torch.int32, device="cuda")
    rows = dev(synth.normal_bf16((B, Q, 512), 1, synth.STREAM_Q))
    keep = torch.full((B,), 3, dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ta, tt = [], []
    for k in range(args.warmup + args.steps):
        lens.fill_(L0)
        ev[0].record(); m.mla_cache_append_dense(cache, lens, rows, st); ev[1].record()
        m.mla_cache_truncate_dense(cache, lens, keep, Q, st); ev[2].record()
        torch.cuda.synchronize()
        if k >= args.warmup:
            ta.append(ev[0].elapsed_time(ev[1])); tt.append(ev[1].elapsed_time(ev[2]))
    B2, L2, pool, topk = args.kpool_seqs, 131072, 64, 2048
    c2 = dev(synth.normal_bf16((B2, L2, 512), 2, synth.STREAM_CACHE))
    l2 = torch.full((B2,), L2, dtype=torch.int32, device="cuda")
    wq = dev(synth.normal_bf16((B2, 1, 512), 3, synth.STREAM_Q))
    pooled = torch.zeros(B2, L2 // pool, 512, dtype=torch.float32, device="cuda")
    tk, ts = [], []
    for k in range(args.warmup + args.steps):
        ev[0].record(); m.mla_kpool_keys(c2, pool, l2, pooled); ev[1].record()
        m.mla_kpool_select(pooled, wq, pool, topk, l2, True, Lmax=L2); ev[2].record()
        torch.cuda.synchronize()
        if k >= args.warmup:
            tk.append(ev[0].elapsed_time(ev[1])); ts.append(ev[1].elapsed_time(ev[2]))
    assert int(st.item()) == 0, m.status_string(int(st.item()))
    med = lambda x: float(np.median(x)) * 1e3  # noqa: E731
    print(json.dumps({
        "next_rows": True, "unit": "us", "steps": args.steps, "warmup": args.warmup,
        "cache_append_dense_us": med(ta), "cache_truncate_dense_us": med(tt),
        "cache_shape": {"B": B, "q_len": Q, "prefix": L0, "keep": 3},
        "kpool_keys_us": med(tk), "kpool_keys_gbs": B2 * L2 * 1024 / (med(tk) * 1e-6) / 1e9,
        "kpool_select_us": med(ts),
        "kpool_shape": {"B": B2, "rows": L2, "pool": pool, "topk": topk, "tail": True, "queries": B2},
    }))


CONFIG_NAMES = ("tiny_dense_decode", "dense_decode", "mtp_verify", "ragged_paged_decode", "indexed_sparse_decode")
# the largest of the five workloads that fit one GPU: the line's headline
HEADLINE = "ragged_paged_decode"
# host->device bytes the end-to-end leg may copy per configuration (a few seconds of PCIe)
E2E_BYTES_CAP = 24e9


def steps_per_graph(K, n_rot=1, cap=32):
    """Steps captured per CUDA graph: the largest divisor of K up to `cap`, preferring a
    multiple of the number of index-list sets the steps rotate through."""
    divisors = [g for g in range(1, min(K, cap) + 1) if K % g == 0]
    rot = [g for g in divisors if g % n_rot == 0]
    return max(rot) if rot else max(divisors)


def capture(fn, n, idx_turn=None, keep=False):
    """A CUDA graph of n calls of fn (the library's launches go to torch's capture stream).
    The index-list rotation restarts at the first set in every graph.  keep: the captured
    graph stays inspectable (graph_kernel_nodes)."""
    import torch
    if idx_turn is not None:
        idx_turn[0] = 0
    g = torch.cuda.CUDAGraph(keep_graph=keep)
    with torch.cuda.graph(g):
        for _ in range(n):
            fn()
    if keep:
        g.instantiate()
    return g


def graph_kernel_nodes(g):
    """Kernel launches recorded in a graph captured with keep=True.  The captured steps call
    only this library, so every kernel node is one of its kernels."""
    from cuda.bindings import runtime as rt
    h = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
    err, _, n = rt.cudaGraphGetNodes(h, 0)
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaGraphGetNodes: {err}")
    err, nodes, n = rt.cudaGraphGetNodes(h, n)
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaGraphGetNodes: {err}")
    kernels = 0
    for node in nodes[:n]:
        err, kind = rt.cudaGraphNodeGetType(node)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaGraphNodeGetType: {err}")
        kernels += kind == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
    return kernels


def _seq_len(name, args):
    """Rows per sequence for a profiling-size run (MTP verify: prefix + the 6 window rows)."""
    if args.seq_len is None:
        return None
    return args.seq_len + (6 if name == "mtp_verify" else 0)


def measure_config(name, args, device, rank, world, clocks, peaks, peak_kind, src_hash, cpu_seconds):
    """One configuration: the timed steps, the stage breakdown, the chained attend timing for
    the roofline, the end-to-end leg with host buffers, and (rank 0 of a 1-GPU run) the CPU
    oracle on a sample, whose outputs are also compared with this run's.  Returns the
    configuration's record; every rank takes the same collective steps."""
    import numpy as np
    import torch

    import mla_absorbed_latent_mtp_b200 as m
    import synth

    wl = synth.make_workload(name, seed=rank, with_data=False, B=args.batch, L=_seq_len(name, args))
    acc = step_bytes(wl)
    B, Q = wl.B, wl.Q

    def dev_bits(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)

    host_cache = torch.empty(wl.extra["cache_shape"], dtype=torch.int16, pin_memory=True)
    synth.fill_cache(wl, host_cache.data_ptr())
    host_q = torch.from_numpy(np.ascontiguousarray(wl.q).view(np.int16)).pin_memory()
    cache = host_cache.to(device).view(torch.bfloat16)
    q = host_q.to(device).view(torch.bfloat16)
    w_uk, w_uv = dev_bits(wl.w_uk), dev_bits(wl.w_uv)
    lens = torch.from_numpy(wl.seq_lens).to(device)
    host_lens = torch.from_numpy(wl.seq_lens).pin_memory()
    table = torch.from_numpy(wl.page_table).to(device) if wl.mode == "paged" else None
    idx = torch.from_numpy(wl.indices).to(device) if wl.mode == "indexed" else None
    # the rows one indexed step gathers (B*Q*K KiB) fit in L2: consecutive steps cycle
    # through independently seeded index lists whose rows together exceed it
    idx_sets = [idx]
    if wl.mode == "indexed":
        K_idx = wl.indices.shape[2]
        for r in range(1, index_list_sets(wl)):
            idx_sets.append(torch.from_numpy(synth.index_lists(B, Q, K_idx, wl.seq_lens,
                                                               seed=1000 * (rank + 1) + r)).to(device))
    idx_turn = [0]
    ws = m.new_workspace(B, Q)
    qt = torch.empty(B, Q, 64, 512, dtype=torch.bfloat16, device=device)
    o = torch.empty(B, Q, 64, 512, dtype=torch.bfloat16, device=device)
    lse = torch.empty(B, Q, 64, dtype=torch.float32, device=device)
    out = torch.empty(B, Q, 64, 256, dtype=torch.bfloat16, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    host_out = torch.empty(out.shape, dtype=torch.int16, pin_memory=True)

    def absorb():
        m.mla_absorb_q(q, w_uk, qt)

    def attend():
        if wl.mode == "dense":
            m.mla_attend_dense(qt, cache, lens, wl.scale, ws, o, lse, status)
        elif wl.mode == "paged":
            m.mla_attend_paged(qt, cache, table, lens, wl.scale, ws, o, lse, status)
        else:
            m.mla_attend_indexed(qt, cache, idx_sets[idx_turn[0] % len(idx_sets)], lens, wl.scale, ws, o, lse,
                                 status)
            idx_turn[0] += 1

    def up():
        m.mla_up_proj(o, w_uv, out)

    # the fused path: the up-projection runs inside the split-L merge (mla_attend_up_*)
    def attend_up():
        if wl.mode == "dense":
            m.mla_attend_up_dense(qt, cache, w_uv, lens, wl.scale, ws, out, None, lse, status)
        elif wl.mode == "paged":
            m.mla_attend_up_paged(qt, cache, table, lens, w_uv, wl.scale, ws, out, None, lse, status)
        else:
            m.mla_attend_up_indexed(qt, cache, idx_sets[idx_turn[0] % len(idx_sets)], w_uv, lens, wl.scale, ws, out,
                                    None, lse, status)
            idx_turn[0] += 1

    def chained_step():
        absorb(); attend(); up()

    def fused_step():
        absorb(); attend_up()

    for _ in range(args.warmup):
        chained_step()
        fused_step()
    torch.cuda.synchronize()
    assert int(status.item()) == 0, m.status_string(int(status.item()))

    # Every timed loop replays CUDA graphs: the host-side cost of a launch through Python
    # (tens of microseconds) would otherwise set the pace of the short workloads.  A graph
    # holds G steps (for the index-list workload a multiple of the list sets it cycles
    # through); the loops replay K / G of them, so exactly K steps run.
    K = args.steps
    G = steps_per_graph(K, len(idx_sets))
    g_chained = capture(chained_step, G, idx_turn, keep=True)
    g_fused = capture(fused_step, G, idx_turn, keep=True)
    # kernels per step, counted in the captured graphs (the index-list attend merges inside
    # its clusters when they fit, so its step has no combine kernel)
    per_step = {"chained": graph_kernel_nodes(g_chained) / G, "fused": graph_kernel_nodes(g_fused) / G}
    for _ in range(max(1, -(-args.warmup // G))):
        g_chained.replay()
        g_fused.replay()
    torch.cuda.synchronize()

    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    wall0 = time.time()
    # the timed steps: nothing between the launches, so each kernel may start while the
    # previous one drains (the library chains its launches)
    start.record()
    for _ in range(K // G):
        g_chained.replay()
    stop.record()
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier()
    local_ms = start.elapsed_time(stop) / K
    ms, value = aggregate(local_ms, acc["total"], device)

    f_start, f_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    fw0 = time.time()
    f_start.record()
    for _ in range(K // G):
        g_fused.replay()
    f_stop.record()
    torch.cuda.synchronize()
    fw1 = time.time()
    barrier()
    fused_ms, fused_value = aggregate(f_start.elapsed_time(f_stop) / K, acc["total"], device)
    # the step the line reports: whichever path (chained or fused) is faster on this workload
    best = "fused" if fused_ms < ms else "chained"
    launches = int(round(K * per_step[best]))

    # Each stage alone, Kb times back to back in one graph (stage time = graph time / Kb),
    # and the attend call (attend + split-L combine) the same way: its duration as it runs
    # inside the step, for the roofline.  The fused attend (attend + merge + up-projection)
    # likewise.
    Kb = max(len(idx_sets), min(K, 50) // len(idx_sets) * len(idx_sets))

    def timed_graph(fn, reps, replays=3):
        # the average call over `replays` back-to-back replays of a graph of `reps` calls
        g = capture(fn, reps, idx_turn)
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(replays):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / (reps * replays)

    stage = reduce_max([timed_graph(absorb, Kb), timed_graph(attend, Kb), timed_graph(up, Kb)], device)
    aw0 = time.time()
    att_ms = reduce_max([timed_graph(attend, max(Kb, 20))], device)[0]
    aw1 = time.time()
    attend_up_ms = reduce_max([timed_graph(attend_up, max(Kb, 20))], device)[0]
    del g_chained, g_fused

    # End to end through the public API with host buffers, as a serving step runs: the
    # step's inputs come from pinned host memory -- the queries, the latent rows of the
    # step's own positions (the last q_len of each sequence) and, for index lists, the
    # lists -- the previous step's rows are rolled back (mla_cache_truncate_*, keep 0) and
    # the new ones appended (mla_cache_append_*), then absorb, attend and up-project, and
    # the output is read back.  The history cache stays resident, as a server keeps it.
    # The rows are the workload's own, so every step leaves the cache as it found it.
    Qw = wl.Q
    hc = host_cache.numpy()
    if wl.mode == "paged":
        rows_np = np.stack([np.stack([hc[wl.page_table[b, j // 64], j % 64]
                                      for j in range(int(wl.seq_lens[b]) - Qw, int(wl.seq_lens[b]))])
                            for b in range(B)])
    else:
        rows_np = np.stack([hc[b, int(wl.seq_lens[b]) - Qw:int(wl.seq_lens[b])] for b in range(B)])
    host_rows = torch.from_numpy(np.ascontiguousarray(rows_np)).pin_memory()
    rows_dev = torch.empty(host_rows.shape, dtype=torch.int16, device=device)
    keep0 = torch.zeros(B, dtype=torch.int32, device=device)
    host_idx = [t.cpu().pin_memory() for t in idx_sets] if wl.mode == "indexed" else []

    def roll_in(rows_buf):
        if wl.mode == "paged":
            m.mla_cache_truncate_paged(cache, table, lens, keep0, Qw, status)
            m.mla_cache_append_paged(cache, table, lens, rows_buf.view(torch.bfloat16), status)
        else:
            m.mla_cache_truncate_dense(cache, lens, keep0, Qw, status)
            m.mla_cache_append_dense(cache, lens, rows_buf.view(torch.bfloat16), status)

    def timed_serving(steps):
        """Serving steps as a server would run them: a copy stream brings step i + 1's inputs
        in (and takes step i - 1's output out) while the compute stream runs step i, inputs
        and outputs double-buffered, the rest in order on the compute stream.  Like the
        timed steps, they are replayed from CUDA graphs of G steps (copies included), so
        that the host's per-call cost does not set the pace."""
        nonlocal q, out
        q0, out0 = q, out
        Cs = torch.cuda.Stream()
        qb, rb = [q0, torch.empty_like(q0)], [rows_dev, torch.empty_like(rows_dev)]
        ob = [out0, torch.empty_like(out0)]
        hob = [host_out, torch.empty(host_out.shape, dtype=torch.int16, pin_memory=True)]
        G = steps_per_graph(steps, len(idx_sets))

        def one_graph():
            nonlocal q, out
            S = torch.cuda.current_stream()
            Cs.wait_stream(S)
            ev_in, ev_used, ev_copied = [None] * G, [None] * G, [None] * G

            def inputs(i):
                k = i % 2
                with torch.cuda.stream(Cs):
                    if i >= 2:
                        Cs.wait_event(ev_used[i - 2])  # step i - 2 has consumed this buffer pair
                    qb[k].view(torch.int16).copy_(host_q, non_blocking=True)
                    rb[k].copy_(host_rows, non_blocking=True)
                    if wl.mode == "indexed":
                        j = i % len(idx_sets)
                        idx_sets[j].copy_(host_idx[j], non_blocking=True)
                    ev_in[i] = torch.cuda.Event()
                    ev_in[i].record(Cs)

            inputs(0)
            for i in range(G):
                k = i % 2
                if i + 1 < G:
                    inputs(i + 1)
                S.wait_event(ev_in[i])
                if i >= 2:
                    S.wait_event(ev_copied[i - 2])  # step i - 2's output has left this buffer
                q, out = qb[k], ob[k]
                roll_in(rb[k])
                if best == "fused":
                    absorb(); attend_up()
                else:
                    absorb(); attend(); up()
                ev_used[i] = torch.cuda.Event()
                ev_used[i].record(S)
                with torch.cuda.stream(Cs):
                    Cs.wait_event(ev_used[i])
                    hob[k].copy_(ob[k].view(torch.int16), non_blocking=True)
                    ev_copied[i] = torch.cuda.Event()
                    ev_copied[i].record(Cs)
            S.wait_stream(Cs)

        gr = capture(one_graph, 1, idx_turn)
        q, out = q0, out0
        gr.replay()
        torch.cuda.synchronize()
        e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e_start.record()
        for _ in range(steps // G):
            gr.replay()
        e_stop.record()
        torch.cuda.synchronize()
        del gr
        # the last serving step's output, as read back, equals a plain step's on the same
        # inputs (the roll-back and append left the cache as it was)
        last = hob[(G - 1) % 2].clone()
        idx_turn[0] = G - 1
        if best == "fused":
            absorb(); attend_up()
        else:
            absorb(); attend(); up()
        torch.cuda.synchronize()
        assert torch.equal(last, out.view(torch.int16).cpu()), "serving step output differs from a plain step"
        return aggregate(e_start.elapsed_time(e_stop) / steps, acc["total"], device)

    def timed_cold(steps):
        e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        idx_turn[0] = 0
        barrier()
        torch.cuda.synchronize()
        e_start.record()
        for _ in range(steps):
            cache.view(torch.int16).copy_(host_cache, non_blocking=True)
            q.view(torch.int16).copy_(host_q, non_blocking=True)
            lens.copy_(host_lens, non_blocking=True)
            if best == "fused":
                absorb(); attend_up()
            else:
                absorb(); attend(); up()
            host_out.copy_(out.view(torch.int16), non_blocking=True)
        e_stop.record()
        torch.cuda.synchronize()
        return aggregate(e_start.elapsed_time(e_stop) / steps, acc["total"], device)

    h2d = host_q.numel() * 2 + host_rows.numel() * 2 + (host_idx[0].numel() * 4 if host_idx else 0)
    d2h = host_out.numel() * 2
    Ke = max(1, min(args.e2e_steps, K))
    e_ms, e_value = timed_serving(Ke)
    # the same with the whole cache uploaded every step (no resident state at all)
    h2d_cold = host_cache.numel() * 2 + host_q.numel() * 2 + host_lens.numel() * 4
    Kc = max(1, min(args.e2e_steps, K, int(E2E_BYTES_CAP // h2d_cold)))
    c_ms, c_value = timed_cold(Kc)
    assert int(status.item()) == 0, m.status_string(int(status.item()))

    in_cluster = per_step["chained"] < 4  # absorb, attend, up-projection: no combine kernel
    roofline = attend_roofline(acc, att_ms, peaks, peak_kind, TRAFFIC.get((name, src_hash)),
                               "attend_kernel, merging in its clusters (mla_attend_indexed)" if in_cluster
                               else "attend_kernel + combine_kernel (mla_attend_*)")
    label = name if args.batch is None and args.seq_len is None else \
        f"{name} at a profiling size (B={B}, rows={args.seq_len})"
    rec = {
        "workload": arm_config(wl, label, world),
        "value": fused_value if best == "fused" else value, "unit": UNIT,
        "ms_per_step": fused_ms if best == "fused" else ms, "steps": K, "step_path": best,
        "paths": {"chained": {"ms_per_step": ms, "value": value, "kernels_per_step": per_step["chained"],
                              "kernels": "absorb, attend, split-L merge (a combine kernel, or inside the "
                                         "attend kernel's clusters for index lists), up-projection"},
                  "fused": {"ms_per_step": fused_ms, "value": fused_value, "kernels_per_step": per_step["fused"],
                            "kernels": "absorb, attend, split-L merge fused with the up-projection",
                            "attend_and_merge_up_ms": attend_up_ms}},
        "stages_ms": {"absorb_q": stage[0], "attend": stage[1], "up_proj": stage[2], "attend_chained": att_ms},
        "attend_tflops": acc["flops_attend"] / (att_ms * 1e-3) / 1e12,
        "attend_cache_bytes": acc["cache"], "attend_flops": acc["flops_attend"],
        "roofline": roofline,
        "e2e": {"value": e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e_ms, "steps": Ke,
                "step": "serving step: H2D of q, the step's q_len latent rows per sequence"
                        + (" and the index lists" if wl.mode == "indexed" else "")
                        + "; roll back + append them (mla_cache_truncate/append); absorb, attend, "
                          "up-project; D2H of out.  The history cache stays resident; copies run on a "
                          "second stream, double-buffered, overlapping the previous step's compute."},
        "e2e_cache_upload": {"value": c_value, "unit": UNIT, "h2d_bytes_per_step": h2d_cold,
                             "d2h_bytes_per_step": d2h, "ms_per_step": c_ms, "steps": Kc,
                             "step": "the whole cache, q and lengths uploaded every step, then the step; "
                                     "PCIe-bound"},
        "gpu_launches": launches,
        "roofline_fused": dict(attend_roofline(acc, attend_up_ms, peaks, peak_kind, None),
                               kernel="attend_kernel + merge_up_kernel (mla_attend_up_*: attend, split-L merge "
                                      "and W_UV up-projection)"),
        "clocks": clocks.summary(wall0, wall1) if best == "chained" else clocks.summary(fw0, fw1),
        "clocks_attend_chained": clocks.summary(aw0, aw1),
        "timing": f"device time (CUDA events) around replays of CUDA graphs of {G} steps",
    }
    if cpu_seconds > 0:
        if wl.mode == "indexed":
            # one more step on the workload's own index lists, whose output the sample checks
            idx_turn[0] = 0
            absorb(); attend(); up()
            torch.cuda.synchronize()
        wl_cpu = synth.make_workload(name, with_data=False, B=args.batch, L=_seq_len(name, args))
        wl_cpu.cache = host_cache.numpy().view(np.uint16) if wl.mode != "paged" else None
        wl_cpu.pool = host_cache.numpy().view(np.uint16) if wl.mode == "paged" else None
        host_out.copy_(out.view(torch.int16))  # the last timed step's output (same inputs every step)
        got = host_out.numpy().view(np.uint16)
        rec["cpu_baseline"] = cpu_baseline(wl_cpu, cpu_seconds, got)
    del cache, host_cache, idx_sets, ws
    torch.cuda.empty_cache()
    return rec


def prefill_flops(L, B=1):
    """Algorithmic FLOPs of one causal prefill of B sequences of L tokens (64 heads, head 256,
    latent 512): causal (query, key) pairs L(L+1)/2 per sequence and head."""
    H, D, R = 64, 256, 512
    pairs = B * L * (L + 1) // 2
    expand = 2 * (2 * B * L * R * H * D)          # k and v from the latents
    attn_expanded = pairs * H * 2 * (2 * D)       # q.k and p.v over 256-wide heads
    proj = 2 * (2 * B * L * H * D * R)            # absorb q and up-project o
    attn_absorbed = pairs * H * 2 * (2 * R)       # q~.c and p.c over the 512-wide latent
    return {"expanded": expand + attn_expanded, "absorbed": proj + attn_absorbed,
            "expanded_attention": attn_expanded, "absorbed_attention": attn_absorbed}


def measure_prefill(lengths, device, peaks, reps=5):
    """Module 05 section 5's comparison on B200: one causal prefill of L tokens in the
    expanded form (mla_expand_kv + mla_prefill_expanded) and in the absorbed form
    (mla_absorb_q + mla_attend_dense with q_len = L + mla_up_proj), timed with CUDA events
    (warm-up first, median of `reps`)."""
    import numpy as np
    import torch

    import mla_absorbed_latent_mtp_b200 as m
    import synth

    res = []
    for L in lengths:
        wl = synth.make_workload(mode="dense", B=1, Q=L, L=L, with_data=True, seed=5)
        dev = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(  # noqa: E731
            torch.bfloat16)
        q, wk, wv, cache = dev(wl.q), dev(wl.w_uk), dev(wl.w_uv), dev(wl.cache)
        lens = torch.from_numpy(wl.seq_lens).to(device)
        st = torch.zeros(1, dtype=torch.int32, device=device)
        k = torch.empty(1, L, 64, 256, dtype=torch.bfloat16, device=device)
        v = torch.empty_like(k)
        out_e = torch.empty_like(k)
        qt = torch.empty(1, L, 64, 512, dtype=torch.bfloat16, device=device)
        o = torch.empty_like(qt)
        out_a = torch.empty_like(k)
        ws = m.new_workspace(1, L)

        def expanded():
            m.mla_expand_kv(cache[0], wk, wv, k[0], v[0])
            m.mla_prefill_expanded(q, k, v, wl.scale, out_e, want_lse=False, status=st)

        def absorbed():
            m.mla_absorb_q(q, wk, qt)
            m.mla_attend_dense(qt, cache, lens, wl.scale, ws, o, None, st, want_lse=False)
            m.mla_up_proj(o, wv, out_a)

        def timed(fn):
            for _ in range(2):
                fn()
            ts = []
            for _ in range(reps):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(); fn(); b.record()
                torch.cuda.synchronize()
                ts.append(a.elapsed_time(b))
            return float(np.median(ts))

        te, ta = timed(expanded), timed(absorbed)
        assert int(st.item()) == 0, m.status_string(int(st.item()))
        diff = float((out_e.float() - out_a.float()).abs().max())
        fl = prefill_flops(L)
        peak = peaks["bf16_tflops"]
        res.append({"L": L, "B": 1,
                    "expanded": {"ms": te, "flops": fl["expanded"], "tflops": fl["expanded"] / (te * 1e-3) / 1e12,
                                 "frac_of_tensor_peak": fl["expanded"] / (te * 1e-3) / 1e12 / peak},
                    "absorbed": {"ms": ta, "flops": fl["absorbed"], "tflops": fl["absorbed"] / (ta * 1e-3) / 1e12,
                                 "frac_of_tensor_peak": fl["absorbed"] / (ta * 1e-3) / 1e12 / peak},
                    "faster": "expanded" if te < ta else "absorbed", "speedup": max(te, ta) / min(te, ta),
                    "max_abs_difference_between_forms": diff})
        del k, v, out_e, qt, o, out_a, ws, q, cache
        torch.cuda.empty_cache()
    return res


def main(argv=None):
    args = parse_args(argv)
    world, rank, local = dist_env()
    if args.next_rows:
        if rank == 0:
            run_next_rows(args)
        return
    names = list(CONFIG_NAMES) if args.config == "all" else [args.config]
    headline = HEADLINE if args.config == "all" else args.config
    if args.impl == "reference":
        # under torchrun rank 0 alone runs the oracle; the other ranks exit without work
        # (no process group: nothing is exchanged)
        run_reference(args, headline)
        return

    import torch

    import mla_absorbed_latent_mtp_b200 as m

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    from mla_absorbed_latent_mtp_b200 import _build
    if rank == 0:
        _build.build()
    barrier()
    m.lib()

    props = torch.cuda.get_device_properties(local)
    bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
    clocks = ClockSampler(local, bus)
    clocks.start()
    time.sleep(0.3)
    peaks, peak_kind = load_peaks()
    src_hash = kernel_source_hash()
    want_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    per_cfg = {}
    for name in names:
        per_cfg[name] = measure_config(name, args, device, rank, world, clocks, peaks, peak_kind, src_hash,
                                       args.cpu_seconds / len(names) if want_cpu else 0.0)
    prefill = None
    if args.prefill_lengths:
        lengths = [int(x) for x in args.prefill_lengths.split(",") if x]
        prefill = measure_prefill(lengths, device, peaks)
    time.sleep(0.1)
    clocks.stop()

    head = per_cfg[headline]
    result = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded SplitMix64/Box-Muller; random-init weights of the stated shapes)",
        "config": head["workload"],
        "stages_ms": head["stages_ms"],
        "attend_tflops": head["attend_tflops"],
        "roofline": head["roofline"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
        "kernel_src": src_hash,
        "peaks": {k: peaks.get(k) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")},
        "configs": {n: {k: v for k, v in r.items() if k != "workload"} | {"config": r["workload"]}
                    for n, r in per_cfg.items()},
    }
    if "cpu_baseline" in head:
        result["cpu_baseline"] = head["cpu_baseline"]
    if prefill is not None:
        result["prefill_comparison"] = prefill
    if rank == 0:
        print(json.dumps(result))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
