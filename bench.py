"""Benchmark of the MXFP8 learner/sampler-grid hot path on B200.

Headline workload (one "step"): the Qwen3-8B weight synchronization of "End-to-End MXFP8
Reinforcement Learning on Blackwell" (Figure 1, Table 11): the learner quantizes all 144 BF16
linear weights (36 layers x qkv 6144x4096, o 4096x4096, gate_up 24576x4096, down 4096x12288)
rowwise with the scales written straight into the tensor-core layout, then the byte comparison
checks the learner's grid (elements and swizzled scales) against the sampler's copy, which was
re-derived from the dequantized grid at set-up. Metric: algorithmic GB/s of the whole step
(quantize reads 2 B and writes 1 + 1/32 B per element; the comparison reads both grids).

Also reported (same run, "secondary"): block-scaled GEMM TFLOP/s on the dense forward linear
(M = 1300 / 5200 / 10300 tokens x 24576 x 4096), the dense update micro-batch (fprop, dgrad,
wgrad at 12288 tokens) and the Qwen3-30B-A3B MoE grouped GEMMs; and quantize GB/s on activation
tensors.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mx|reference] [--no-secondary]

N > 1 runs under torchrun, one process per GPU; every rank quantizes and checks its own full set
of weights (weak scaling, no collective on the data path); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
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

METRIC = "MXFP8 quantize+swizzle GB/s and block-scaled GEMM TFLOP/s, % of B200 roofline"
UNIT = "GB/s"
WORKLOAD = "qwen3-8b weight sync: quantize+swizzle 144 BF16 weights (36 layers), grid_equal vs sampler copy"
QUANT_BYTES_PER_ELEM = 2.0 + 1.0 + 1.0 / 32.0
NOMINAL_FP8_OVER_BF16 = 2.0           # dense fp8 / bf16 tensor throughput (4.5 / 2.25 PFLOP/s)
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def sync_shapes():
    from mxfp8_block_scaled_07_b200 import synth

    return [(layer, idx, r, c) for layer in range(synth.QWEN3_8B_LAYERS) for idx, (_, r, c) in
            enumerate(synth.QWEN3_8B_LINEARS)]


# ---------------------------------------------------------------------------------------------
# clocks sampling during the timed region
# ---------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.times = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())
            self.times.append(time.monotonic())

    def window(self, t0: float, t1: float) -> dict:
        """SM clock and power of the samples taken between t0 and t1 (time.monotonic()), or of the
        nearest sample when the window is shorter than the sampling interval."""
        rows = []
        for t, ln in zip(list(self.times), list(self.lines)):
            parts = [p.strip() for p in ln.split(",")]
            try:
                rows.append((t, float(parts[0]), float(parts[2]), parts[4:8]))
            except (ValueError, IndexError):
                continue
        if not rows:
            return {}
        inside = [r for r in rows if t0 <= r[0] <= t1] or [min(rows, key=lambda r: abs(r[0] - 0.5 * (t0 + t1)))]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for *_, flags in inside for i, f in enumerate(flags) if f.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "power_w": round(statistics.median(r[2] for r in inside), 1), "reasons": reasons,
                "samples": len(inside)}

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, f in enumerate(flags) if f.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------------------------
# reference arm / CPU baseline: the oracle on the host cores, bounded sample
# ---------------------------------------------------------------------------------------------

def oracle_sync_sample(budget_s: float = 12.0):
    """Times the oracle on the weight-sync workload: quantize rowwise + scale layout + byte
    comparison of whole rows of the first layer's tensors, until about budget_s of CPU work.
    Returns (GB/s of algorithmic bytes, description)."""
    import numpy as np

    import oracle
    from mxfp8_block_scaled_07_b200 import synth

    oracle.build()
    done_bytes = 0.0
    elapsed = 0.0
    rows_done = 0
    tensors = 0
    for layer, idx, r, c in sync_shapes():
        W = synth.sync_weight(layer, idx, rows=256, cols=c)    # 256 rows of the tensor (same seed recipe)
        t0 = time.perf_counter()
        q, s = oracle.quantize_rowwise(W)
        sw = oracle.swizzle(s)
        oracle.grid_equal(q, q.copy())
        oracle.grid_equal(sw, sw.copy())
        elapsed += time.perf_counter() - t0
        n = W.numel()
        done_bytes += n * QUANT_BYTES_PER_ELEM + 2 * (q.size + sw.size)
        rows_done += W.shape[0]
        tensors += 1
        if elapsed >= budget_s:
            break
    desc = (f"oracle (plain C, 1 thread): quantize+swizzle+grid_equal of the first 256 rows of {tensors} "
            f"weight tensors ({rows_done} rows, {done_bytes / 1e9:.2f} GB algorithmic) in {elapsed:.1f} s")
    return done_bytes / elapsed / 1e9, desc


def _oracle_tensor_job(job):
    """One tensor's oracle work in a worker process: returns (algorithmic bytes, seconds)."""
    import oracle
    from mxfp8_block_scaled_07_b200 import synth

    layer, idx, c = job
    W = synth.sync_weight(layer, idx, rows=256, cols=c)
    t0 = time.perf_counter()
    q, s = oracle.quantize_rowwise(W)
    sw = oracle.swizzle(s)
    oracle.grid_equal(q, q.copy())
    oracle.grid_equal(sw, sw.copy())
    dt = time.perf_counter() - t0
    return W.numel() * QUANT_BYTES_PER_ELEM + 2 * (q.size + sw.size), dt


def _warm_worker(_):
    import oracle

    oracle._load()
    return os.getpid()


def host_cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sync_sample_parallel(max_procs: int = 16):
    """The same per-tensor oracle work as oracle_sync_sample (256 rows of every one of the 144
    tensors), spread over worker processes (spawned: this runs after GPU work). Every job times
    only its own oracle calls while the others run beside it, so memory contention is included;
    the job's GB/s = bytes / (summed job seconds / processes). Returns (GB/s, processes, text)."""
    import multiprocessing as mp

    import oracle

    oracle.build()
    procs = max(1, min(max_procs, len(os.sched_getaffinity(0))))
    jobs = [(layer, idx, c) for layer, idx, _, c in sync_shapes()]
    with mp.get_context("spawn").Pool(procs) as pool:
        pool.map(_warm_worker, range(procs))
        res = pool.map(_oracle_tensor_job, jobs, chunksize=1)
    total_bytes = sum(b for b, _ in res)
    cpu_s = sum(t for _, t in res)
    gbs = total_bytes / (cpu_s / procs) / 1e9
    desc = (f"oracle (plain C) in {procs} processes on {host_cpu_model()}: quantize+swizzle+grid_equal of "
            f"the first 256 rows of all 144 weight tensors ({total_bytes / 1e9:.2f} GB algorithmic), "
            f"{cpu_s:.1f} s of summed job time")
    return gbs, procs, desc


def oracle_gemm_sample(rows: int = 2):
    """The oracle GEMM (plain fp64 C, one thread) on a row sample of the dense forward config
    (10300 x 24576 x 4096): `rows` full output rows. Returns (FLOP/s, description with the
    full-size time extrapolated from it)."""
    import oracle
    from mxfp8_block_scaled_07_b200 import synth

    oracle.build()
    X = synth.fwd_activations(rows)                   # the first rows of the forward activations
    W = synth.sync_weight(0, 2)                        # gate_up 24576 x 4096
    qx, sx = oracle.quantize_rowwise(X)
    qw, sw = oracle.quantize_rowwise(W)
    t0 = time.perf_counter()
    oracle.gemm(qx, sx, qw, sw)
    dt = time.perf_counter() - t0
    flops = 2.0 * rows * W.shape[0] * W.shape[1]
    full = 2.0 * 10300 * W.shape[0] * W.shape[1] / (flops / dt)
    return flops / dt, (f"oracle GEMM (plain C, fp64, 1 thread): {rows} full rows of fwd 10300x24576x4096 in "
                        f"{dt:.1f} s; full size extrapolated: {full / 3600:.1f} h")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    steps, warmup = args.steps, args.warmup
    per = max(2.0, 60.0 / max(1, steps + warmup))     # bounded CPU work per step
    for _ in range(warmup):
        oracle_sync_sample(budget_s=min(per, 3.0))
    vals = []
    t0 = time.perf_counter()
    desc = ""
    for _ in range(steps):
        v, desc = oracle_sync_sample(budget_s=per)
        vals.append(v)
    wall = time.perf_counter() - t0
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": args.gpus,
        "steps": steps, "warmup": warmup, "ms_per_step": round(wall / steps * 1e3, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample": "bounded row sample per step"},
        "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------------

class SyncWorkload:
    """Device-resident weights, learner outputs and the sampler's copy for one rank."""

    def __init__(self, rank: int, device):
        import torch

        from mxfp8_block_scaled_07_b200 import mx, synth

        self.items = []
        L = mx.lib()
        self.total_elems = 0
        self.compare_bytes = 0
        for layer, idx, r, c in sync_shapes():
            W = synth.normal_bf16((r, c), std=0.02, seed=rank_seed(layer, idx, rank), device=device,
                                  outlier_frac=1e-3, outlier_scale=50.0)
            # Sampler copy: dequantize the learner's grid to BF16 (exact here: every scale >= 2^-124)
            # and let the sampler re-derive elements and the tensor-core scale layout from it.
            q0, s0, _, _ = mx.quantize(W, True, False, swizzle=False)
            deq = (q0.view(torch.float8_e4m3fn).float() *
                   torch.exp2(s0.float() - 127.0).repeat_interleave(32, dim=1)).to(torch.bfloat16)
            del q0, s0
            qs, ss, _, _ = mx.quantize(deq, True, False, swizzle=True)
            del deq
            q = torch.empty_like(qs)
            s = torch.empty_like(ss)
            self.items.append((W, q, s, qs, ss))
            self.total_elems += W.numel()
            self.compare_bytes += 2 * (q.numel() + s.numel())
        torch.cuda.synchronize()
        # Pair 2i: elements of tensor i; pair 2i + 1: its swizzled scales. results[0] = mismatch
        # counts, results[1] = first indices.
        self.results = torch.zeros((2, 2 * len(self.items)), dtype=torch.int64, device=device)
        # Pre-marshalled C-ABI arguments (plain pointers and sizes): one multi-tensor quantization
        # of all weights and one multi-pair byte comparison per step.
        self.qarr = mx.quant_tensor_array([it[0] for it in self.items],
                                          [(q, s, None, None) for (_, q, s, _, _) in self.items])
        pairs = []
        for (_, q, s, qs, ss) in self.items:
            pairs += [(q, qs), (s, ss)]
        self.parr = mx.compare_pair_array(pairs)
        self.n_pairs = len(pairs)
        self.L = L
        self.quant_bytes = self.total_elems * QUANT_BYTES_PER_ELEM
        self.step_bytes = self.quant_bytes + self.compare_bytes

    LAUNCHES_PER_STEP = 3      # mx_quantize_multi: 1 launch; mx_grid_equal_multi: reset + compare

    def quantize_all(self, sp):
        st = self.L.mx_quantize_multi(ctypes.cast(self.qarr, ctypes.c_void_p), len(self.items), 1 | 4, sp)
        if st:
            raise RuntimeError(f"mx_quantize_multi failed: {st}")

    def compare_all(self, sp):
        st = self.L.mx_grid_equal_multi(ctypes.cast(self.parr, ctypes.c_void_p), self.n_pairs,
                                        ctypes.c_void_p(self.results[0].data_ptr()),
                                        ctypes.c_void_p(self.results[1].data_ptr()), sp)
        if st:
            raise RuntimeError(f"mx_grid_equal_multi failed: {st}")

    def step(self, stream_ptr, ev_q0=None, ev_q1=None, ev_c1=None, stream=None):
        sp = ctypes.c_void_p(stream_ptr)
        if ev_q0 is not None:
            ev_q0.record(stream)
        self.quantize_all(sp)
        if ev_q1 is not None:
            ev_q1.record(stream)
        self.compare_all(sp)
        if ev_c1 is not None:
            ev_c1.record(stream)


def run_fused_sync(wl, stream, step_ms, quant_ms, cmp_ms, steps=10):
    """The same synchronization check through mx_quantize_compare_multi: one pass quantizes the 144
    weights (the same grid) and compares what it writes with the sampler's copy, instead of a
    quantize launch followed by a compare launch that reads the written grid back."""
    import torch

    from mxfp8_block_scaled_07_b200 import mx

    refs = (mx.GridRef * len(wl.items))()
    for i, (_, _, _, qs, ss) in enumerate(wl.items):
        refs[i] = mx.GridRef(qs.data_ptr(), ss.data_ptr())
    res = torch.empty((2, 2 * len(wl.items)), dtype=torch.int64, device=wl.results.device)
    sp = ctypes.c_void_p(stream.cuda_stream)

    def call():
        st = wl.L.mx_quantize_compare_multi(ctypes.cast(wl.qarr, ctypes.c_void_p), ctypes.cast(refs, ctypes.c_void_p),
                                            len(wl.items), ctypes.c_void_p(res[0].data_ptr()),
                                            ctypes.c_void_p(res[1].data_ptr()), sp)
        if st:
            raise RuntimeError(f"mx_quantize_compare_multi failed: {st}")

    for _ in range(3):
        call()
    mx.device_error()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):          # 28 GB touched per call: far beyond L2, no flush needed
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    fused_ms = e0.elapsed_time(e1) / steps
    ref_bytes = wl.compare_bytes / 2
    fused_bytes = wl.quant_bytes + ref_bytes           # BF16 read + grid written + sampler copy read
    out = {"workload": "qwen3-8b weight sync, 144 tensors: quantize + byte check in one pass "
                       "(mx_quantize_compare_multi) against the quantize launch + compare launch step",
           "fused_ms": round(fused_ms, 4), "two_launch_step_ms": round(step_ms, 4),
           "two_launch_quantize_ms": round(quant_ms, 4), "two_launch_compare_ms": round(cmp_ms, 4),
           "speedup": round(step_ms / fused_ms, 3),
           "fused_algorithmic_gb": round(fused_bytes / 1e9, 3),
           "fused_gbs": round(fused_bytes / (fused_ms * 1e-3) / 1e9, 1),
           "mismatches": int(res[0].sum().item()),
           "results_equal_two_launch": bool(torch.equal(res[0], wl.results[0]) and torch.equal(res[1], wl.results[1]))}
    out.update(device_status())
    return out


def dist_setup(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    return world, rank, local, pg


def barrier_sync(pg):
    import torch

    torch.cuda.synchronize()
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()


def max_over_ranks(pg, value: float, device="cuda") -> float:
    """The slowest rank's time: the job's time (every rank does the same work, weak scaling)."""
    if pg is None:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(pg, value: int, device="cuda") -> int:
    if pg is None:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.int64, device=device)
    pg.all_reduce(t)
    return int(t.item())


def job_throughput_gbs(world: int, bytes_per_rank_step: int, ms_max: float) -> float:
    """Whole-job GB/s: the bytes all ranks processed in one step over the slowest rank's step time."""
    return world * bytes_per_rank_step / (ms_max * 1e-3) / 1e9


def rank_seed(layer: int, idx: int, rank: int) -> int:
    """Seed of one weight tensor of one rank: every rank synchronizes its own 144 tensors."""
    return layer * 4 + idx + 144 * rank


def traffic_record():
    """DRAM bytes per element of the multi-tensor quantize launch from a committed ncu summary,
    valid only while the kernel source is unchanged (sha256 of quantize.cuh, which holds the whole
    kernel and its device helpers)."""
    import hashlib

    p = os.path.join(ROOT, "profiles", "quantize_rowwise_traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    h = hashlib.sha256()
    for f in ("quantize.cuh",):
        with open(os.path.join(ROOT, "mxfp8_block_scaled_07_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    if rec.get("source_sha256") != h.hexdigest():
        return None
    return rec


E2E_CHUNK = 16          # tensors per pipeline chunk of the end-to-end step


def run_e2e(wl, args, device):
    """Same metric through the C ABI with host buffers: per step, every BF16 weight goes
    host(pinned) -> device, is quantized and compared on the device, and the learner grid (elements
    + swizzled scales) and the comparison results come back to pinned host memory. The 144 tensors
    move in chunks of E2E_CHUNK on three streams (copies in, kernels, copies out), so chunk c's
    kernels overlap chunk c+1's upload and chunk c-1's download; each chunk is one
    mx_quantize_multi and one mx_grid_equal_multi call. A chunk's device buffers are reused by the
    next step only after its kernels (for the upload) and its download (for the kernels) are done."""
    import torch

    s_in, s_k, s_out = (torch.cuda.Stream(device) for _ in range(3))
    host_w = [W.cpu().pin_memory() for (W, _, _, _, _) in wl.items]
    host_q = [torch.empty(q.shape, dtype=torch.uint8).pin_memory() for (_, q, _, _, _) in wl.items]
    host_s = [torch.empty(s.shape, dtype=torch.uint8).pin_memory() for (_, _, s, _, _) in wl.items]
    host_r = torch.empty(wl.results.shape, dtype=torch.int64).pin_memory()
    h2d = sum(t.numel() * 2 for t in host_w)
    d2h = sum(t.numel() for t in host_q) + sum(t.numel() for t in host_s) + host_r.numel() * 8
    n = len(wl.items)
    chunks = [(i0, min(n, i0 + E2E_CHUNK)) for i0 in range(0, n, E2E_CHUNK)]
    from mxfp8_block_scaled_07_b200 import mx

    qarrs = [mx.quant_tensor_array([it[0] for it in wl.items[i0:i1]], [(q, s, None, None) for (_, q, s, _, _) in
                                                                      wl.items[i0:i1]]) for i0, i1 in chunks]
    parrs = []
    for i0, i1 in chunks:
        pairs = []
        for (_, q, s, qs, ss) in wl.items[i0:i1]:
            pairs += [(q, qs), (s, ss)]
        parrs.append(mx.compare_pair_array(pairs))
    done_k = [None] * len(chunks)       # kernels of chunk c finished (its inputs may be overwritten)
    done_out = [None] * len(chunks)     # download of chunk c finished (its outputs may be overwritten)

    def one_step():
        for c, (i0, i1) in enumerate(chunks):
            if done_k[c] is not None:
                s_in.wait_event(done_k[c])
            with torch.cuda.stream(s_in):
                for i in range(i0, i1):
                    wl.items[i][0].copy_(host_w[i], non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
            s_k.wait_event(ev_in)
            if done_out[c] is not None:
                s_k.wait_event(done_out[c])
            sk = ctypes.c_void_p(s_k.cuda_stream)
            st = wl.L.mx_quantize_multi(ctypes.cast(qarrs[c], ctypes.c_void_p), i1 - i0, 1 | 4, sk)
            if st:
                raise RuntimeError(f"mx_quantize_multi failed: {st}")
            st = wl.L.mx_grid_equal_multi(ctypes.cast(parrs[c], ctypes.c_void_p), 2 * (i1 - i0),
                                          ctypes.c_void_p(wl.results[0, 2 * i0:].data_ptr()),
                                          ctypes.c_void_p(wl.results[1, 2 * i0:].data_ptr()), sk)
            if st:
                raise RuntimeError(f"mx_grid_equal_multi failed: {st}")
            done_k[c] = torch.cuda.Event()
            done_k[c].record(s_k)
            s_out.wait_event(done_k[c])
            with torch.cuda.stream(s_out):
                for i in range(i0, i1):
                    host_q[i].copy_(wl.items[i][1], non_blocking=True)
                    host_s[i].copy_(wl.items[i][2], non_blocking=True)
                for row in range(2):
                    host_r[row, 2 * i0:2 * i1].copy_(wl.results[row, 2 * i0:2 * i1], non_blocking=True)
            done_out[c] = torch.cuda.Event()
            done_out[c].record(s_out)

    one_step()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 3))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for _ in range(steps):
        one_step()
    e1.record(s_out)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    ok = int(host_r[0].sum()) == 0
    del host_w, host_q, host_s
    return {"value": round(wl.step_bytes / (ms * 1e-3) / 1e9, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 2), "steps": steps, "grid_equal": ok,
            "pipeline": f"{len(chunks)} chunks of <= {E2E_CHUNK} tensors on 3 streams (copy in, kernels, copy out)"}


def aggregate_e2e(pg, local: dict, world: int, bytes_per_rank_step: int, device="cuda") -> dict:
    """Whole-job end-to-end figures from each rank's run_e2e: the slowest rank's step time, all
    ranks' bytes, and grid equality on every rank."""
    ms = max_over_ranks(pg, local["ms_per_step"], device=device)
    bad = sum_over_ranks(pg, 0 if local["grid_equal"] else 1, device=device)
    return {"value": round(job_throughput_gbs(world, bytes_per_rank_step, ms), 2), "unit": UNIT,
            "h2d_bytes_per_step": world * local["h2d_bytes_per_step"],
            "d2h_bytes_per_step": world * local["d2h_bytes_per_step"],
            "ms_per_step": round(ms, 2), "steps": local["steps"], "grid_equal": bad == 0}


def flush_l2(buf):
    """Evicts the timed kernel's data from L2 before a timed launch: writes a buffer larger than L2,
    then reads a second one, so that the written lines are written back here and not during the
    timed launch (a flush that only writes leaves up to 126 MB of dirty lines that the next kernel
    pays to write back). `buf` holds both halves."""
    h = buf.numel() // 2
    buf[:h].add_(1)
    buf[h:].sum()


def time_gpu(fn, reps, flush_buf, stream):
    """Median CUDA-event time (ms) of fn over reps runs, L2 flushed before each. The wall-clock
    window of the runs is kept in time_gpu.window (for the clock samples taken meanwhile)."""
    import torch

    times = []
    t_start = time.monotonic()
    for _ in range(reps):
        flush_l2(flush_buf)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    time_gpu.window = (t_start, time.monotonic())
    return statistics.median(times)


def device_status() -> dict:
    """Reads and clears libmx's device status word after a timed region (synchronizes). A set bit
    means some launch stopped early (an expired bounded wait, bad grouped offsets), so the time
    beside it does not measure the whole computation: the line is then marked invalid."""
    from mxfp8_block_scaled_07_b200 import mx

    bits = mx.device_error()
    return {"device_error": bits, "invalid": True} if bits else {"device_error": 0}


def scaled_mm_fn(qa, sa, qb, sb):
    """cuBLAS MXFP8 GEMM through torch `scaled_mm` (BlockWise1x32 scales in the SWIZZLE_32_4_4
    layout) on this library's bytes and swizzled scales, BF16 out; None if torch lacks the path."""
    import torch
    import torch.nn.functional as F

    try:
        fa, fb = qa.view(torch.float8_e4m3fn), qb.view(torch.float8_e4m3fn).t()
        ea, eb = sa.view(torch.float8_e8m0fnu), sb.view(torch.float8_e8m0fnu)
        return lambda: F.scaled_mm(fa, fb, ea, F.ScalingType.BlockWise1x32, eb, F.ScalingType.BlockWise1x32,
                                   swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                                   output_dtype=torch.bfloat16)
    except (AttributeError, TypeError):
        return None


def scaled_grouped_mm_fn(qa, sa_grp, qb, sb, row_offsets):
    """torch `scaled_grouped_mm` (MXFP8, BlockWise1x32 scales in the SWIZZLE_32_4_4 layout) on this
    library's bytes: A [rows, K] with its grouped scale layout (each expert padded to 128 rows) as a
    2-D [padded rows, padded K/32] tensor, B [G, N, K] seen as [G, K, N] with its G per-expert
    layouts as [G, bytes per expert]; group ends from the row offsets. None if torch lacks it."""
    import torch
    import torch.nn.functional as F

    try:
        G, N, K = qb.shape
        kb_pad = (K // 32 + 3) // 4 * 4
        fa, fb = qa.view(torch.float8_e4m3fn), qb.view(torch.float8_e4m3fn).transpose(-2, -1)
        ea = sa_grp.view(torch.float8_e8m0fnu).reshape(-1, kb_pad)
        eb = sb.view(torch.float8_e8m0fnu).reshape(G, -1)
        ends = row_offsets[1:].contiguous()
        return lambda: F.scaled_grouped_mm(fa, fb, ea, F.ScalingType.BlockWise1x32, eb, F.ScalingType.BlockWise1x32,
                                           swizzle_a=F.SwizzleType.SWIZZLE_32_4_4,
                                           swizzle_b=F.SwizzleType.SWIZZLE_32_4_4, offs=ends,
                                           output_dtype=torch.bfloat16)
    except (AttributeError, TypeError):
        return None


def cublas_line(fn, flops, reps, flush, stream, key="cublas") -> dict:
    """Times a library MXFP8 GEMM on the same bytes; keys <key>_mxfp8_tflops / <key>_ms."""
    try:
        fn()
        ms = time_gpu(fn, reps, flush, stream)
        return {f"{key}_mxfp8_tflops": round(flops / (ms * 1e-3) / 1e12, 1), f"{key}_ms": round(ms, 4)}
    except (RuntimeError, TypeError, NotImplementedError) as e:
        return {f"{key}_mxfp8_tflops": None, f"{key}_note": f"torch MXFP8 GEMM unavailable: {type(e).__name__}"}


def guarded(fn):
    """A characterization line that fails reports its error in the JSON line instead of taking
    the headline measurement down with it."""
    try:
        return fn()
    except Exception as e:  # noqa: BLE001
        return {"error": f"{type(e).__name__}: {e}"[:300]}


def run_secondary(device, peaks, reps=10):
    """GEMM TFLOP/s on the dense forward, update and MoE configs; quantize GB/s on activations.
    Each line carries the SM clock and power sampled while it was timed (`clocks`): these lines run
    after the headline, on a GPU the GEMMs have heated, and a power-capped clock moves them."""
    with ClockSampler(device.index or 0) as sampler:
        return _run_secondary(device, peaks, reps, sampler)


def _run_secondary(device, peaks, reps, sampler):
    import torch

    from mxfp8_block_scaled_07_b200 import mx, synth

    def line_clocks():
        return {"clocks": sampler.window(*time_gpu.window)}

    stream = torch.cuda.current_stream()
    flush = torch.zeros(4 * L2_BYTES // 4, dtype=torch.float32, device=device)   # 2 x (2 x L2)
    fp8_peak = peaks["bf16_tflops"] * NOMINAL_FP8_OVER_BF16
    out = {"gemm": [], "quantize": [], "swizzle": [], "fp8_peak_tflops": round(fp8_peak, 1),
           "fp8_peak_source": f"{peaks['source']} bf16 {peaks['bf16_tflops']} x nominal fp8/bf16 ratio 2",
           "spec_fp8_tflops": 4500.0}

    def add_gemm(name, flops, fn, lib_fn=None, lib_key="cublas"):
        for _ in range(2):
            fn()
        mx.device_error()                     # clear before the timed launches
        ms = time_gpu(fn, reps, flush, stream)
        tf = flops / (ms * 1e-3) / 1e12
        rec = {"workload": name, "tflops": round(tf, 1), "ms": round(ms, 4),
               "frac_of_fp8_peak": round(tf / fp8_peak, 3), "frac_of_spec_4500": round(tf / 4500.0, 3)}
        rec.update(line_clocks())
        rec.update(device_status())
        if lib_fn is not None:
            lib = cublas_line(lib_fn, flops, reps, flush, stream, lib_key)
            rec.update(lib)
            if lib.get(f"{lib_key}_mxfp8_tflops"):
                rec[f"mx_over_{lib_key}"] = round(tf / lib[f"{lib_key}_mxfp8_tflops"], 3)
        out["gemm"].append(rec)

    def add_quant(name, x, row, col):
        bufs = mx.quantize(x, row, col, swizzle=True)
        M, K = x.shape
        nbytes = M * K * 2 + (M * K + bufs[1].numel() if row else 0) + (M * K + bufs[3].numel() if col else 0)
        fn = lambda: mx.quantize(x, row, col, swizzle=True, out=bufs)
        fn()
        mx.device_error()
        ms = time_gpu(fn, reps, flush, stream)
        gbs = nbytes / (ms * 1e-3) / 1e9
        rec = {"workload": name, "gbs": round(gbs, 1), "ms": round(ms, 4),
               "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 3)}
        rec.update(line_clocks())
        rec.update(device_status())
        out["quantize"].append(rec)

    def add_swizzle(name, s_raw, groups=None):
        """Standalone scale rearrangement (Table 6): raw scales read once, the layout written once."""
        o = mx.swizzle_scales(s_raw, groups)
        fn = lambda: mx.swizzle_scales(s_raw, groups, out=o)
        fn()
        mx.device_error()
        ms = time_gpu(fn, reps, flush, stream)
        gbs = (s_raw.numel() + o.numel()) / (ms * 1e-3) / 1e9
        rec = {"workload": name, "gbs": round(gbs, 1), "ms": round(ms, 4), "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 3)}
        rec.update(line_clocks())
        rec.update(device_status())
        out["swizzle"].append(rec)

    # Dense forward linear (Table 5 micro-batch token counts) against gate_up.
    W = synth.sync_weight(0, 2, device=device)
    qw, sw, _, _ = mx.quantize(W, True, False)
    add_swizzle("gate_up weight scales 24576x128", mx.quantize(W, True, False, swizzle=False)[1])
    for M in synth.FWD_TOKENS:
        X = synth.fwd_activations(M, device=device)
        add_quant(f"fwd activations {M}x4096 rowwise", X, True, False)
        qx, sx, _, _ = mx.quantize(X, True, False)
        C = torch.empty((M, W.shape[0]), dtype=torch.bfloat16, device=device)
        add_gemm(f"fwd {M}x24576x4096 bf16-out", 2.0 * M * W.shape[0] * W.shape[1],
                 lambda: mx.gemm(qx, sx, qw, sw, out=C), scaled_mm_fn(qx, sx, qw, sw))
        del X, qx, sx, C
    del W, qw, sw
    # Update micro-batch (12288 tokens): row + col quantization, fprop / dgrad / wgrad.
    X, Wu, dY = synth.update_inputs(device=device)
    add_quant("update dY 12288x12288 row+col", dY, True, True)
    qx = mx.quantize(X, True, True)
    qwu = mx.quantize(Wu, True, True)
    qd = mx.quantize(dY, True, True)
    T, H, O = X.shape[0], X.shape[1], Wu.shape[0]
    Y = torch.empty((T, O), dtype=torch.bfloat16, device=device)
    dX = torch.empty((T, H), dtype=torch.bfloat16, device=device)
    dW = torch.empty((O, H), dtype=torch.bfloat16, device=device)
    add_gemm("update fprop 12288x12288x4096", 2.0 * T * O * H, lambda: mx.gemm(qx[0], qx[1], qwu[0], qwu[1], out=Y),
             scaled_mm_fn(qx[0], qx[1], qwu[0], qwu[1]))
    add_gemm("update dgrad 12288x4096x12288", 2.0 * T * H * O, lambda: mx.gemm(qd[0], qd[1], qwu[2], qwu[3], out=dX),
             scaled_mm_fn(qd[0], qd[1], qwu[2], qwu[3]))
    add_gemm("update wgrad 12288x4096x12288", 2.0 * O * H * T, lambda: mx.gemm(qd[2], qd[3], qx[2], qx[3], out=dW),
             scaled_mm_fn(qd[2], qd[3], qx[2], qx[3]))
    del X, Wu, dY, qx, qwu, qd, Y, dX, dW
    # MoE layer: grouped gate_up and down.
    counts, Xp, Hh, W1, W2 = synth.moe_inputs(device=device)
    counts = [int(c) for c in counts]
    offs = torch.tensor(synth.group_offsets(counts), dtype=torch.int32, device=device)
    rows = sum(counts)
    add_quant(f"moe X_perm {rows}x2048 rowwise", Xp, True, False)
    for name, A, Wt in (("moe gate_up", Xp, W1), ("moe down", Hh, W2)):
        G, N, K = Wt.shape
        qa, sa_raw, _, _ = mx.quantize(A, True, False, swizzle=False)
        sa = mx.swizzle_scales(sa_raw, counts)
        add_swizzle(f"{name} A scales {rows}x{K // 32} grouped (128 experts, each padded to 128 rows)", sa_raw,
                    counts)
        qb, sb, _, _ = mx.quantize(Wt.reshape(G * N, K), True, False)
        qb = qb.reshape(G, N, K)
        C = torch.empty((rows, N), dtype=torch.bfloat16, device=device)
        add_gemm(f"{name} grouped {rows}x{N}x{K} (128 experts)", 2.0 * rows * N * K,
                 lambda: mx.grouped_gemm(qa, sa, qb, sb, offs, out=C), scaled_grouped_mm_fn(qa, sa, qb, sb, offs),
                 "torch_grouped")
        del qa, sa_raw, sa, qb, sb, C
    # FP8-blockwise grids of one weight (128 x 128 blocks): FP32 scales (the sampler's) against
    # power-of-two scales (the learner's on SM100), beside the MXFP8 grid both sides share here.
    W = synth.sync_weight(0, 2, device=device)
    Mw, Kw = W.shape
    g32 = mx.quantize_block128(W, False)
    g2 = mx.quantize_block128(W, True)
    ms32 = time_gpu(lambda: mx.quantize_block128(W, False, out=g32), reps, flush, stream)
    ms2 = time_gpu(lambda: mx.quantize_block128(W, True, out=g2), reps, flush, stream)
    cnt, _ = mx.grid_equal(g32[0], g2[0])

    def deq_block(q, sc):
        return q.view(torch.float8_e4m3fn).float() * sc.repeat_interleave(128, 0)[:Mw].repeat_interleave(128, 1)[:, :Kw]

    qm, sm, _, _ = mx.quantize(W, True, False, swizzle=False)
    dm = qm.view(torch.float8_e4m3fn).float() * torch.exp2(sm.float() - 127.0).repeat_interleave(32, dim=1)
    d32, d2, ref = deq_block(*g32), deq_block(*g2), W.float()
    bw_bytes = Mw * Kw * 3 + 4 * (Mw // 128) * (Kw // 128)
    out["fp8_blockwise_gap"] = {
        "workload": f"qwen3-8b gate_up {Mw}x{Kw}: FP8 blockwise (128x128) with FP32 vs power-of-two scales",
        "byte_mismatch_frac": round(int(cnt.item()) / (Mw * Kw), 4),
        "rel_diff_between_grids": round(float((d32 - d2).norm() / d32.norm()), 5),
        "rel_err_fp32_scales": round(float((d32 - ref).norm() / ref.norm()), 5),
        "rel_err_pow2_scales": round(float((d2 - ref).norm() / ref.norm()), 5),
        "rel_err_mxfp8": round(float((dm - ref).norm() / ref.norm()), 5),
        "quantize_gbs": {"fp32_scales": round(bw_bytes / (ms32 * 1e-3) / 1e9, 1),
                         "pow2_scales": round(bw_bytes / (ms2 * 1e-3) / 1e9, 1)}}
    del W, g32, g2, qm, sm, dm, d32, d2, ref
    # gate_up with SwiGLU and the down GEMM's MXFP8 quantization fused into the epilogue, against the
    # unfused chain (gate_up GEMM to BF16, SwiGLU in torch, quantize + grouped scale layout).
    G, N2, K = W1.shape
    n = N2 // 2
    qa, sa_raw, _, _ = mx.quantize(Xp, True, False, swizzle=False)
    sa = mx.swizzle_scales(sa_raw, counts)
    W1i = W1.view(G, 2, n // 128, 128, K).permute(0, 2, 1, 3, 4).reshape(G * N2, K).contiguous()
    qbi, sbi, _, _ = mx.quantize(W1i, True, False)
    qbi = qbi.reshape(G, N2, K)
    hq = mx.grouped_gemm_swiglu_quant(qa, sa, qbi, sbi, offs, counts)
    mx.device_error()
    fused_ms = time_gpu(lambda: mx.grouped_gemm_swiglu_quant(qa, sa, qbi, sbi, offs, counts, out=hq), reps, flush,
                        stream)
    fused_status = device_status()
    qb, sb, _, _ = mx.quantize(W1.reshape(G * N2, K), True, False)
    qb = qb.reshape(G, N2, K)
    C = torch.empty((rows, N2), dtype=torch.bfloat16, device=device)
    hbuf = mx.quantize(torch.empty((rows, n), dtype=torch.bfloat16, device=device), True, False, swizzle=False)
    hs = torch.empty(mx.grouped_swizzled_scale_bytes(counts, n // 32), dtype=torch.uint8, device=device)

    def unfused():
        mx.grouped_gemm(qa, sa, qb, sb, offs, out=C)
        h = (torch.nn.functional.silu(C[:, :n].float()) * C[:, n:].float()).to(torch.bfloat16)
        mx.quantize(h, True, False, swizzle=False, out=hbuf)
        mx.swizzle_scales(hbuf[1], counts, out=hs)

    unfused()
    unfused_ms = time_gpu(unfused, reps, flush, stream)
    flops = 2.0 * rows * N2 * K
    out["moe_gate_up_swiglu_quant"] = {
        "workload": f"moe gate_up {rows}x{N2}x{K} + SwiGLU + MXFP8 quantize of h (128 experts)",
        "fused_ms": round(fused_ms, 4), "fused_tflops": round(flops / (fused_ms * 1e-3) / 1e12, 1),
        "unfused_ms": round(unfused_ms, 4),
        "unfused": "mx_grouped_gemm (BF16 out) + torch SwiGLU + mx_quantize + mx_swizzle_scales",
        "speedup": round(unfused_ms / fused_ms, 3), **fused_status}
    del qa, sa_raw, sa, W1i, qbi, sbi, hq, qb, sb, C, hbuf, hs
    del Xp, Hh, W1, W2
    torch.cuda.synchronize()
    return out


def run_library_gemm_peak(device, reps=10):
    """Dense MXFP8 reference points at 8192^3, BF16 out: cuBLAS through torch `scaled_mm`
    (BlockWise1x32 scales in the SWIZZLE_32_4_4 layout, fed with this library's bytes) and mx_gemm
    on the same operands."""
    import torch
    import torch.nn.functional as F

    from mxfp8_block_scaled_07_b200 import mx, synth

    n = 8192
    stream = torch.cuda.current_stream()
    flush = torch.zeros(4 * L2_BYTES // 4, dtype=torch.float32, device=device)   # 2 x (2 x L2)
    A = synth.normal_bf16((n, n), std=1.0, seed=51, device=device)
    B = synth.normal_bf16((n, n), std=1.0, seed=52, device=device)
    qa, sa, _, _ = mx.quantize(A, True, False)
    qb, sb, _, _ = mx.quantize(B, True, False)
    del A, B
    C = torch.empty((n, n), dtype=torch.bfloat16, device=device)
    flops = 2.0 * n * n * n
    out = {"shape": "8192x8192x8192 bf16-out"}
    mx.gemm(qa, sa, qb, sb, out=C)
    mx.device_error()
    ms = time_gpu(lambda: mx.gemm(qa, sa, qb, sb, out=C), reps, flush, stream)
    out["mx_gemm_tflops"] = round(flops / (ms * 1e-3) / 1e12, 1)
    out.update(device_status())
    try:
        fa, fb = qa.view(torch.float8_e4m3fn), qb.view(torch.float8_e4m3fn).t()
        ea, eb = sa.view(torch.float8_e8m0fnu), sb.view(torch.float8_e8m0fnu)
        fn = lambda: F.scaled_mm(fa, fb, ea, F.ScalingType.BlockWise1x32, eb, F.ScalingType.BlockWise1x32,
                                 swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                                 output_dtype=torch.bfloat16)
        fn()
        ms = time_gpu(fn, reps, flush, stream)
        out["cublas_mxfp8_tflops"] = round(flops / (ms * 1e-3) / 1e12, 1)
    except (RuntimeError, TypeError, NotImplementedError, AttributeError) as e:
        out["cublas_mxfp8_tflops"] = None
        out["cublas_note"] = f"torch scaled_mm MXFP8 unavailable: {type(e).__name__}"
    torch.cuda.synchronize()
    return out


# The pages' micro-batch sweep (Table 5: 1.3k / 2.6k / 5.2k / 10.3k tokens) rounded to multiples of
# 32 (the columnwise copy of the wgrad operands needs it), plus 512 / 3.9k / 7.7k to pin the fit.
BREAKEVEN_TOKENS = (512, 1312, 2592, 3904, 5216, 7744, 10304)
BREAKEVEN_PASSES = 3


def fit_line(xs, ys):
    """Least-squares t = delta + c * x; returns (delta, c)."""
    n = len(xs)
    mx_, my = sum(xs) / n, sum(ys) / n
    c = sum((x - mx_) * (y - my) for x, y in zip(xs, ys)) / sum((x - mx_) ** 2 for x in xs)
    return my - c * mx_, c


def breakeven_fit(points):
    """The pages' stage cost model t = delta + c * tokens fitted per path over one sweep, and the
    break-even tokens per micro-batch m* = (delta_mxfp8 - delta_bf16) / (c_bf16 - c_mxfp8). When the
    points carry the paired difference "diff_ms" (MXFP8 - BF16, measured replay by replay), the
    difference line is fitted directly: d = d_delta - d_c * tokens."""
    xs = [p["tokens"] for p in points]
    d_b, c_b = fit_line(xs, [p["bf16_ms"] for p in points])
    d_m, c_m = fit_line(xs, [p["mxfp8_ms"] for p in points])
    if all("diff_ms" in p for p in points):
        dd, neg_dc = fit_line(xs, [p["diff_ms"] for p in points])
        dc = -neg_dc
    else:
        dd, dc = d_m - d_b, c_b - c_m
    return {"bf16": {"delta_ms": round(d_b, 4), "c_us_per_token": round(c_b * 1e3, 5)},
            "mxfp8": {"delta_ms": round(d_m, 4), "c_us_per_token": round(c_m * 1e3, 5)},
            "delta_delta_ms": round(dd, 4), "delta_c_us_per_token": round(dc * 1e3, 5),
            "m_star_tokens": (round(dd / dc, 1) if dc > 0 else None)}


def run_breakeven(device, reps=20, passes=BREAKEVEN_PASSES):
    """Kernel-level fixed cost and per-token cost of one update micro-batch of a Qwen3-8B linear
    (W 12288 x 4096, the TP-2 gate_up shard): BF16 (cuBLAS fprop, dgrad, wgrad) against MXFP8
    (X and dY quantized row+col with the scale layout in one multi-tensor launch, then the three
    MXFP8 GEMMs), each micro-batch one CUDA graph, L2 flushed before each replay. At each token count the two paths' replays
    alternate one by one (the SM clock moves with the power cap, and pairing puts both paths under
    the same conditions); the sweep is repeated `passes` times. Per pass the pages' stage cost model
    t = delta + c * tokens (Table 7) is fitted to each path, and the paired difference MXFP8 - BF16
    to a line d_delta - d_c * tokens, whose root m* = d_delta / d_c is the break-even tokens per
    micro-batch; the result is the fit over all passes' per-point medians, with each pass's m*
    beside it. The weight's own quantization happens once per optimizer step, not per micro-batch,
    and is reported beside the fit."""
    import torch

    from mxfp8_block_scaled_07_b200 import mx, synth

    stream = torch.cuda.Stream(device)
    cur = torch.cuda.current_stream()
    flush = torch.zeros(4 * L2_BYTES // 4, dtype=torch.float32, device=device)   # 2 x (2 x L2)
    O, H = 12288, 4096
    W = synth.normal_bf16((O, H), std=0.02, seed=61, device=device)
    qw = mx.quantize(W, True, True)
    wq_ms = time_gpu(lambda: mx.quantize(W, True, True, out=qw), reps, flush, cur)
    graphs = {}               # tokens -> (bf16 graph, mxfp8 graph); buffers kept alive in `keep`
    keep = []
    for T in BREAKEVEN_TOKENS:
        X = synth.normal_bf16((T, H), std=1.0, seed=62, device=device)
        dY = synth.normal_bf16((T, O), std=1e-3, seed=63, device=device)
        Y = torch.empty((T, O), dtype=torch.bfloat16, device=device)
        dX = torch.empty((T, H), dtype=torch.bfloat16, device=device)
        dW = torch.empty((O, H), dtype=torch.bfloat16, device=device)
        qx = mx.quantize(X, True, True)
        qd = mx.quantize(dY, True, True)
        keep.append((X, dY, Y, dX, dW, qx, qd))

        def bf16_step(X=X, dY=dY, Y=Y, dX=dX, dW=dW):
            torch.matmul(X, W.t(), out=Y)
            torch.matmul(dY, W, out=dX)
            torch.matmul(dY.t(), X, out=dW)

        def mxfp8_step(X=X, dY=dY, Y=Y, dX=dX, dW=dW, qx=qx, qd=qd):
            mx.quantize_multi([X, dY], True, True, swizzle=True, outs=[qx, qd])   # one launch for both
            mx.gemm(qx[0], qx[1], qw[0], qw[1], out=Y)
            mx.gemm(qd[0], qd[1], qw[2], qw[3], out=dX)
            mx.gemm(qd[2], qd[3], qx[2], qx[3], out=dW)

        pair = []
        for fn in (bf16_step, mxfp8_step):
            with torch.cuda.stream(stream):
                fn()                                  # warm-up outside capture
            stream.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                fn()
            pair.append(g)
        graphs[T] = pair
    torch.cuda.synchronize()
    mx.device_error()

    def one(g):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(cur)
        g.replay()
        e1.record(cur)
        e1.synchronize()
        return e0.elapsed_time(e1)

    per_pass = []
    for _ in range(passes):
        pts = []
        for T in BREAKEVEN_TOKENS:
            gb, gm = graphs[T]
            one(gb), one(gm)
            tb, tm = [], []
            for _ in range(reps):
                tb.append(one(gb))
                tm.append(one(gm))
            pts.append({"tokens": T, "bf16_ms": round(statistics.median(tb), 4),
                        "mxfp8_ms": round(statistics.median(tm), 4),
                        "diff_ms": round(statistics.median(m - b for b, m in zip(tb, tm)), 4)})
        per_pass.append(pts)
    status = device_status()
    del graphs, keep
    torch.cuda.synchronize()
    fits = [breakeven_fit(p) for p in per_pass]
    med = [{"tokens": T, **{k: round(statistics.median(p[i][k] for p in per_pass), 4)
                            for k in ("bf16_ms", "mxfp8_ms", "diff_ms")}}
           for i, T in enumerate(BREAKEVEN_TOKENS)]
    out = {"linear": "W 12288x4096 (fprop, dgrad, wgrad per micro-batch)", "points": med, **breakeven_fit(med)}
    ms_ = [f["m_star_tokens"] for f in fits if f["m_star_tokens"] is not None]
    out["m_star_per_pass"] = [f["m_star_tokens"] for f in fits]
    out["delta_delta_ms_per_pass"] = [f["delta_delta_ms"] for f in fits]
    out["delta_c_us_per_token_per_pass"] = [f["delta_c_us_per_token"] for f in fits]
    if ms_:
        out["m_star_range"] = [min(ms_), max(ms_)]
    out["weight_quantize_row_col_ms_per_step"] = round(wq_ms, 4)
    out["timing"] = (f"one CUDA graph per micro-batch and path; BF16 and MXFP8 replays alternated, {reps} pairs per "
                     f"point and pass, {passes} passes, L2 flushed before each replay; m* from the paired "
                     "difference line fitted to the per-point medians over passes")
    out.update(status)
    return out


CASES = ("quant-gate-up", "quant-dy-rowcol", "quant-dy-col", "quant-sync-subset", "quant-fwd-1300", "gemm-fwd-10300",
         "gemm-update-fprop", "gemm-update-dgrad", "gemm-moe-gate-up", "gemm-moe-down", "grid-equal-gate-up",
         "swizzle-moe-gate-up", "swizzle-moe-down", "block128-pow2-gate-up", "block128-fp32-gate-up",
         "sync-fused-subset")
SUBSET_LAYERS = 2      # quant-sync-subset: the first 2 layers' 8 weights (0.39 G elements, ~1.2 GB on the device)


def run_case(name: str, reps: int):
    """One kernel on one config, `reps` launches, for profiler captures (prints its CUDA-event time)."""
    import torch

    from mxfp8_block_scaled_07_b200 import build as mxbuild
    from mxfp8_block_scaled_07_b200 import mx, synth

    mxbuild.build()
    dev = torch.device("cuda", 0)
    if name == "quant-gate-up":
        x = synth.sync_weight(0, 2, device=dev)
        bufs = mx.quantize(x, True, False)
        fn = lambda: mx.quantize(x, True, False, out=bufs)
    elif name == "quant-sync-subset":
        # The headline launch (mx_quantize_multi ROWWISE|SWIZZLE) over a subset of the 144 weights,
        # for DRAM-traffic captures: per-element traffic scales to the full launch.
        xs = [synth.sync_weight(layer, idx, device=dev) for layer in range(SUBSET_LAYERS) for idx in range(4)]
        outs = mx.quantize_multi(xs, True, False, True)
        fn = lambda: mx.quantize_multi(xs, True, False, True, outs=outs)
        print(json.dumps({"case": name, "tensors": len(xs), "elements": int(sum(x.numel() for x in xs))}))
    elif name == "quant-fwd-1300":
        x = synth.fwd_activations(1300, device=dev)
        bufs = mx.quantize(x, True, False)
        fn = lambda: mx.quantize(x, True, False, out=bufs)
    elif name == "quant-dy-rowcol":
        _, _, x = synth.update_inputs(device=dev)
        bufs = mx.quantize(x, True, True)
        fn = lambda: mx.quantize(x, True, True, out=bufs)
    elif name == "quant-dy-col":
        _, _, x = synth.update_inputs(device=dev)
        bufs = mx.quantize(x, False, True)
        fn = lambda: mx.quantize(x, False, True, out=bufs)
    elif name == "grid-equal-gate-up":
        x = synth.sync_weight(0, 2, device=dev)
        q, _, _, _ = mx.quantize(x, True, False)
        q2 = q.clone()
        fn = lambda: mx.grid_equal(q, q2)
    elif name == "sync-fused-subset":
        # mx_quantize_compare_multi over the first SUBSET_LAYERS layers' weights against their
        # sampler copy (here: the learner grid itself), for DRAM-traffic captures.
        xs = [synth.sync_weight(layer, idx, device=dev) for layer in range(SUBSET_LAYERS) for idx in range(4)]
        outs = mx.quantize_multi(xs, True, False, True)
        refs = [(q.clone(), s.clone()) for q, s, _, _ in outs]
        res = torch.empty((2, 2 * len(xs)), dtype=torch.int64, device=dev)
        fn = lambda: mx.quantize_compare_multi(xs, refs, outs=outs, results=res)
        print(json.dumps({"case": name, "tensors": len(xs), "elements": int(sum(x.numel() for x in xs))}))
    elif name.startswith("block128"):
        x = synth.sync_weight(0, 2, device=dev)
        pow2 = name == "block128-pow2-gate-up"
        g = mx.quantize_block128(x, pow2)
        fn = lambda: mx.quantize_block128(x, pow2, out=g)
    elif name.startswith("swizzle-moe"):
        # The grouped A-operand scale layout of the MoE GEMMs (raw scales of X_perm or H).
        counts, Xp, Hh, _, _ = synth.moe_inputs(device=dev)
        counts = [int(c) for c in counts]
        _, s_raw, _, _ = mx.quantize(Xp if name == "swizzle-moe-gate-up" else Hh, True, False, swizzle=False)
        del Xp, Hh
        o = mx.swizzle_scales(s_raw, counts)
        fn = lambda: mx.swizzle_scales(s_raw, counts, out=o)
    elif name.startswith("gemm-moe"):
        counts, Xp, Hh, W1, W2 = synth.moe_inputs(device=dev)
        counts = [int(c) for c in counts]
        A, Wt = (Xp, W1) if name == "gemm-moe-gate-up" else (Hh, W2)
        G, N, K = Wt.shape
        qa, sa_raw, _, _ = mx.quantize(A, True, False, swizzle=False)
        sa = mx.swizzle_scales(sa_raw, counts)
        qb, sb, _, _ = mx.quantize(Wt.reshape(G * N, K), True, False)
        offs = torch.tensor(synth.group_offsets(counts), dtype=torch.int32, device=dev)
        C = torch.empty((A.shape[0], N), dtype=torch.bfloat16, device=dev)
        fn = lambda: mx.grouped_gemm(qa, sa, qb.reshape(G, N, K), sb, offs, out=C)
    elif name == "gemm-update-dgrad":
        _, W, dY = synth.update_inputs(device=dev)
        qd, sd, _, _ = mx.quantize(dY, True, False)
        _, _, qwc, swc = mx.quantize(W, False, True)
        C = torch.empty((dY.shape[0], W.shape[1]), dtype=torch.bfloat16, device=dev)
        fn = lambda: mx.gemm(qd, sd, qwc, swc, out=C)
    else:
        if name == "gemm-fwd-10300":
            A = synth.fwd_activations(10300, device=dev)
            B = synth.sync_weight(0, 2, device=dev)
        else:
            A, B, _ = synth.update_inputs(device=dev)
        qa, sa, _, _ = mx.quantize(A, True, False)
        qb, sb, _, _ = mx.quantize(B, True, False)
        C = torch.empty((A.shape[0], B.shape[0]), dtype=torch.bfloat16, device=dev)
        fn = lambda: mx.gemm(qa, sa, qb, sb, out=C)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    print(json.dumps({"case": name, "reps": reps, "ms_per_launch": e0.elapsed_time(e1) / reps,
                      "device_error": mx.device_error()}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=CASES, help="run one kernel config only (for profiler captures)")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--gemm-variant", type=int, default=0, choices=[0, 1],
                    help="GEMM kernel for --case runs: 0 CTA pair (default), 1 single CTA")
    ap.add_argument("--quant-variant", type=int, default=0, choices=[0, 1],
                    help="quantizer kernel for --case runs: 0 register-staged (default), 1 TMA-staged")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="mx", choices=["mx", "reference"])
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.case:
        from mxfp8_block_scaled_07_b200 import build as mxbuild
        from mxfp8_block_scaled_07_b200 import mx

        mxbuild.build()
        mx.set_gemm_variant(args.gemm_variant)
        mx.set_quantize_variant(args.quant_variant)
        return run_case(args.case, args.reps)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import torch

    from mxfp8_block_scaled_07_b200 import build as mxbuild
    from mxfp8_block_scaled_07_b200 import mx

    world, rank, local, pg = dist_setup(args)
    if rank == 0:
        mxbuild.build()
    if pg is not None:
        pg.barrier()
    mx.lib()
    device = torch.device("cuda", local)
    peaks = load_peaks()
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream

    wl = SyncWorkload(rank, device)
    for _ in range(args.warmup):
        wl.step(sp)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier_sync(pg)
    with ClockSampler(local) as clocks:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for k in range(args.steps):
            wl.step(sp, *evs[k], stream=stream)
        t1.record(stream)
        torch.cuda.synchronize()
        time.sleep(0.25)
    if pg is not None:
        pg.barrier()
    headline_err = sum_over_ranks(pg, mx.device_error())     # any rank's status bits mark the run
    ms_local = t0.elapsed_time(t1) / args.steps
    quant_ms = statistics.mean(a.elapsed_time(b) for a, b, _ in evs)
    cmp_ms = statistics.mean(b.elapsed_time(c) for _, b, c in evs)
    ms = max_over_ranks(pg, ms_local)
    mismatches = sum_over_ranks(pg, int(wl.results[0].sum().item()))
    value = job_throughput_gbs(world, wl.step_bytes, ms)

    quant_launch_ms = quant_ms          # one mx_quantize_multi launch per step
    quant_bytes_per_launch = wl.quant_bytes
    achieved = quant_bytes_per_launch / (quant_launch_ms * 1e-3) / 1e9
    trec = traffic_record()
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": (round(trec["dram_bytes_per_elem"] * wl.total_elems)
                            if trec else None),
                "kernel": "quantize_rowwise_kernel<192, split loads> (mx_quantize_multi ROWWISE|SWIZZLE, 144 tensors)",
                "traffic_source": (trec.get("scaling", "full-launch capture")[:160] if trec else None),
                "peak_source": f"{peaks['source']} hbm copy (MEASURED_PEAKS.json)" if peaks["source"] == "measured"
                else "fallback 6.65 TB/s",
                "algorithmic_bytes_per_launch": round(quant_bytes_per_launch),
                "avg_launch_ms": round(quant_launch_ms, 5),
                "frac_of_8TBs_spec": round(achieved / 8000.0, 4)}

    secondary = None
    e2e = None
    cpu = None
    fused = None
    if rank == 0 and not args.no_secondary and world == 1:
        fused = guarded(lambda: run_fused_sync(wl, stream, ms, quant_ms, cmp_ms))
    if not args.no_e2e:                  # every rank: the whole job's end-to-end step
        e2e = aggregate_e2e(pg, run_e2e(wl, args, device), world, wl.step_bytes)
        e2e_err = mx.device_error()
        if e2e_err:
            e2e["device_error"] = e2e_err
            e2e["invalid"] = True
    del wl
    torch.cuda.empty_cache()
    # Kernel characterization lines (one GPU's kernels) only in single-GPU runs: the other ranks
    # of a multi-GPU run would otherwise wait for them inside a collective.
    if rank == 0 and not args.no_secondary and world == 1:
        secondary = guarded(lambda: run_secondary(device, peaks))
        secondary["sync_fused"] = fused
        secondary["dense_8192_reference"] = guarded(lambda: run_library_gemm_peak(device))
        secondary["update_breakeven"] = guarded(lambda: run_breakeven(device))
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        v1, desc1 = oracle_sync_sample(12.0)
        vp, procs, descp = oracle_sync_sample_parallel()
        gf, gdesc = oracle_gemm_sample()
        cpu = {"value": round(vp, 4), "unit": UNIT, "cores": procs, "kind": "oracle", "sample": descp,
               "single_thread": {"value": round(v1, 4), "cores": 1, "sample": desc1},
               "gemm": {"value": round(gf / 1e9, 3), "unit": "GFLOP/s", "cores": 1, "sample": gdesc}}
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16->e4m3/e8m0 (u8)", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tensors_per_rank": 144,
                       "elements_per_rank": int(sum(r * c for _, _, r, c in sync_shapes())),
                       "algorithmic_bytes_per_rank_step": int(world and (value * ms * 1e-3 * 1e9 / world)),
                       "parallelism": f"weak x{world} (each rank its own 144 tensors)",
                       "l2": "inputs larger than L2 (13.9 GB BF16 per rank per step)",
                       "phase_ms": {"quantize": round(quant_ms, 4), "grid_equal": round(cmp_ms, 4)}},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps * SyncWorkload.LAUNCHES_PER_STEP,
            "clocks": clocks.summary(),
            "grid_equal_mismatches": mismatches,
            "device_error": headline_err,
            "secondary": secondary,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
