#!/usr/bin/env python3
"""Benchmark of the fused Q4_K dequant + GEMV hot path on B200.

One step = one q4k_gemv call (+ argmax epilogue) over the Q4_K LM-head
workload (N = 248320 vocab rows x K = 4096, batch 1, ~572 MB of blocks; seed
4; x ~ N(0,1)/64): activation staging (per-super-block fixed point), block
streaming, header decode, quant unpack, integer dot products, scale/min
combine in fp64, reduction, logits + argmax.  The matrix is larger than the
126 MB L2, so no flush is needed between steps.

Metric: effective HBM GB/s = (weight bytes + activation bytes) / time.
  value  - device time of K steps (CUDA events, inputs resident in HBM), max over ranks
  e2e    - the same metric through the same C-ABI call, with each step's x copied
           host->device from pinned memory and its logits + argmax copied back, both
           copies on their own streams into double buffers so that they overlap the
           neighbouring steps (weights stay resident, as a decode loop keeps them)
  roofline - dominant kernel (q4k_gemv_fx_kernel) timed alone with CUDA events on its
           stream, against the measured HBM copy bandwidth in MEASURED_PEAKS.json
           (and, as frac_of_nominal_8tbs, against the nominal 8 TB/s)
  secondary - the same roofline record for the down projection at batch 1
           (4096 x 12288) and the fused SwiGLU (2 x 12288 x 4096), timed under
           CUDA-graph replay over weight copies that exceed L2 (N = 1 only)
  cpu_baseline / cpu_baseline_all_cores - the CPU oracle timed on this host (rank 0,
           N = 1): one thread, and one thread per core over disjoint rows

--table prints per-workload device times under CUDA-graph replay instead: the
decode shapes, grouped QKV, a decode step, the FFN block and the W4A16 prefill
(--only selects cases by name).

--impl reference times the CPU oracle itself (there is no other implementation
of this path to install): each step is a bounded row sample of the workload.

Multi-GPU (torchrun, one process per GPU): every rank runs its own independent
problem (rows do not interact; no collective on the data path); value is the
total bytes of all ranks over the max-over-ranks time ("scaling": "weak").
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

import numpy as np  # noqa: E402

METRIC = "dequant-GEMV effective HBM GB/s and % of B200 peak (Q4_K, batch 1)"
UNIT = "GB/s"
WORKLOAD = "q4k_lmhead_248320x4096"
FALLBACK_HBM_GBS = 6650.0

NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e, nominal

# DRAM bytes (read + write) per launch of q4k_gemv_fx_kernel, from one ncu
# capture per workload, valid only for the kernel sources whose hash is recorded.
NCU_TRAFFIC = {"sources_sha1": "4aeb0b3924fb4e8ffb6faa31e154a8d4f969214f",
               "bytes_per_launch": {"q4k_lmhead_248320x4096": 572227584 + 3427072,
                                    "q4k_down_4096x12288": 28427776 + 0,
                                    "q4k_swiglu_12288x4096": 56720640 + 9472}}


def kernel_sources_sha1() -> str:
    h = hashlib.sha1()
    for f in ("q4k_gemv.cu", "q4k_fx.cuh", "q4k_exact.cuh", "q4k_stream.cuh", "dq_common.cuh"):
        with open(os.path.join(ROOT, "dequant_gemv_q4_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--rows", type=int, default=0,
                    help="override N (a smaller case of the same kernel, e.g. for ncu captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the roofline records of the down projection and the SwiGLU")
    ap.add_argument("--table", action="store_true",
                    help="print one JSON line per workload: device time per call under CUDA-graph replay "
                         "(weights rotated through enough copies to exceed L2), then exit")
    ap.add_argument("--only", default="",
                    help="with --table: run only the cases whose name contains this text")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="approximate CPU budget of the oracle baseline")
    return ap.parse_args()


def algorithmic_bytes(wl, B=1):
    from dequant_gemv_q4_b200 import synth
    per_block = synth.Q4K_BLOCK_BYTES if wl.fmt == "q4k" else synth.Q8_0_BLOCK_BYTES
    elems = synth.Q4K_BLOCK_ELEMS if wl.fmt == "q4k" else synth.Q8_0_BLOCK_ELEMS
    nmat = 2 if wl.op == "swiglu" else 1
    return nmat * wl.N * (wl.K // elems) * per_block + 4 * B * wl.K


def rank_workload(wl, rank: int, world: int):
    """The workload a rank runs: with several ranks each one gets its own
    independent problem of the same shape (seed offset by rank)."""
    from dequant_gemv_q4_b200 import synth
    if world <= 1:
        return wl
    return synth.Workload(wl.name, wl.fmt, wl.op, wl.N, wl.K, wl.batches, wl.seed + 1000 * rank, wl.x_scale)


def max_over_ranks(v: float, world: int, device=None) -> float:
    """Largest value over all ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbps(nbytes_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job GB/s: the bytes every rank processed in one step over the step time."""
    return nbytes_per_rank * world / (ms_per_step * 1e-3) / 1e9


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False

    def _poll(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.002)

    def _sample(self):
        try:
            self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
            self.reasons |= int(self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
        except Exception:
            pass

    def sample_now(self):
        """One sample from the calling thread (the poller may be starved while the
        launching thread holds the interpreter)."""
        if self._ok:
            self._sample()

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._poll, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._ok:
            self._stop.set()
            self._t.join()
            self._sample()

    def summary(self):
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline_all_cores(wl, inp, budget_s):
    """Time the CPU oracle (as it stands) over rows split across every host core:
    one thread per core, each running the oracle on its own consecutive rows (the
    oracle's C loop releases the interpreter, so the threads run in parallel)."""
    import concurrent.futures
    import oracle
    from dequant_gemv_q4_b200 import synth
    cores = host_cores()
    weights_per_row = wl.K * (2 if wl.op == "swiglu" else 1)
    rows = int(max(64 * cores, min(wl.N, budget_s * cores * 9.0e7 / weights_per_row)))
    parts = [p for p in np.array_split(np.arange(rows, dtype=np.int64), cores) if p.size]

    def run(sel):
        if wl.op == "swiglu":
            g, _ = oracle.q4k_gemv(inp["w_gate"], wl.N, wl.K, inp["x"], rows=sel)
            u, _ = oracle.q4k_gemv(inp["w_up"], wl.N, wl.K, inp["x"], rows=sel)
            return oracle.swiglu(g, u)
        if wl.fmt == "q4k":
            return oracle.q4k_gemv(inp["w"], wl.N, wl.K, inp["x"], rows=sel)[0]
        return oracle.q8_0_gemv(inp["w"], wl.N, wl.K, inp["x"], rows=sel)[0]

    t = time.perf_counter()
    with concurrent.futures.ThreadPoolExecutor(cores) as ex:
        ys = list(ex.map(run, parts))
    if wl.op == "gemv_argmax":
        oracle.argmax(np.concatenate([y[0] for y in ys]))
    dt = time.perf_counter() - t
    per_block = synth.Q4K_BLOCK_BYTES if wl.fmt == "q4k" else synth.Q8_0_BLOCK_BYTES
    elems = synth.Q4K_BLOCK_ELEMS if wl.fmt == "q4k" else synth.Q8_0_BLOCK_ELEMS
    nbytes = (2 if wl.op == "swiglu" else 1) * rows * (wl.K // elems) * per_block + 4 * wl.K
    return {"value": nbytes / dt / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(), "nproc": os.cpu_count(),
            "sample": "%d of %d rows (%.3g weights), %d threads (one per core), %.1f s" % (
                rows, wl.N, rows * weights_per_row, cores, dt)}


def cpu_baseline(wl, inp, budget_s):
    """Time the CPU oracle (single thread, as it stands) on a bounded row sample."""
    import oracle
    from dequant_gemv_q4_b200 import synth
    # ~90 M weights/s per thread: size the sample to the budget
    weights_per_row = wl.K * (2 if wl.op == "swiglu" else 1)
    rows = int(max(64, min(wl.N, budget_s * 9.0e7 / weights_per_row)))
    sel = np.arange(rows, dtype=np.int64)
    t = time.perf_counter()
    if wl.op == "swiglu":
        g, _ = oracle.q4k_gemv(inp["w_gate"], wl.N, wl.K, inp["x"], rows=sel)
        u, _ = oracle.q4k_gemv(inp["w_up"], wl.N, wl.K, inp["x"], rows=sel)
        oracle.swiglu(g, u)
    elif wl.fmt == "q4k":
        y, _ = oracle.q4k_gemv(inp["w"], wl.N, wl.K, inp["x"], rows=sel)
        if wl.op == "gemv_argmax":
            oracle.argmax(y[0])
    else:
        oracle.q8_0_gemv(inp["w"], wl.N, wl.K, inp["x"], rows=sel)
    dt = time.perf_counter() - t
    per_block = synth.Q4K_BLOCK_BYTES if wl.fmt == "q4k" else synth.Q8_0_BLOCK_BYTES
    elems = synth.Q4K_BLOCK_ELEMS if wl.fmt == "q4k" else synth.Q8_0_BLOCK_ELEMS
    nbytes = (2 if wl.op == "swiglu" else 1) * rows * (wl.K // elems) * per_block + 4 * wl.K
    return {"value": nbytes / dt / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
            "cpu_model": cpu_model(), "nproc": os.cpu_count(),
            "sample": "%d of %d rows (%.3g weights), single thread, %.1f s" % (rows, wl.N, rows * weights_per_row, dt)}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle on host cores, rank 0 only."""
    if rank != 0:
        return
    from dequant_gemv_q4_b200 import synth
    import oracle
    wl = synth.WORKLOADS[args.workload]
    inp = synth.make_inputs(wl)
    # each step: a bounded sample of rows so that warmup + steps stay within minutes
    weights_per_row = wl.K * (2 if wl.op == "swiglu" else 1)
    per_step_s = min(2.0, 150.0 / max(1, args.steps + args.warmup))
    rows = int(max(16, min(wl.N, per_step_s * 9.0e7 / weights_per_row)))
    elems = synth.Q4K_BLOCK_ELEMS if wl.fmt == "q4k" else synth.Q8_0_BLOCK_ELEMS
    per_block = synth.Q4K_BLOCK_BYTES if wl.fmt == "q4k" else synth.Q8_0_BLOCK_BYTES
    nbytes = (2 if wl.op == "swiglu" else 1) * rows * (wl.K // elems) * per_block + 4 * wl.K

    def step(i):
        start = (i * rows) % max(1, wl.N - rows + 1)
        sel = np.arange(start, start + rows, dtype=np.int64)
        if wl.op == "swiglu":
            g, _ = oracle.q4k_gemv(inp["w_gate"], wl.N, wl.K, inp["x"], rows=sel)
            u, _ = oracle.q4k_gemv(inp["w_up"], wl.N, wl.K, inp["x"], rows=sel)
            oracle.swiglu(g, u)
        elif wl.fmt == "q4k":
            y, _ = oracle.q4k_gemv(inp["w"], wl.N, wl.K, inp["x"], rows=sel)
            if wl.op == "gemv_argmax":
                oracle.argmax(y[0])
        else:
            oracle.q8_0_gemv(inp["w"], wl.N, wl.K, inp["x"], rows=sel)

    for i in range(args.warmup):
        step(i)
    t = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    dt = (time.perf_counter() - t) / max(1, args.steps)
    value = nbytes / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "N": wl.N, "K": wl.K, "B": 1, "format": "Q4_K" if wl.fmt == "q4k" else "Q8_0",
                   "sample_rows_per_step": rows},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": "%d consecutive rows per step of %d, single thread" % (rows, wl.N)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def graph_us_per_call(fn, copies, reps=20):
    """Device time per call of fn(0) .. fn(copies - 1), captured once in a CUDA graph
    and replayed `reps` times back to back (3 untimed replays first); CUDA events on
    the replay stream."""
    import torch
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for i in range(copies):
            fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(copies):
            fn(i)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(reps):
            g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * copies)
    del g
    return us


def graph_table(only=""):
    """Per-workload device time per call, each call captured in a CUDA graph and
    replayed back to back; every workload's weights rotate through enough copies
    (more than 1.3 x the 126 MB L2) that each call streams them from HBM.  `only`
    keeps the cases whose name contains it."""
    import torch
    import dequant_gemv_q4_b200 as dq
    from dequant_gemv_q4_b200 import synth

    torch.cuda.set_device(0)
    l2 = 126e6

    def timed(name, fn, nbytes, copies, reps=20, flops=0):
        us = graph_us_per_call(fn, copies, reps)
        rec = {"case": name, "us_per_call": round(us, 2), "GBps": round(nbytes / us / 1e3, 1), "bytes": nbytes,
               "copies": copies}
        if flops:
            rec["TFLOPs"] = round(flops / us / 1e6, 1)
        print(json.dumps(rec), flush=True)

    cases = [("q4k_lmhead_248320x4096", 1, "gemv"), ("q4k_lmhead_248320x4096", 1, "argmax"),
             ("q4k_down_4096x12288", 1, "gemv"), ("q4k_down_4096x12288", 2, "gemv"),
             ("q4k_down_4096x12288", 4, "gemv"), ("q4k_down_4096x12288", 8, "gemv"),
             ("q4k_swiglu_12288x4096", 1, "gemv"), ("q4k_gemv_4096x1024", 1, "gemv"),
             ("q4k_gemv_4096x1024", 1, "split_qg"), ("q8_0_gemv_1024x1024", 1, "gemv")]
    def want(name):
        return only in name

    for wname, B, mode in cases:
        if not want("%s:B%d:%s" % (wname, B, mode)):
            continue
        wl = synth.WORKLOADS[wname]
        inp = synth.make_inputs(wl, B=B)
        keys = ["w_gate", "w_up"] if wl.op == "swiglu" else ["w"]
        wbytes = sum(inp[k].nbytes for k in keys)
        copies = min(64, max(1, int(np.ceil(1.3 * l2 / wbytes))))
        ws = [[torch.from_numpy(inp[k]).cuda() for k in keys]]
        for _ in range(1, copies):
            ws.append([t.clone() for t in ws[0]])
        x = torch.from_numpy(inp["x"]).cuda()
        y = torch.empty((B, wl.N), device="cuda")
        scratch = torch.empty(1 << 24, dtype=torch.uint8, device="cuda")
        nbytes = wbytes + inp["x"].nbytes
        if wl.op == "swiglu":
            fn = lambda i: dq.q4k_swiglu_gemv(ws[i][0], ws[i][1], x, wl.N, wl.K, out=y, workspace=scratch)
        elif wl.fmt == "q8_0":
            fn = lambda i: dq.q8_0_gemv(ws[i][0], x, wl.N, wl.K, y=y, workspace=scratch)
        elif mode == "split_qg":
            qo = torch.empty((B, wl.N // 2), device="cuda")
            go = torch.empty((B, wl.N // 2), device="cuda")
            fn = lambda i: dq.q4k_gemv_split_qg(ws[i][0], x, wl.N, wl.K, 128, q=qo, g=go, workspace=scratch)
        else:
            am = mode == "argmax"
            fn = lambda i: dq.q4k_gemv(ws[i][0], x, wl.N, wl.K, y=y, argmax=am, workspace=scratch)
        timed("%s:B%d:%s" % (wname, B, mode), fn, nbytes, copies)
        del ws
        torch.cuda.empty_cache()

    if want("qkv_4096+1024+1024x4096"):
        qkv_table(timed, l2)
    if want("decode_step:qproj_split+swiglu+down"):
        decode_step_table(timed)
    if want("ffn_block_4096x12288:one_call") or want("ffn_block_4096x12288:separate"):
        ffn_table(timed, want)
    prefill_table(timed, l2, want)


def ffn_table(timed, want):
    """A decoder layer's FFN block, x = x + W_down(silu(W_gate x) * (W_up x)) with H =
    4096 and F = 12288: the one-call entry point and the two separate calls."""
    import torch
    import dequant_gemv_q4_b200 as dq
    from dequant_gemv_q4_b200 import synth

    rng = np.random.default_rng(45)
    H, F = 4096, 12288
    mats = [[torch.from_numpy(synth.q4k_matrix(rng, n, k)).cuda() for n, k in ((F, H), (F, H), (H, F))]
            for _ in range(2)]
    x = torch.from_numpy(synth.activations(rng, 1, H)).cuda()
    y = torch.empty((1, H), device="cuda")
    hid = torch.empty((1, F), device="cuda")
    scratch = torch.empty(1 << 26, dtype=torch.uint8, device="cuda")
    nbytes = sum(m.numel() for m in mats[0]) + 4 * (2 * H + F)
    if want("ffn_block_4096x12288:one_call"):
        timed("ffn_block_4096x12288:one_call",
              lambda i: dq.q4k_ffn_block(mats[i][0], mats[i][1], mats[i][2], x, H, F, residual=x, y=y,
                                         workspace=scratch), nbytes, 2)

    def separate(i):
        dq.q4k_swiglu_gemv(mats[i][0], mats[i][1], x, F, H, out=hid, workspace=scratch)
        dq.q4k_gemv_residual(mats[i][2], hid, x, H, F, y=y, workspace=scratch)

    if want("ffn_block_4096x12288:separate"):
        timed("ffn_block_4096x12288:separate", separate, nbytes, 2)
    del mats
    torch.cuda.empty_cache()


def qkv_table(timed, l2):
    """Q, K and V projections of a hidden-4096 layer (8 KV heads of 128): one
    grouped launch, and three separate calls."""
    import torch
    import dequant_gemv_q4_b200 as dq
    from dequant_gemv_q4_b200 import synth

    rng = np.random.default_rng(43)
    Hq, Ns = 4096, (4096, 1024, 1024)
    per_set = sum(n * (Hq // 256) * 144 for n in Ns)
    copies = min(64, max(1, int(np.ceil(1.3 * l2 / per_set))))
    qkv = [[torch.from_numpy(synth.q4k_matrix(rng, n, Hq)).cuda() for n in Ns]]
    for _ in range(1, copies):
        qkv.append([t.clone() for t in qkv[0]])
    xq = torch.from_numpy(synth.activations(rng, 1, Hq)).cuda()
    outs = [torch.empty(n, device="cuda") for n in Ns]
    scratch = torch.empty(1 << 24, dtype=torch.uint8, device="cuda")
    timed("qkv_4096+1024+1024x4096:group", lambda i: dq.q4k_gemv_group(qkv[i], xq[0], list(Ns), Hq, ys=outs,
                                                                       workspace=scratch), per_set + 4 * Hq, copies)

    def separate(i):
        for m, n in enumerate(Ns):
            dq.q4k_gemv(qkv[i][m], xq, n, Hq, y=outs[m].view(1, n), workspace=scratch)

    timed("qkv_4096+1024+1024x4096:separate", separate, per_set + 4 * Hq, copies)
    del qkv
    torch.cuda.empty_cache()


def decode_step_table(timed):
    """One decode step's GEMV sequence: q-projection with the Q/gate split (16
    heads of 128), SwiGLU 2 x 12288 x 4096, and the down projection 4096 x 12288
    of its output."""
    import torch
    import dequant_gemv_q4_b200 as dq
    from dequant_gemv_q4_b200 import synth

    rng = np.random.default_rng(41)
    H, F, NQ, KQ = 4096, 12288, 4096, 1024
    shapes = ((NQ, KQ), (F, H), (F, H), (H, F))
    mats = [[torch.from_numpy(synth.q4k_matrix(rng, n, k)).cuda() for n, k in shapes] for _ in range(2)]
    xq = torch.from_numpy(synth.activations(rng, 1, KQ)).cuda()
    xh = torch.from_numpy(synth.activations(rng, 1, H)).cuda()
    qo = torch.empty((1, NQ // 2), device="cuda")
    go = torch.empty((1, NQ // 2), device="cuda")
    hid = torch.empty((1, F), device="cuda")
    out = torch.empty((1, H), device="cuda")
    scratch = torch.empty(1 << 24, dtype=torch.uint8, device="cuda")

    def decode_step(i):
        wq, wg, wu, wd = mats[i]
        dq.q4k_gemv_split_qg(wq, xq, NQ, KQ, 128, q=qo, g=go, workspace=scratch)
        dq.q4k_swiglu_gemv(wg, wu, xh, F, H, out=hid, workspace=scratch)
        dq.q4k_gemv(wd, hid, H, F, y=out, workspace=scratch)

    nbytes = sum(m.numel() for m in mats[0]) + 4 * (KQ + H + F)
    timed("decode_step:qproj_split+swiglu+down", decode_step, nbytes, 2)
    del mats
    torch.cuda.empty_cache()


def prefill_table(timed, l2, want):
    """W4A16 prefill on the tensor cores: M binary16 tokens through the down
    projection and through one gate/up matrix (bytes: weights + activations;
    flops: 2 M N K)."""
    import torch
    import dequant_gemv_q4_b200 as dq
    from dequant_gemv_q4_b200 import synth

    rng = np.random.default_rng(44)
    Ms = (16, 64, 128, 256, 512)
    for N, K in ((4096, 12288), (12288, 4096)):
        if not any(want("prefill_%dx%d:M%d" % (N, K, M)) for M in Ms):
            continue
        wbytes = N * (K // 256) * 144
        copies = max(1, int(np.ceil(1.3 * l2 / wbytes)))
        pw = [torch.from_numpy(synth.q4k_matrix(rng, N, K)).cuda()]
        for _ in range(1, copies):
            pw.append(pw[0].clone())
        for M in Ms:
            if not want("prefill_%dx%d:M%d" % (N, K, M)):
                continue
            x16 = torch.from_numpy(synth.activations_f16(rng, M, K)).cuda()
            yp = torch.empty((M, N), device="cuda")
            scratch = torch.empty(max(1, dq.dq_workspace_bytes(dq.DQ_OP_Q4K_PREFILL, N, K, M)), dtype=torch.uint8,
                                  device="cuda")
            timed("prefill_%dx%d:M%d" % (N, K, M),
                  lambda i: dq.q4k_prefill_gemm(pw[i], x16, N, K, y=yp, workspace=scratch),
                  wbytes + 2 * M * K, copies, flops=2 * M * N * K)
        del pw
        torch.cuda.empty_cache()


def secondary_rooflines(peak, peak_kind, reps=50):
    """Roofline records of the other HBM-bound decode shapes, on the same device:
    the down projection at batch 1 (4096 x 12288, gated like the LM head) and the
    fused SwiGLU (2 x 12288 x 4096).  Each launch's weights rotate through enough
    copies to exceed L2 (> 1.3 x 126 MB), the calls are replayed from a CUDA graph,
    and achieved = algorithmic bytes per call / device time per call."""
    import torch
    import dequant_gemv_q4_b200 as dq
    from dequant_gemv_q4_b200 import synth
    out = []
    for wname in ("q4k_down_4096x12288", "q4k_swiglu_12288x4096"):
        wl = synth.WORKLOADS[wname]
        inp = synth.make_inputs(wl, B=1)
        keys = ["w_gate", "w_up"] if wl.op == "swiglu" else ["w"]
        wbytes = sum(inp[k].nbytes for k in keys)
        copies = max(1, int(np.ceil(1.3 * 126e6 / wbytes)))
        ws = [[torch.from_numpy(inp[k]).cuda() for k in keys]]
        for _ in range(1, copies):
            ws.append([t.clone() for t in ws[0]])
        x = torch.from_numpy(inp["x"]).cuda()
        y = torch.empty((1, wl.N), device="cuda")
        scratch = torch.empty(1 << 24, dtype=torch.uint8, device="cuda")
        if wl.op == "swiglu":
            fn = lambda i: dq.q4k_swiglu_gemv(ws[i][0], ws[i][1], x, wl.N, wl.K, out=y, workspace=scratch)
            split = dq.dq_workspace_bytes(dq.DQ_OP_Q4K_SWIGLU, wl.N, wl.K, 1) > 0
        else:
            fn = lambda i: dq.q4k_gemv(ws[i][0], x, wl.N, wl.K, y=y, workspace=scratch)
            split = dq.dq_workspace_bytes(dq.DQ_OP_Q4K_GEMV, wl.N, wl.K, 1) > 0
        us = graph_us_per_call(fn, copies, reps)
        nbytes = algorithmic_bytes(wl, 1)
        achieved = nbytes / (us * 1e-6) / 1e9
        traffic = NCU_TRAFFIC["bytes_per_launch"].get(wname) \
            if NCU_TRAFFIC["sources_sha1"] == kernel_sources_sha1() else None
        out.append({"workload": wname, "B": 1, "us_per_call": us,
                    "launches_per_call": 2 if split else 1,
                    "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": UNIT,
                                 "frac": achieved / peak, "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                                 "traffic": traffic, "kernel": "q4k_gemv_fx_kernel",
                                 "peak_kind": peak_kind,
                                 "timing": "CUDA-graph replay of %d calls over %d weight copies, %d replays" % (
                                     copies, copies, reps)}})
        del ws
        torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.table:
        graph_table(args.only)
        return

    import torch
    import torch.distributed as dist

    import dequant_gemv_q4_b200 as dq
    from dequant_gemv_q4_b200 import synth

    torch.cuda.set_device(local_rank)
    dist_on = world > 1
    if dist_on:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))

    wl = synth.WORKLOADS[args.workload]
    B = 1
    if args.rows:
        wl = synth.Workload("%s_rows%d" % (wl.name, args.rows), wl.fmt, wl.op, args.rows, wl.K, wl.batches,
                            wl.seed, wl.x_scale)
    wl = rank_workload(wl, rank, world)
    inp = synth.make_inputs(wl, B=B)
    dev = torch.device("cuda", local_rank)
    argmax = wl.op == "gemv_argmax"
    if wl.op == "swiglu":
        wg = torch.from_numpy(inp["w_gate"]).to(dev)
        wu = torch.from_numpy(inp["w_up"]).to(dev)
        op = dq.DQ_OP_Q4K_SWIGLU
    else:
        w = torch.from_numpy(inp["w"]).to(dev)
        op = dq.DQ_OP_Q4K_GEMV if wl.fmt == "q4k" else dq.DQ_OP_Q8_0_GEMV
    x = torch.from_numpy(inp["x"]).to(dev)
    y = torch.empty((B, wl.N), dtype=torch.float32, device=dev)
    ws_bytes = dq.dq_workspace_bytes(op, wl.N, wl.K, B, argmax)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    split = dq.dq_workspace_bytes(op, wl.N, wl.K, B, False) > 0
    launches_per_step = 1 + (1 if split else 0) + (1 if argmax else 0)
    stream = torch.cuda.current_stream(dev)

    def step(xin, yout, with_argmax=argmax):
        if wl.op == "swiglu":
            dq.q4k_swiglu_gemv(wg, wu, xin, wl.N, wl.K, out=yout, workspace=ws)
            return None
        if wl.fmt == "q4k":
            r = dq.q4k_gemv(w, xin, wl.N, wl.K, y=yout, argmax=with_argmax, workspace=ws)
            return r[1] if with_argmax else None
        dq.q8_0_gemv(w, xin, wl.N, wl.K, y=yout, workspace=ws)
        return None

    def barrier():
        if dist_on:
            dist.barrier(device_ids=[local_rank])
        torch.cuda.synchronize(dev)

    nbytes = algorithmic_bytes(wl, B)

    # ---- device-resident steps (the headline value) ----
    for _ in range(max(3, args.warmup)):
        step(x, y)
    barrier()
    sampler = ClockSampler(local_rank)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # clocks are sampled over the device-timed steps and the kernel-alone loop
    sampler.__enter__()
    e0.record(stream)
    for _ in range(args.steps):
        step(x, y)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    sampler.sample_now()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world, dev)
    value = job_gbps(nbytes, world, ms)

    # ---- dominant kernel alone (one launch per call, no epilogue kernels) ----
    if not split:
        for _ in range(3):
            step(x, y, with_argmax=False)
        torch.cuda.synchronize(dev)
        # median of three timed runs of `steps` back-to-back launches
        reps = []
        for _ in range(3):
            k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            k0.record(stream)
            for _ in range(args.steps):
                step(x, y, with_argmax=False)
            k1.record(stream)
            torch.cuda.synchronize(dev)
            sampler.sample_now()
            reps.append(k0.elapsed_time(k1) / args.steps)
        kms = statistics.median(reps)
    else:
        kms = ms
    sampler.__exit__(None, None, None)
    barrier()

    # ---- end to end: host x in, host logits + argmax out ----
    # Every step copies its x host->device (pinned), runs the same C-ABI call
    # and copies its logits (+ argmax) device->host (pinned).  Both copies run
    # on their own streams, into one of two buffers each: the copy-in of step
    # i+1 overlaps step i, the copy-back of step i overlaps step i+1, and the
    # timed region ends when the last copy-back is done.
    x_host = torch.from_numpy(inp["x"]).pin_memory()
    y_host = [torch.empty((B, wl.N), dtype=torch.float32).pin_memory() for _ in range(2)]
    i_host = [torch.empty(1, dtype=torch.int64).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x), torch.empty_like(x)]
    y_dev = [y, torch.empty_like(y)]
    copy_stream = torch.cuda.Stream(dev)
    h2d_stream = torch.cuda.Stream(dev)
    done = [torch.cuda.Event(), torch.cuda.Event()]     # step using buffer j has computed
    freed = [torch.cuda.Event(), torch.cuda.Event()]    # output buffer j has been copied back
    x_ready = [torch.cuda.Event(), torch.cuda.Event()]  # input buffer j holds its step's x

    def e2e_copy_in(i):
        j = i & 1
        h2d_stream.wait_event(done[j])   # the step that last read buffer j has finished
        with torch.cuda.stream(h2d_stream):
            x_dev[j].copy_(x_host, non_blocking=True)
        x_ready[j].record(h2d_stream)

    def e2e_step(i, last):
        j = i & 1
        stream.wait_event(freed[j])
        stream.wait_event(x_ready[j])
        idx = step(x_dev[j], y_dev[j])
        done[j].record(stream)
        if i + 1 < last:
            e2e_copy_in(i + 1)
        copy_stream.wait_event(done[j])
        with torch.cuda.stream(copy_stream):
            y_host[j].copy_(y_dev[j], non_blocking=True)
            if idx is not None:
                idx.record_stream(copy_stream)
                i_host[j].copy_(idx, non_blocking=True)
        freed[j].record(copy_stream)

    for j in range(2):
        freed[j].record(copy_stream)
        done[j].record(stream)
    e2e_copy_in(0)
    for i in range(3):
        e2e_step(i, 3)
    torch.cuda.synchronize(dev)
    barrier()
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(stream)
    h2d_stream.wait_stream(stream)   # the first copy-in starts inside the timed region
    e2e_copy_in(0)
    for i in range(args.steps):
        e2e_step(i, args.steps)
    for j in range(2):
        stream.wait_event(freed[j])
    h1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(h0.elapsed_time(h1) / args.steps, world, dev)
    e2e_value = job_gbps(nbytes, world, e2e_ms)
    h2d = x_host.numel() * 4
    d2h = y_host[0].numel() * 4 + (8 if argmax else 0)

    peak, peak_kind = measured_peak()
    achieved = nbytes / (kms * 1e-3) / 1e9
    traffic = None
    if NCU_TRAFFIC["sources_sha1"] == kernel_sources_sha1():
        traffic = NCU_TRAFFIC["bytes_per_launch"].get(wl.name)
    peak_label = peak_kind + " (MEASURED_PEAKS.json hbm_gbs, burst)" if peak_kind == "measured" else "fallback"
    secondary = []
    if not args.no_secondary and world == 1 and wl.name == WORKLOAD:
        with ClockSampler(local_rank) as sec_clocks:
            secondary = secondary_rooflines(peak, peak_label)
        for rec in secondary:
            rec["clocks"] = sec_clocks.summary()

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "s8xu8->s32 dp4a, f64 combine", "data": "synthetic",
        "config": {"workload": wl.name, "N": wl.N, "K": wl.K, "B": B,
                   "format": "Q4_K" if wl.fmt == "q4k" else "Q8_0", "layout": "aos",
                   "epilogue": "argmax" if argmax else ("swiglu" if wl.op == "swiglu" else "none"),
                   "bytes_per_step": nbytes,
                   "l2": "weights %.0f MB > 126 MB L2; no flush" % (nbytes / 1e6) if nbytes > 126e6
                   else "weights fit in L2: NOT flushed (value is L2-assisted)",
                   "parallelism": "replicas x%d (independent problems, no collective)" % world},
        "pct_of_peak_hbm": 100.0 * value / world / peak,
        "pct_of_nominal_8tbs": 100.0 * value / world / NOMINAL_HBM_GBS,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": UNIT, "frac": achieved / peak,
                     "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                     "traffic": traffic, "kernel": "q4k_gemv_fx_kernel", "kernel_ms": kms,
                     "peak_kind": peak_label},
        "secondary": secondary,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms,
                "note": "weights resident; per step x in (pinned H2D on its own stream, overlapping the "
                        "previous step) and logits+argmax out (pinned D2H on a copy stream, overlapping the next "
                        "step); both double-buffered"},
        "gpu_launches": launches_per_step * args.steps,
        "gpu_launches_note": "device-timed loop; the roofline loop adds 3 x steps GEMV launches and the e2e loop "
                             "launches_per_step x steps more",
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, inp, args.cpu_seconds)
        line["cpu_baseline_all_cores"] = cpu_baseline_all_cores(wl, inp, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        dist.barrier(device_ids=[local_rank])
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
