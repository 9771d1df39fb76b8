#!/usr/bin/env python3
"""Benchmark: fused fp8 MQA logits + top-2048 on the causal-prefill workload.

One step = one pass of the whole indexer hot path over the workload
m = 8192 query rows x n = 35000 keys (H = 32, D = 128, ks = 0,
ke[i] = n - m + i + 1, top-k = 2048): range resolution, TMA staging,
tcgen05 fp8 contraction, fused ReLU / head-weight / scale / mask epilogue,
streaming top-k filter and exact per-row select, in one persistent kernel.

Prints ONE JSON line (rank 0).  `value` is algorithmic TFLOP/s over all
ranks: 8192 flop (2 * H * D) per valid (row, key) pair, divided by the max
over ranks of the device time of K steps.  Inputs are resident in HBM;
L2 is flushed (a 256 MiB write) before every timed step.  `e2e` is the same
metric through the same C-ABI call with the inputs copied from pinned host
memory and the top-k indices copied back inside each timed step.

--impl reference times the float64 CPU oracle instead, on a bounded sample
of the same workload's rows per step (rank 0 only).

--path chained times the unfused comparison path instead: materialised
logits (fp8idx_mqa_logits, rows chunked so that one chunk of logits stays
within 2 GiB) followed by fp8idx_topk_rows on each chunk, the loop of the
pages' chunked benchmark.  Same metric, same algorithmic flops.

--path act_quant (with --workload 4) times the producer of the paged keys:
fp8idx_act_quant_store of every key of the workload's requests (bf16 rows
to e4m3 codes and per-token scales, stored through the block table).  Its
metric is HBM GB/s: 256 B read, 8 B of slot read and 132 B written per key.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fp8_mqa_logits_03_b200 import workloads  # noqa: E402

WORKLOAD = 1
METRIC = "indexer fp8 TFLOP/s & rows·keys/s (fused logits+top-2048), % of roofline"
UNIT = "TFLOP/s"
FLOP_PER_PAIR = 2 * workloads.H * workloads.D  # 8192


def strict_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, allow_abbrev=False)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, choices=sorted(workloads.WORKLOADS), default=WORKLOAD,
                    help="workload index (default 1, the headline causal prefill)")
    ap.add_argument("--path", choices=["fused", "chained", "act_quant"], default="fused",
                    help="fused logits + top-k (default), materialised logits then top-k, "
                         "or the key quantisation into the paged pool (workload 4)")
    ap.add_argument("--quick", action="store_true",
                    help="device timing only: skip the end-to-end pass, the CPU baseline, the fp8 "
                         "GEMM peak and the other workloads")
    ap.add_argument("--suite", action="store_true",
                    help="with --quick: still time the other workloads and the fp8 GEMM peak")
    a = ap.parse_args(argv)
    if a.gpus < 1 or a.steps < 1 or a.warmup < 3:
        ap.error("need --gpus >= 1, --steps >= 1, --warmup >= 3")
    if a.path == "chained" and (a.workload == 4 or a.impl == "reference"):
        ap.error("--path chained is the prefill comparison path of our implementation")
    if a.path == "act_quant" and (a.workload != 4 or a.impl == "reference"):
        ap.error("--path act_quant fills the paged key pool of workload 4")
    return a


def valid_pairs(ks: torch.Tensor, ke: torch.Tensor, n: int) -> int:
    lo = ks.long().clamp(min=0)
    hi = torch.maximum(lo, ke.long().clamp(max=n))
    return int((hi - lo).sum())


def measured_traffic(workload_name: str):
    """DRAM bytes per launch of the fused kernel from the committed ncu record,
    or None when the CUDA sources changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for src in rec["sources"]:
        with open(os.path.join(ROOT, src), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != rec["sources_sha256"]:
        return None
    e = rec["workloads"].get(workload_name)
    return None if e is None else e["dram_read_bytes"] + e["dram_write_bytes"]


NOMINAL_FP8_TFLOPS = 4500.0  # B200 dense fp8 datasheet figure (context only)
NOMINAL_HBM_GBS = 8000.0      # B200 HBM3e datasheet figure (context only)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p.get("hbm_gbs", 6650.0)), "measured"
    return 1590.0, 6650.0, "fallback"


def measure_fp8_peak(dev, size: int = 8192, reps: int = 10):
    """Dense e4m3 x e4m3 -> bf16 GEMM throughput of the library routine
    torch._scaled_mm at size^3 (best of `reps`, CUDA events): a denominator
    only, nothing of the indexer runs through it.  None if unavailable."""
    try:
        g = torch.Generator(device=dev).manual_seed(0)
        a = torch.randn(size, size, device=dev, generator=g).to(torch.float8_e4m3fn)
        b = torch.randn(size, size, device=dev, generator=g).to(torch.float8_e4m3fn)
        one = torch.ones((), device=dev, dtype=torch.float32)
        for _ in range(3):
            torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return 2.0 * size ** 3 / (best / 1e3) / 1e12
    except Exception as exc:  # pragma: no cover - depends on the torch build
        print(f"fp8 peak measurement unavailable: {exc}", file=sys.stderr)
        return None


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # pragma: no cover - no NVML
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- distributed

def dist_setup(gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != gpus:
        raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local, pg


def barrier(pg):
    if pg is not None:
        pg.barrier()


def max_over_ranks(pg, x: float) -> float:
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world, pg):
    import oracle
    if rank != 0:
        return None
    d = workloads.make_workload(WORKLOAD)
    q, k, s, w = (d[x].numpy() for x in ("q", "k", "s", "w"))
    ks, ke = d["ks"].numpy(), d["ke"].numpy()
    m, n = d["m"], d["n"]
    per_step = 4  # rows per step, walked through the workload with a fixed stride
    order = (np.arange(m, dtype=np.int64) * 2459) % m
    threads = oracle.host_threads()

    def step(i):
        rows = order[(i * per_step) % m: (i * per_step) % m + per_step]
        oracle.mqa_logits_topk_rows(q, k, s, w, ks, ke, workloads.TOPK, rows=rows, threads=threads)
        return sum(max(0, min(int(ke[r]), n) - max(int(ks[r]), 0)) for r in rows)

    for i in range(args.warmup):
        step(i)
    pairs = 0
    t0 = time.perf_counter()
    for i in range(args.steps):
        pairs += step(args.warmup + i)
    dt = time.perf_counter() - t0
    value = FLOP_PER_PAIR * pairs / dt / 1e12
    sample = (f"{args.steps} steps x {per_step} query rows of {d['name']} "
              f"({pairs} valid (row, key) pairs), float64 logits + full-sort top-2048")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": d["name"], "m": m, "n": n, "H": workloads.H, "D": workloads.D,
                   "topk": workloads.TOPK, "seed": d["seed"]},
        "rows_keys_per_s": pairs / dt,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def cpu_baseline(d, budget_s: float = 12.0):
    """The oracle as it stands on this host's cores, on a strided row sample."""
    import oracle
    q, k, s, w = (d[x].numpy() for x in ("q", "k", "s", "w"))
    ks, ke = d["ks"].numpy(), d["ke"].numpy()
    m, n = d["m"], d["n"]
    threads = oracle.host_threads()
    order = (np.arange(m, dtype=np.int64) * 2459) % m
    batch = max(threads, 16)
    pairs, done, t0 = 0, 0, time.perf_counter()
    while done < m and time.perf_counter() - t0 < budget_s:
        rows = order[done: done + batch]
        oracle.mqa_logits_topk_rows(q, k, s, w, ks, ke, workloads.TOPK, rows=rows, threads=threads)
        pairs += sum(max(0, min(int(ke[r]), n) - max(int(ks[r]), 0)) for r in rows)
        done += len(rows)
    dt = time.perf_counter() - t0
    return {"value": FLOP_PER_PAIR * pairs / dt / 1e12, "unit": UNIT, "cores": threads,
            "kind": "oracle",
            "sample": f"{done} of {m} query rows of {d['name']} (strided), {pairs} valid pairs, "
                      f"{dt:.1f} s wall, float64 logits + full-sort top-2048"}


# ----------------------------------------------------------------------------- our arm

CHUNK_BYTES = 2 << 30  # logits bytes per row chunk of the chained path


def make_case(fx, index, dev, path="fused"):
    """Device-resident inputs, outputs, workspace and the C-ABI call for one workload."""
    d = workloads.make_workload(index)
    topk = workloads.TOPK
    if index == 4 and path == "act_quant":
        # every key of every request, as bf16, into its slot of a fresh pool
        L = d["seq_lens"].long()
        bt = d["block_table"].long()
        slot = torch.cat([bt[b, torch.arange(int(L[b])) // 64] * 64 + torch.arange(int(L[b])) % 64
                          for b in range(d["B"])])
        T = slot.numel()
        g = torch.Generator().manual_seed(d["seed"] + 1000)
        xk = (torch.randn(T, workloads.D, generator=g) * 2).to(torch.bfloat16)
        host = {"x": xk.pin_memory(), "slot": slot.pin_memory()}
        dv = {x: host[x].to(dev) for x in host}
        P = d["P"]
        out = torch.empty((P, 64, workloads.D), dtype=torch.uint8, device=dev)
        sp = torch.empty((P, 64), dtype=torch.float32, device=dev)
        out_host = torch.empty(out.shape, dtype=torch.uint8).pin_memory()

        def call():
            fx.act_quant_store(dv["x"], dv["slot"], out, sp)
        return dict(d=d, call=call, host=host, dv=dv, out=out, out_host=out_host, ws=None, pairs=T,
                    flops=0, bytes=T * (2 * workloads.D + 8 + workloads.D + 4),
                    kernel="act_quant_store_kernel (bf16 keys -> e4m3 pool + scales)", bound="hbm",
                    launches=1, metric="k-pool fp8 quantise+store GB/s (act_quant, workload 4 keys)",
                    unit="GB/s")
    if index == 4:
        keys = ("q", "k_pages", "s_pages", "w", "block_table", "seq_lens")
        host = {x: d[x].pin_memory() for x in keys}
        dv = {x: host[x].to(dev) for x in keys}
        rows, R = d["B"] * d["R"], d["R"]
        out = torch.empty((rows, topk), dtype=torch.int32, device=dev)
        ws = fx.alloc_workspace(fx.paged_workspace_size(d["B"], R, d["max_blocks"], topk), dev)
        L = d["seq_lens"].long()
        ke = torch.stack([(L - R + t + 1).clamp(min=0) for t in range(R)], 1).clamp(max=L[:, None])
        pairs = int(ke.sum())
        # algorithmic bytes: every key row + scale read once per request, the block-table
        # entries in use, q and w of the request's rows, and the top-k written
        nbytes = int((L * (workloads.D + 4)).sum() + ((L + 63) // 64).sum() * 4
                     + rows * (workloads.H * workloads.D + workloads.H * 4 + topk * 4))

        def call():
            fx.paged_mqa_logits_topk(**dv, R=R, topk=topk, out=out, workspace=ws)
        kernel = "indexer_kernel<4,true,32,1> (paged fused logits + top-k) + merge_kernel + repair launch"
        bound = "hbm"
    else:
        keys = ("q", "k", "s", "w", "ks", "ke")
        host = {x: d[x].pin_memory() for x in keys}
        dv = {x: host[x].to(dev) for x in keys}
        out = torch.empty((d["m"], topk), dtype=torch.int32, device=dev)
        ws = fx.alloc_workspace(fx.mqa_logits_topk_workspace_size(d["m"], d["n"], topk), dev)
        pairs = valid_pairs(d["ks"], d["ke"], d["n"])
        nbytes = int(d["m"] * (workloads.H * workloads.D + workloads.H * 4 + 8 + topk * 4)
                     + d["n"] * (workloads.D + 4))

        def call():
            fx.mqa_logits_topk(**dv, topk=topk, out=out, workspace=ws)
        kernel = "indexer_kernel<8,false,32,1> (fused logits + top-k) + repair launch"
        bound = "tensor"
        if path == "chained":
            m, n = d["m"], d["n"]
            rows = max(1, min(m, CHUNK_BYTES // (4 * max(n, 1))))
            logits = torch.empty((rows, n), dtype=torch.float32, device=dev)
            chunks = [(r0, min(m, r0 + rows)) for r0 in range(0, m, rows)]

            def call():
                for r0, r1 in chunks:
                    lg = logits[: r1 - r0]
                    fx.mqa_logits(dv["q"][r0:r1], dv["k"], dv["s"], dv["w"][r0:r1], dv["ks"][r0:r1],
                                  dv["ke"][r0:r1], logits=lg)
                    fx.topk_rows(lg, dv["ks"][r0:r1], dv["ke"][r0:r1], topk, out=out[r0:r1])
            kernel = (f"indexer_kernel<8,false,32,0> (materialised logits) + topk_rows_kernel, "
                      f"{len(chunks)} row chunk(s) of <= {rows} rows")
            ws = None
            launches = 2 * len(chunks)
    out_host = torch.empty(out.shape, dtype=torch.int32).pin_memory()
    if path == "fused":
        # the indexer, the merge when the key axis is split, and the repair launch
        # (which ends at once when no estimated threshold was rejected)
        launches = 3 if index in (0, 4) else 2
    return dict(d=d, call=call, host=host, dv=dv, out=out, out_host=out_host, ws=ws, pairs=pairs,
                flops=FLOP_PER_PAIR * pairs, bytes=nbytes, kernel=kernel, bound=bound,
                launches=launches, metric=METRIC, unit=UNIT)


def time_device(call, steps: int, warmup: int, flush, stream):
    """Per-step device times (ms) of `call` with CUDA events on `stream`; L2 is
    flushed (untimed) before every step."""
    for _ in range(warmup):
        call()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize()
    # an untimed spin of about a millisecond first, so that the host has the
    # next steps queued before the GPU reaches them: a host-side delay then
    # cannot leave the GPU idle inside a timed step
    with torch.cuda.stream(stream):
        torch.cuda._sleep(2_000_000)
    for i in range(steps):
        flush.zero_()
        starts[i].record(stream)
        call()
        ends[i].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in zip(starts, ends)]


def time_e2e(call, host, dv, out, out_host, flush, stream, steps, dev, pg):
    """Total device time (ms, max over ranks) of `steps` end-to-end steps:
    each step copies its inputs from pinned host memory, runs the call and
    copies the result back to pinned host memory.  Steps are pipelined the way
    a caller streaming batches would run them: two input and two result
    buffers, uploads and downloads on their own streams, so that one step's
    copies overlap the neighbouring steps' compute (and each other).  Every
    copy of every step, and the L2 flush before each call, lie inside the
    timed region, from the first upload to the last download."""
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    sets = [dict(dv), {x: torch.empty_like(dv[x]) for x in host}]
    outs = [torch.empty_like(out), torch.empty_like(out)]
    hout = [out_host, torch.empty_like(out_host).pin_memory()]
    ready, done, fetched = [None] * steps, [None] * steps, [None] * steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(pg)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):  # untimed: the host queues the steps ahead of the GPU
        torch.cuda._sleep(2_000_000)
    start.record(stream)
    up.wait_stream(stream)
    down.wait_stream(stream)
    for i in range(steps):
        b = i & 1
        with torch.cuda.stream(up):
            if i >= 2:
                up.wait_event(done[i - 2])  # input set b is free once step i - 2's call ran
            for x in host:
                sets[b][x].copy_(host[x], non_blocking=True)
            ready[i] = up.record_event()
        stream.wait_event(ready[i])
        if i >= 2:
            stream.wait_event(fetched[i - 2])  # result buffer b is free once it was read back
        flush.zero_()
        dv.update(sets[b])
        call()
        outs[b].copy_(out, non_blocking=True)
        done[i] = stream.record_event()
        with torch.cuda.stream(down):
            down.wait_event(done[i])
            hout[b].copy_(outs[b], non_blocking=True)
            fetched[i] = down.record_event()
    stream.wait_stream(up)
    stream.wait_stream(down)
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(pg)
    dv.update(sets[0])
    return max_over_ranks(pg, start.elapsed_time(end))


def roofline_of(case, mean_s, peaks):
    """The dominant kernel's achieved figure against its measured peak (and, as
    context, against the nominal datasheet peak and the measured fp8 GEMM)."""
    bf16_peak, hbm_peak, peak_src, fp8_meas = peaks
    fp8_peak = 2.0 * bf16_peak  # measured bf16 burst x nominal fp8/bf16 ratio (4.5 / 2.25)
    if case["bound"] == "tensor":
        achieved = case["flops"] / mean_s / 1e12
        r = {"bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
             "frac": achieved / fp8_peak, "traffic": None,
             "peak_source": f"{peak_src} bf16 burst {bf16_peak} TFLOP/s x 2 (fp8/bf16 nominal ratio)",
             "frac_of_nominal_fp8": achieved / NOMINAL_FP8_TFLOPS}
        if fp8_meas:
            r["frac_of_measured_fp8_gemm"] = achieved / fp8_meas
    else:
        achieved = case["bytes"] / mean_s / 1e9
        r = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
             "frac": achieved / hbm_peak, "traffic": None,
             "peak_source": f"{peak_src} HBM copy bandwidth", "algorithmic_bytes": case["bytes"],
             "frac_of_nominal_hbm": achieved / NOMINAL_HBM_GBS}
    r["kernel"] = case["kernel"]
    return r


SUITE = [(0, "fused"), (2, "fused"), (3, "fused"), (4, "fused"), (4, "act_quant")]

# Index preparation at the shape of the "reuse inference metadata" page: 8
# requests of 1M tokens, 1 (decode), 4 (MTP verify) or 16 (prefill chunk)
# query rows each; a step prepares the rows' key ranges and maps every row's
# top-2048 positions to KV slots through the token table.  The page's H200
# figures after its change are quoted as context.
INDEX_PREP = [("decode", 1, 1.77), ("mtp4", 4, 1.81), ("prefill16", 16, 3.63)]


def time_graph(call, reps_target_ms=200.0, samples=3, per_graph=20):
    """Median over `samples` of the mean time (us) of one `call`, from replays
    of a CUDA graph holding `per_graph` calls back to back (so the graph's own
    launch cost is spread over them), each sample replaying for about
    reps_target_ms."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(3):
            call()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(per_graph):
            call()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(20):
        g.replay()
    e1.record()
    e1.synchronize()
    per = max(e0.elapsed_time(e1) / 20, 1e-4)
    reps = max(20, int(reps_target_ms / per))
    out = []
    for _ in range(samples):
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        e1.synchronize()
        out.append(e0.elapsed_time(e1) / reps / per_graph * 1e3)
    del g
    return statistics.median(out)


def run_index_prep(fx, dev, B=8, L=1 << 20, topk=workloads.TOPK, seed=20270):
    """Index preparation + top-k transform at 8 x 1M tokens (CUDA-graph
    replays), and the parallel long-context ragged copy."""
    gen = torch.Generator().manual_seed(seed)
    table_rows = B + 1
    table = torch.randint(0, 1 << 30, (table_rows, L), generator=gen, dtype=torch.int32).to(dev)
    seq = torch.full((B,), L, dtype=torch.int32, device=dev)
    req = torch.arange(B, dtype=torch.int32, device=dev)
    res = {}
    for name, qn, h200_us in INDEX_PREP:
        rows = B * qn
        q_len = torch.full((B,), qn, dtype=torch.int32, device=dev)
        ks = torch.empty(rows, dtype=torch.int32, device=dev)
        ke = torch.empty_like(ks)
        rt = torch.empty_like(ks)
        # top-k positions inside each row's request segment (ragged key space)
        base = (torch.arange(rows, device=dev) // qn).to(torch.int64) * L
        pos = (torch.randint(0, L - qn, (rows, topk), generator=gen).to(dev) + base[:, None]).to(torch.int32)
        out = torch.empty_like(pos)

        def step():
            fx.prepare_ragged(seq, q_len, req, table, q_cap=rows, with_ragged=False, ks=ks, ke=ke, row_table=rt)
            fx.topk_transform(pos, table, 1, row_base=ks, row_table=rt, out=out)
        us = time_graph(step)
        res[name] = {"us_per_step": us, "rows": rows, "topk": topk, "requests": B, "tokens_per_request": L,
                     "launches": 2, "page_h200_us_context": h200_us}
    # the ragged index copy of the whole batch (8M token slots), read + write
    q1 = torch.ones(B, dtype=torch.int32, device=dev)
    ragged = torch.empty(B * L, dtype=torch.int32, device=dev)
    ks = torch.empty(B, dtype=torch.int32, device=dev)
    ke, rt = torch.empty_like(ks), torch.empty_like(ks)

    def copy():
        fx.prepare_ragged(seq, q1, req, table, q_cap=B, ragged=ragged, ks=ks, ke=ke, row_table=rt)
    us = time_graph(copy, reps_target_ms=100.0)
    res["ragged_copy_8x1M"] = {"us_per_step": us, "gbs": 2 * 4 * B * L / (us * 1e-6) / 1e9,
                              "bytes_per_step": 2 * 4 * B * L}
    del table, ragged
    torch.cuda.empty_cache()
    return res


def run_suite(fx, dev, flush, stream, peaks, steps=10, warmup=3):
    """Device time, throughput and roofline fraction of every other workload
    (and of the key quantisation), each timed like the headline."""
    out = {}
    for index, path in SUITE:
        case = make_case(fx, index, dev, path)
        ms = time_device(case["call"], steps, warmup, flush, stream)
        status = fx.read_device_status(case["ws"]) if case["ws"] is not None else 0
        mean_s = statistics.mean(ms) / 1e3
        roof = roofline_of(case, mean_s, peaks)
        name = case["d"]["name"] + ("" if path == "fused" else f"+{path}")
        out[name] = {"ms_per_step": statistics.mean(ms), "steps": steps, "warmup": warmup,
                     "achieved": roof["achieved"], "unit": roof["unit"], "frac": roof["frac"],
                     "bound": roof["bound"], "kernel": roof["kernel"], "device_status": status,
                     "rows_keys_per_s": case["pairs"] / mean_s if path == "fused" else None}
        for key in ("frac_of_nominal_fp8", "frac_of_nominal_hbm", "frac_of_measured_fp8_gemm"):
            if key in roof:
                out[name][key] = roof[key]
        del case
        torch.cuda.empty_cache()
    return out


def run_ours(args, rank, world, local, pg):
    import fp8_mqa_logits_03_b200 as fx
    from fp8_mqa_logits_03_b200 import build
    if rank == 0 or not os.path.exists(fx.LIB_PATH):
        build.build()
    barrier(pg)
    fx.lib()
    dev = torch.device("cuda", local)
    case = make_case(fx, args.workload, dev, args.path)  # every rank: one independent slice
    d, call, host, dv, out, out_host, ws = (case[x] for x in
                                            ("d", "call", "host", "dv", "out", "out_host", "ws"))
    pairs, flops = case["pairs"], case["flops"]
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    warm_status = fx.read_device_status(ws)  # ws None: the last logits call's status
    if warm_status != 0:
        raise RuntimeError(f"device status {warm_status:#x} set during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(pg)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        with torch.cuda.stream(stream):  # untimed: the host queues the steps ahead of the GPU
            torch.cuda._sleep(2_000_000)
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            call()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    barrier(pg)
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, ends)]
    total_ms = max_over_ranks(pg, sum(step_ms))
    ms_per_step = total_ms / args.steps
    work = flops / 1e12 if case["unit"] == UNIT else case["bytes"] / 1e9  # per step, in the unit's terms
    value = world * work * args.steps / (total_ms / 1e3)
    status = fx.read_device_status(ws)
    kstats = fx.read_device_stats(ws) if ws is not None else None  # counters of the last timed call

    # end to end through the same call: pinned H2D of the inputs, D2H of the top-k
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()
    e2e_value = e2e_ms = None
    if not args.quick:
        e2e_ms = time_e2e(call, host, dv, out, out_host, flush, stream, args.steps, dev, pg)
        e2e_value = world * work * args.steps / (e2e_ms / 1e3)

    mean_s = statistics.mean(step_ms) / 1e3
    roof = roofline_of(case, mean_s, load_peaks() + (None,))
    metric, unit, launches = case["metric"], case["unit"], case["launches"]

    # every rank takes the same steps: the suite runs everywhere, rank 0 reports it
    suite = fp8_meas = None
    if not args.quick or args.suite:
        del case, call, dv, host, out, out_host, ws
        torch.cuda.empty_cache()
        fp8_meas = measure_fp8_peak(dev)
        suite = run_suite(fx, dev, flush, stream, load_peaks() + (fp8_meas,))
        suite["index_prep_8x1M"] = run_index_prep(fx, dev)
        barrier(pg)
    if rank != 0:
        return None
    if fp8_meas and roof["bound"] == "tensor":
        roof["frac_of_measured_fp8_gemm"] = roof["achieved"] / fp8_meas
    # bytes per launch from the ncu record of the fused kernel (other paths have none)
    roof["traffic"] = measured_traffic(d["name"]) if args.path == "fused" else None
    line = {
        "metric": metric, "value": value, "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8e4m3", "data": "synthetic",
        "config": {"workload": d["name"], "H": workloads.H, "D": workloads.D, "topk": workloads.TOPK,
                   "seed": d["seed"], "valid_pairs": pairs,
                   "l2": "flushed before every timed step (256 MiB write, untimed)",
                   "parallelism": f"replicas x{world} (one independent slice per GPU)"},
        "rows_keys_per_s": world * pairs * args.steps / (total_ms / 1e3),
        "roofline": roof,
        "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "ms_per_step": None if e2e_ms is None else e2e_ms / args.steps,
                "pipelined": "two buffer sets; each step's upload and download overlap the neighbouring steps"},
        "gpu_launches": args.steps * launches,
        "clocks": clocks.summary(),
        "device_status": status,
        "kernel_stats": kstats,
        "step_ms": {"min": min(step_ms), "median": statistics.median(step_ms), "max": max(step_ms)},
    }
    if fp8_meas:
        line["fp8_tflops_measured"] = fp8_meas
    if suite is not None:
        line["workloads"] = suite
    for key in ("m", "n", "B", "R"):
        if key in d:
            line["config"][key] = d[key]
    if args.path != "fused":
        line["config"]["path"] = args.path
    if args.workload != 4 and not args.quick and args.path == "fused":  # the oracle's own metric
        line["cpu_baseline"] = cpu_baseline(d)
    return line


def main():
    args = strict_args()
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        if args.workload != WORKLOAD:
            raise SystemExit("--impl reference times the headline workload only")
        line = run_reference(args, 0, args.gpus, None)
        print(json.dumps(line), flush=True)
        return
    rank, world, local, pg = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world, pg)
        else:
            line = run_ours(args, rank, world, local, pg)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if pg is not None:
            pg.destroy_process_group()


if __name__ == "__main__":
    main()
