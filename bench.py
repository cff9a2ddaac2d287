#!/usr/bin/env python
"""Benchmark of the Engram hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
engram_hash_gather (n-gram hash + gather of 16 table rows per token),
engram_gate_fwd and engram_gate_bwd_fused (the gate backward with the
weight-gradient reduction in the same kernel) -- three launches -- and, on
more than one GPU, an all-reduce of dwh/dwe, the path's one exchange step
(NCCL by default; --dist-backend gloo runs the same step over gloo).

Default workload ("full_path"): 4 x 16384 = 65536 tokens with Zipf(1.1) ids
over a 129280-id vocabulary, 2 n-gram layers (2-, 3-grams) x 8 tables of
~1,000,003 rows x 64 bf16 (2.05 GB), gate at H = 7168 with x, k, v and the
upstream gradient drawn N(0,1) in bf16.  Every input is larger than the 126 MB
L2 (each gate tensor is 940 MB), so no L2 flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  After the default workload the same process
measures the other workloads (tiny, gate_fwd, gate_fwdbwd, hash_gather) and
reports them under "configs".  Every "frac" is a fraction of the measured
copy bandwidth (MEASURED_PEAKS.json hbm_gbs); every "frac_nominal" a fraction
of the nominal 8 TB/s HBM3e bandwidth.  With --impl reference the fp64 CPU
oracle is timed instead, on a bounded sample of tokens per step.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Engram gate fwd+bwd tokens/s and HBM GB/s (% of B200 peak) at H=7168"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0     # the ~8 TB/s of B200 HBM3e the targets are stated against
BAR_FRACTION = 0.7           # target: every kernel at >= 70% of the nominal bandwidth
L2_FLUSH_BYTES = 2 * 126 * 1024 * 1024
_CSRC = "engram_conditional_memory_hash_b200/csrc/"
# the sources that define each kernel and its launch (a change to any of them
# makes the committed DRAM counters of that kernel stale)
KERNEL_SOURCES = {
    "hash_gather": ["hash_gather.cuh", "common.cuh", "engram_abi.cu"],
    "gate_fwd": ["gate_kernels.cuh", "common.cuh", "engram_abi.cu"],
    "gate_bwd": ["gate_kernels.cuh", "common.cuh", "engram_abi.cu"],
    "gather_bwd": ["gather_bwd.cuh", "gather_bwd_abi.inl", "hash_gather.cuh", "common.cuh"],
}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


# ------------------------------------------------------------------ helpers --

def algorithmic_bytes(T: int, H: int, L: int, J: int, D: int, G: int) -> dict:
    """Bytes each kernel must move per launch (the minimum: every input read
    once, every output written once; table rows counted per gathered row).
    gate_bwd is the fused backward: its own bytes plus the reduction's
    (partial rows written and read back, dwh and dwe written)."""
    rows = T * L * J
    reduce = G * 4 * H + 2 * 4 * H + 2 * 2 * H
    return {
        # tokens read + idx written + rows read + rows written
        "hash_gather": T * 8 + rows * 8 + 2 * rows * D * 2,
        # x, k, v read; out written; gate written; wh, we read
        "gate_fwd": T * (4 * 2 * H + 4) + 2 * 2 * H,
        # g, x, k, v read; dx, dk, dv written; partial rows written; wh, we
        # read; then the reduction of the partial rows
        "gate_bwd": T * 7 * 2 * H + G * 4 * H + 2 * 2 * H + reduce,
    }


def kernel_entry(us: float, nbytes: int, peak: float) -> dict:
    """Time, algorithmic bandwidth and its fractions of the measured and the
    nominal peak for one launch; us_at_bar is the time at 70% of nominal."""
    gbs = nbytes / (us / 1e6) / 1e9
    return {"us": round(us, 2), "algorithmic_bytes": int(nbytes), "GB/s": round(gbs, 1),
            "frac": round(gbs / peak, 4), "frac_nominal": round(gbs / NOMINAL_HBM_GBS, 4),
            "us_at_bar": round(nbytes / (BAR_FRACTION * NOMINAL_HBM_GBS * 1e9) * 1e6, 2)}


def source_digest(kernel: str) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, _CSRC + rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def committed_traffic(kernel: str, units_per_launch: int):
    """dram bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
    except Exception:
        return None
    e = d.get(kernel)
    if not e or e.get("source_digest") != source_digest(kernel):
        return None
    per_unit = e["dram_bytes"] / e["units"]
    return per_unit * units_per_launch


class ClockSampler:
    """nvidia-smi clocks/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "10", "-i", str(self.idx)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0: float, t1: float):
        rows = [s for (t, s) in self.samples if t0 <= t <= t1] or [s for (_, s) in self.samples]
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


# --------------------------------------------------------- CPU oracle timing --

def oracle_sample_rate(w, hin, gin, n_tokens: int, threads: int = 0):
    """Time the oracle (as it stands) on the first n_tokens of the workload:
    hash + gather + gate forward + gate backward with weight gradients.
    Returns (tokens/s, seconds, threads used)."""
    import oracle
    o = oracle.default()
    if threads:
        o.set_threads(threads)
    S = w.S
    nseq = max(1, n_tokens // S) if n_tokens >= S else 1
    ntok_hash = nseq * S if n_tokens >= S else n_tokens
    toks = hin["tokens"][:nseq] if n_tokens >= S else hin["tokens"][:1, :n_tokens]
    t0 = time.perf_counter()
    idx = o.engram_hash(toks, hin["multipliers"], hin["ngram_n"], hin["table_sizes"],
                        pad_id=hin["pad_id"])
    o.engram_gather(idx, hin["table_sizes"], hin["tables"], w.D)
    t1 = time.perf_counter()
    sub = {n: (a[:n_tokens] if a.ndim == 2 else a) for n, a in gin.items()}
    t2 = time.perf_counter()
    o.engram_gate_fwd(sub["x"], sub["k"], sub["v"], sub["wh"], sub["we"], eps=w.eps)
    o.engram_gate_bwd(sub["g"], sub["x"], sub["k"], sub["v"], sub["wh"], sub["we"], eps=w.eps)
    t3 = time.perf_counter()
    per_token = (t1 - t0) / ntok_hash + (t3 - t2) / n_tokens
    return 1.0 / per_token, (t1 - t0) + (t3 - t2), o.max_threads()


def workload(args):
    """The named workload, optionally cut to its first --tokens tokens (whole
    sequences where possible; used for small profiling runs)."""
    from engram_conditional_memory_hash_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    if getattr(args, "hidden", 0):
        w = dataclasses.replace(w, H=args.hidden)
    if args.tokens and args.tokens < w.T:
        if args.tokens >= w.S:
            w = dataclasses.replace(w, B=args.tokens // w.S)
        else:
            w = dataclasses.replace(w, B=1, S=args.tokens)
    return w


def gather_bwd_bytes(T: int, L: int, J: int, D: int, unique_rows: int) -> int:
    """Bytes engram_gather_bwd must move per call: every entry's index (8 B) and
    bf16 gradient row (2D B) read once, and each of the unique_rows table rows it
    touches read and written once in fp32 (2 x 4D B)."""
    return T * L * J * (8 + 2 * D) + unique_rows * 2 * 4 * D


class L2Flush:
    """Empties L2 between timed launches: writes a buffer twice the L2 size,
    then reads another one, so that the lines the write left dirty are
    written back before the timed launch starts (which then begins on a cold,
    clean L2)."""

    WHAT = "a 252 MB buffer written, then another 252 MB read"

    def __init__(self, dev):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.max()


def time_calls(call, stream, dev, warmup: int, calls: int) -> float:
    """Microseconds per call of `call` (which enqueues GPU work on `stream`):
    `warmup` calls, then `calls` calls enqueued back to back between two CUDA
    events, so that the host's time to issue a call overlaps the GPU's work
    on the previous one."""
    import torch
    for _ in range(warmup):
        call()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(calls):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1) * 1e3 / calls


def host_inputs(w, rank: int):
    from engram_conditional_memory_hash_b200 import inputs
    wr = dataclasses.replace(w, index=w.index + 1000 * rank)
    return inputs.hash_inputs(wr), inputs.gate_inputs(wr)


# ----------------------------------------------------------------- our arm --

def run_ours(args):
    import torch
    import torch.distributed as dist

    import engram_conditional_memory_hash_b200 as eng
    from engram_conditional_memory_hash_b200 import step as engram_step

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        kw = {"device_id": dev} if args.dist_backend == "nccl" else {}
        dist.init_process_group(args.dist_backend, timeout=datetime.timedelta(seconds=120), **kw)
    w = workload(args)
    T, H, L, J, D = w.T, w.H, w.L, w.J, w.D

    t_gen = time.perf_counter()
    hin, gin = host_inputs(w, rank)
    t_gen = time.perf_counter() - t_gen

    def to_dev(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    tables = to_dev(hin["tables"]).view(-1, D)
    st = engram_step.EngramStep(w.B, w.S, H, dev, tables, to_dev(gin["wh"]), to_dev(gin["we"]),
                                hin["multipliers"], hin["ngram_n"], hin["table_sizes"],
                                pad_id=hin["pad_id"], eps=w.eps)
    G = st.G

    def fill(b):
        b.tokens.copy_(torch.from_numpy(hin["tokens"]))
        for n in ("x", "k", "v", "g"):
            getattr(b, n).copy_(torch.from_numpy(gin[n].view(np.int16)).view(torch.bfloat16))
        return b

    buf0 = fill(st.buffers())
    stream = torch.cuda.current_stream(dev)
    names = list(engram_step.LAUNCHES)

    for _ in range(args.warmup):
        st.run(buf0, stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
           for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    start.record(stream)
    for i in range(args.steps):
        st.run(buf0, stream, events=evs[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    wall1 = time.time()
    if world > 1:
        dist.barrier()
    time.sleep(0.2)
    clocks.stop()
    elapsed_ms = start.elapsed_time(end)
    per_kernel_ms = {n: float(np.mean([e[i].elapsed_time(e[i + 1]) for e in evs]))
                     for i, n in enumerate(names)}
    if world > 1:
        t = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_ms = float(t.item())
    ms_per_step = elapsed_ms / args.steps
    tokens_per_s = world * T / (ms_per_step / 1e3)

    ab = algorithmic_bytes(T, H, L, J, D, G)
    peak, peak_kind = measured_peak()

    # Cache-cold control for the gather: the same hash_gather launch on ids drawn
    # uniformly over the vocabulary (no hot rows), L2 flushed before each launch.
    uniform = l2_state = None
    if args.uniform_control and rank == 0 and w.vocab > 0:
        from engram_conditional_memory_hash_b200 import inputs as _inp
        utok = torch.from_numpy(_inp.uniform_ids(w.seed, 99, (w.B, w.S), 0, w.vocab)).to(dev)
        flush = L2Flush(dev)
        # its own outputs: the step's indices in buf0 stay those of the step's
        # tokens (the gather backward below runs on them)
        uidx, urows = torch.empty_like(buf0.idx), torch.empty_like(buf0.rows)
        ts = []
        for it in range(13):
            flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            eng.engram_hash_gather(utok, hin["multipliers"], hin["ngram_n"], hin["table_sizes"],
                                   tables, pad_id=hin["pad_id"], idx_out=uidx,
                                   rows_out=urows, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if it >= 3:
                ts.append(e0.elapsed_time(e1))
        uniform = kernel_entry(float(np.median(ts)) * 1e3, ab["hash_gather"], peak)
        uniform["ids"] = (f"uniform over [0, {w.vocab}), L2 flushed before each launch "
                          f"({L2Flush.WHAT})")
        # The step's own launch (its Zipf ids) after L2 was emptied (clean) and
        # after it was filled with dirty lines (a write of a buffer twice its
        # size): inside the step the launch follows the gate backward, whose
        # last output writes are still in L2 and are written back meanwhile.
        after = {}
        for mode in ("clean", "dirty"):
            ts = []
            for it in range(13):
                if mode == "clean":
                    flush()
                else:
                    flush.w.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                eng.engram_hash_gather(buf0.tokens, hin["multipliers"], hin["ngram_n"],
                                       hin["table_sizes"], tables, pad_id=hin["pad_id"],
                                       idx_out=uidx, rows_out=urows, stream=stream)
                e1.record(stream)
                torch.cuda.synchronize(dev)
                if it >= 3:
                    ts.append(e0.elapsed_time(e1))
            after[mode] = kernel_entry(float(np.median(ts)) * 1e3, ab["hash_gather"], peak)
        l2_state = after
        del flush, uidx, urows

    # Gather backward (the transpose of the gather: row gradients summed into
    # the fp32 table gradient), timed on its own: it is not one of the calls of
    # the step.  d_rows is a synthetic N(0,1) gradient of the gathered rows;
    # d_tables (4.1 GB) accumulates across iterations, which does not change
    # the work.
    gbwd = None
    if args.gather_bwd and rank == 0 and w.has_hash:
        from engram_conditional_memory_hash_b200 import inputs as _inp
        d_rows = torch.from_numpy(_inp.gather_grad_inputs(w).view(np.int16)).view(
            torch.bfloat16).to(dev)
        R = int(hin["table_sizes"].sum())
        d_tables = torch.zeros((R, D), dtype=torch.float32, device=dev)
        ws = torch.empty((eng.engram_gather_bwd_workspace_size(T, L, J, D, R),), dtype=torch.uint8,
                         device=dev)
        first = torch.from_numpy(np.concatenate(
            [[0], np.cumsum(hin["table_sizes"].ravel())[:-1]])).to(dev)
        uniq = int(torch.unique(buf0.idx.view(T, L * J) + first[None]).numel())
        us = time_calls(lambda: eng.engram_gather_bwd(buf0.idx, hin["table_sizes"], d_rows,
                                                      d_tables, workspace=ws, stream=stream),
                        stream, dev, warmup=5, calls=100)
        # idx read + d_rows read + one read and one write of every touched fp32 table row
        gbwd = kernel_entry(us, gather_bwd_bytes(T, L, J, D, uniq), peak)
        gbwd.update({"traffic": committed_traffic("gather_bwd", T), "unique_rows": uniq,
                     "entries": T * L * J, "launches": GATHER_BWD_LAUNCHES,
                     "what": "engram_gather_bwd on the step's indices: rows read once updated "
                             "in place, the rest listed, radix-sorted by row and summed in fp64 "
                             "on a side stream beside the update; fp32 table-gradient update; "
                             "100 calls back to back after 5, CUDA events around them"})
        del d_rows, d_tables, ws

    kern = {n: kernel_entry(per_kernel_ms[n] * 1e3, ab[n], peak) for n in names}
    kern["gate_bwd"]["what"] = ("engram_gate_bwd_fused: backward and weight-gradient reduction "
                                "in one kernel")
    step_bytes = sum(ab.values())
    dominant = max(names, key=lambda n: per_kernel_ms[n])
    roof = {
        "kernel": dominant,
        "bound": "hbm",
        "achieved": round(kern[dominant]["GB/s"], 1),
        "peak": peak,
        "unit": "GB/s",
        "frac": kern[dominant]["frac"],
        "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, a copy-kernel bandwidth)"
        if peak_kind == "measured" else "fallback 6650 GB/s",
        "frac_nominal": kern[dominant]["frac_nominal"],
        "peak_nominal": NOMINAL_HBM_GBS,
        "traffic": committed_traffic(dominant, T),
    }

    # ---- end to end: host buffers in, host buffers out, copies timed -------
    e2e = None
    if args.e2e_steps > 0:
        # Host buffers in and out: pinned host inputs are uploaded on a copy
        # stream, the step's C-ABI calls run on the compute stream, every output
        # is downloaded on a second copy stream.  Two device buffer sets let the
        # upload of step i+1 and the download of step i-1 overlap step i.
        in_names, out_names = engram_step.StepBuffers.INPUTS, engram_step.StepBuffers.OUTPUTS
        host_in = {"tokens": torch.from_numpy(hin["tokens"]).pin_memory()}
        for n in ("x", "k", "v", "g"):
            host_in[n] = torch.from_numpy(gin[n].view(np.int16)).view(torch.bfloat16).pin_memory()
        host_out = {n: torch.empty(getattr(buf0, n).shape, dtype=getattr(buf0, n).dtype,
                                   pin_memory=True) for n in out_names}
        bufs = [buf0, st.buffers()]
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        comp_s = stream
        ev_h2d = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_d2h = [torch.cuda.Event() for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out.values())

        def e2e_step(i):
            bi = i % 2
            b = bufs[bi]
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(ev_comp[bi])        # inputs of step i-2 consumed
                for n in in_names:
                    getattr(b, n).copy_(host_in[n], non_blocking=True)
                ev_h2d[bi].record(h2d_s)
            comp_s.wait_event(ev_h2d[bi])
            if i >= 2:
                comp_s.wait_event(ev_d2h[bi])            # outputs of step i-2 downloaded
            st.run(b, comp_s)
            ev_comp[bi].record(comp_s)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_comp[bi])
                for n in out_names:
                    host_out[n].copy_(getattr(b, n), non_blocking=True)
                ev_d2h[bi].record(d2h_s)

        for i in range(2):                                # warm-up
            e2e_step(i)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(h2d_s)
        for i in range(args.e2e_steps):
            e2e_step(i)
        s1.record(d2h_s)
        torch.cuda.synchronize(dev)
        e_ms = s0.elapsed_time(s1)
        if world > 1:
            t = torch.tensor([e_ms], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        e2e = {"value": round(world * T / (e_ms / args.e2e_steps / 1e3), 1), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": args.e2e_steps,
               "path": "pinned host inputs -> H2D (copy stream) -> the step's three C-ABI calls "
                       "-> D2H of every output (second copy stream); two device buffer sets "
                       "overlap step i's compute with the neighbouring steps' copies"}
        del bufs, host_in, host_out
    del buf0, st, tables
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()

    # ---- the other workloads, one GPU, same process (rank 0 only) -----------
    configs = None
    if args.configs and rank == 0:
        configs = {name: measure_config(name, dev, peak)
                   for name in ("tiny", "gate_fwd", "gate_fwdbwd", "hash_gather")}

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1) -------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n = 64
        rate, secs, cores = oracle_sample_rate(w, hin, gin, n)
        target = args.cpu_seconds
        for _ in range(3):   # small samples overstate the per-token cost: refine the size
            if secs >= 0.8 * target or n >= w.T:
                break
            n = int(min(w.T, max(n, n * 1.1 * target / max(secs, 1e-3))))
            rate, secs, cores = oracle_sample_rate(w, hin, gin, n)
        cpu = {"value": round(rate, 1), "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"first {n} tokens of the workload (hash+gather, gate fwd+bwd with "
                         f"weight gradients), {secs:.1f} s of fp64 CPU work"}
        # the same oracle on one host thread, on a sample sized for about half
        # the all-cores run's time
        n1 = 1024
        rate1, secs1, _ = oracle_sample_rate(w, hin, gin, n1, threads=1)
        if secs1 < 0.4 * target and n1 < w.T:
            n1 = int(min(w.T, n1 * 0.5 * target / max(secs1, 1e-3)))
            rate1, secs1, _ = oracle_sample_rate(w, hin, gin, n1, threads=1)
        import oracle as _oracle
        _oracle.default().set_threads(cores)
        cpu["one_thread"] = {"value": round(rate1, 1), "unit": "tokens/s", "cores": 1,
                             "sample": f"first {n1} tokens, {secs1:.1f} s"}

    clk = clocks.summary(wall0, wall1)
    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(tokens_per_s, 1),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded numpy PCG64: N(0,1) bf16 gate tensors, Zipf(1.1) ids, "
                    "N(0,1) bf16 tables)",
            "config": {
                "workload": f"{w.name}: {w.B}x{w.S} tokens, hash+gather over {L * J} tables of "
                            f"~1M rows x {D} bf16, gate fwd+bwd at H={H}",
                "T": T, "H": H, "L": L, "J": J, "D": D, "G": G,
                "l2": "inputs larger than L2 (940 MB per gate tensor, 2.05 GB tables); no flush",
                "parallelism": f"dp{world} ({args.dist_backend})" if world > 1 else "single GPU",
            },
            "hbm_gbs": round(step_bytes / (ms_per_step / 1e3) / 1e9, 1),
            "hbm_frac": round(step_bytes / (ms_per_step / 1e3) / 1e9 / peak, 4),
            "hbm_frac_nominal": round(step_bytes / (ms_per_step / 1e3) / 1e9 / NOMINAL_HBM_GBS, 4),
            "peaks": {"frac": f"of the measured copy bandwidth, {peak} GB/s ({peak_kind})",
                      "frac_nominal": f"of the nominal {NOMINAL_HBM_GBS:.0f} GB/s",
                      "us_at_bar": f"time at {BAR_FRACTION:.0%} of the nominal bandwidth"},
            "gate_fwd_bwd_tokens_per_s": round(
                world * T / ((per_kernel_ms["gate_fwd"] + per_kernel_ms["gate_bwd"]) / 1e3), 1),
            "kernels": kern,
            "hash_gather_uniform_ids": uniform,
            "hash_gather_after_l2": l2_state,
            "gather_bwd": gbwd,
            "configs": configs,
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": len(names) * args.steps,
            "clocks": clk,
            "input_generation_s": round(t_gen, 1),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


GATHER_BWD_LAUNCHES = 13


def measure_config(name: str, dev, peak: float, iters: int = 20, warmup: int = 3) -> dict:
    """Time the named workload's own calls on one GPU: per launch, the median
    over `iters` iterations of CUDA events around it (after `warmup`).
    Workloads whose inputs fit in L2 (tiny, hash_gather's hot rows) get an L2
    flush before every iteration; the gate workloads' inputs are larger than
    L2 and run back to back."""
    import torch

    import engram_conditional_memory_hash_b200 as eng
    from engram_conditional_memory_hash_b200 import inputs
    from engram_conditional_memory_hash_b200 import step as engram_step

    w = inputs.WORKLOADS[name]
    stream = torch.cuda.current_stream(dev)
    T = w.T

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    calls = {}           # launch name -> callable enqueuing it
    H = w.H
    G = 1
    if w.has_hash:
        h = inputs.hash_inputs(w)
        tokens = torch.from_numpy(h["tokens"]).to(dev)
        tables = bf(h["tables"]).view(-1, w.D)
        idx = torch.empty((w.B, w.S, w.L, w.J), dtype=torch.int64, device=dev)
        rows = torch.empty((w.B, w.S, w.L, w.J, w.D), dtype=torch.bfloat16, device=dev)
        calls["hash_gather"] = lambda: eng.engram_hash_gather(
            tokens, h["multipliers"], h["ngram_n"], h["table_sizes"], tables, pad_id=h["pad_id"],
            idx_out=idx, rows_out=rows, stream=stream)
    if w.has_gate:
        gi = {n: bf(a) for n, a in inputs.gate_inputs(w).items()}
        out = torch.empty_like(gi["x"])
        gate = torch.empty((T,), dtype=torch.float32, device=dev)
        calls["gate_fwd"] = lambda: eng.engram_gate_fwd(
            gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"], eps=w.eps, out=out, gate=gate,
            stream=stream)
        if w.backward:
            G = eng.engram_gate_bwd_num_partials(T, H)
            dx, dk, dv = (torch.empty_like(gi["x"]) for _ in range(3))
            part = torch.empty((G, H), dtype=torch.float32, device=dev)
            tickets = torch.zeros((eng.GATE_BWD_TICKETS,), dtype=torch.int32, device=dev)
            dw = torch.empty((2, H), dtype=torch.float32, device=dev)
            calls["gate_bwd"] = lambda: eng.engram_gate_bwd_fused(
                gi["g"], gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"], eps=w.eps, dx=dx, dk=dk,
                dv=dv, w_partial=part, tickets=tickets, dwh=dw[0], dwe=dw[1], stream=stream)
    names = [n for n in engram_step.LAUNCHES if n in calls]
    flush_l2 = name in ("tiny", "hash_gather")
    flush = L2Flush(dev) if flush_l2 else None
    times = {n: [] for n in names}
    evs = []
    # every iteration enqueued back to back (no host synchronisation between
    # them), events between the launches
    for it in range(warmup + iters):
        if flush is not None:
            flush()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
        ev[0].record(stream)
        for i, n in enumerate(names):
            calls[n]()
            ev[i + 1].record(stream)
        if it >= warmup:
            evs.append(ev)
    torch.cuda.synchronize(dev)
    for ev in evs:
        for i, n in enumerate(names):
            times[n].append(ev[i].elapsed_time(ev[i + 1]))
    assert eng.engram_read_device_error() == 0
    ab = algorithmic_bytes(T, max(H, 1), w.L, w.J, w.D, G)
    kern = {n: kernel_entry(float(np.median(times[n])) * 1e3, ab[n], peak) for n in names}
    total_us = sum(k["us"] for k in kern.values())
    res = {"T": T, "H": H or None, "launches": names, "kernels": kern,
           "tokens_per_s": round(T / (total_us / 1e6), 1),
           "l2": f"flushed before every iteration ({L2Flush.WHAT})" if flush_l2 else
                 "inputs larger than L2; iterations back to back",
           "timing": f"median of {iters} iterations after {warmup}, enqueued back to back, "
                     "CUDA events between the launches"}
    if w.has_hash:
        res["tables"] = f"{w.L * w.J} x ~{w.prime_base} rows x {w.D} bf16, ids {w.ids}"
    return res


# ------------------------------------------- gather backward on its own --

def run_gather_bwd_only(args):
    """Profiling aid: engram_gather_bwd alone on the workload's hash indices
    (no gate tensors, no table values on the device), optionally over tables
    from another prime base (--prime-base) so that a full ncu capture holds a
    few GB.  Prints one JSON line describing this auxiliary measurement."""
    import torch

    import engram_conditional_memory_hash_b200 as eng
    from engram_conditional_memory_hash_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workload(args)
    if args.prime_base:
        w = dataclasses.replace(w, prime_base=args.prime_base)
    T, L, J, D = w.T, w.L, w.J, w.D
    h = inputs.hash_inputs(w, with_tables=False)
    idx, _ = eng.engram_hash_gather(torch.from_numpy(h["tokens"]).to(dev), h["multipliers"],
                                    h["ngram_n"], h["table_sizes"], None, pad_id=h["pad_id"],
                                    want_rows=False)
    d_rows = torch.from_numpy(inputs.gather_grad_inputs(w).view(np.int16)).view(
        torch.bfloat16).to(dev)
    R = int(h["table_sizes"].sum())
    d_tables = torch.zeros((R, D), dtype=torch.float32, device=dev)
    ws = torch.empty((eng.engram_gather_bwd_workspace_size(T, L, J, D, R),), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream(dev)
    us = time_calls(lambda: eng.engram_gather_bwd(idx, h["table_sizes"], d_rows, d_tables,
                                                  workspace=ws, stream=stream),
                    stream, dev, warmup=args.warmup, calls=args.steps)
    assert eng.engram_read_device_error() == 0
    print(json.dumps({"part": "gather_bwd", "workload": w.name, "T": T, "rows": R, "D": D,
                      "us": round(us, 2), "calls": args.steps, "warmup": args.warmup}), flush=True)


def run_hash_gather_only(args):
    """Profiling aid: engram_hash_gather alone on the workload's tokens and
    tables (no gate tensors on the device: about 2.3 GB at the full-path
    workload).  Prints one JSON line describing this auxiliary measurement."""
    import torch

    import engram_conditional_memory_hash_b200 as eng
    from engram_conditional_memory_hash_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workload(args)
    h = inputs.hash_inputs(w)
    tokens = torch.from_numpy(h["tokens"]).to(dev)
    tables = torch.from_numpy(h["tables"].view(np.int16)).view(torch.bfloat16).to(dev)
    idx = torch.empty((w.B, w.S, w.L, w.J), dtype=torch.int64, device=dev)
    rows = torch.empty((w.B, w.S, w.L, w.J, w.D), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    us = time_calls(lambda: eng.engram_hash_gather(tokens, h["multipliers"], h["ngram_n"],
                                                   h["table_sizes"], tables, pad_id=h["pad_id"],
                                                   idx_out=idx, rows_out=rows, stream=stream),
                    stream, dev, warmup=args.warmup, calls=args.steps)
    ab = algorithmic_bytes(w.T, 1, w.L, w.J, w.D, 1)["hash_gather"]
    print(json.dumps({"part": "hash_gather", "workload": w.name, "T": w.T, "us": round(us, 2),
                      "algorithmic_bytes": ab, "GB/s": round(ab / (us / 1e6) / 1e9, 1),
                      "calls": args.steps, "warmup": args.warmup}), flush=True)


def run_gate_only(args):
    """Profiling aid: engram_gate_fwd and engram_gate_bwd_fused alone on the
    workload's gate tensors (no tables on the device; with --tokens 8192 at
    H = 7168 about 1 GB).  Prints one JSON line describing this auxiliary
    measurement."""
    import torch

    import engram_conditional_memory_hash_b200 as eng
    from engram_conditional_memory_hash_b200 import inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workload(args)
    T, H = w.T, w.H
    gi = {n: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
          for n, a in inputs.gate_inputs(w).items()}
    G = eng.engram_gate_bwd_num_partials(T, H)
    out, dx, dk, dv = (torch.empty_like(gi["x"]) for _ in range(4))
    gate = torch.empty((T,), dtype=torch.float32, device=dev)
    part = torch.empty((G, H), dtype=torch.float32, device=dev)
    tickets = torch.zeros((eng.GATE_BWD_TICKETS,), dtype=torch.int32, device=dev)
    dw = torch.empty((2, H), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def fwd():
        eng.engram_gate_fwd(gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"], eps=w.eps, out=out,
                            gate=gate, stream=stream)

    def bwd():
        eng.engram_gate_bwd_fused(gi["g"], gi["x"], gi["k"], gi["v"], gi["wh"], gi["we"],
                                  eps=w.eps, dx=dx, dk=dk, dv=dv, w_partial=part,
                                  tickets=tickets, dwh=dw[0], dwe=dw[1], stream=stream)

    us_f = time_calls(fwd, stream, dev, warmup=args.warmup, calls=args.steps)
    us_b = time_calls(bwd, stream, dev, warmup=args.warmup, calls=args.steps)
    assert eng.engram_read_device_error() == 0
    ab = algorithmic_bytes(T, H, 1, 1, 8, G)
    peak, _ = measured_peak()
    print(json.dumps({"part": "gate", "workload": w.name, "T": T, "H": H, "G": G,
                      "gate_fwd": kernel_entry(us_f, ab["gate_fwd"], peak),
                      "gate_bwd": kernel_entry(us_b, ab["gate_bwd"], peak),
                      "calls": args.steps, "warmup": args.warmup}), flush=True)


# ----------------------------------------------------------- reference arm --

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    w = workload(args)
    hin, gin = host_inputs(w, 0)
    n = args.ref_tokens
    if n <= 0:
        # size each step's sample so that the whole run (warm-up and timed
        # steps) takes about --ref-seconds of CPU time
        rate, _, _ = oracle_sample_rate(w, hin, gin, 256)
        per_step = args.ref_seconds / max(1, args.warmup + args.steps)
        n = int(min(w.T, max(32, rate * per_step)))
    rates, secs_all = [], []
    cores = 0
    for i in range(args.warmup + args.steps):
        rate, secs, cores = oracle_sample_rate(w, hin, gin, n)
        if i >= args.warmup:
            rates.append(rate)
            secs_all.append(secs)
    value = float(np.median(rates))
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * float(np.median(secs_all)), 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (same seeded inputs as the GPU arm)",
        "config": {"workload": f"{w.name}: {w.B}x{w.S} tokens, gate H={w.H}", "T": w.T, "H": w.H},
        "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"first {n} tokens of the workload per step (hash+gather, gate "
                                   "fwd+bwd with weight gradients)"},
        "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="full_path")
    ap.add_argument("--tokens", type=int, default=0,
                    help="cut the workload to its first N tokens (profiling runs)")
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-uniform-control", dest="uniform_control", action="store_false",
                    help="skip the uniform-id hash_gather control measurement")
    ap.add_argument("--no-gather-bwd", dest="gather_bwd", action="store_false",
                    help="skip the separate engram_gather_bwd measurement")
    ap.add_argument("--ref-tokens", type=int, default=0,
                    help="tokens per reference-arm step (0: sized from --ref-seconds)")
    ap.add_argument("--ref-seconds", type=float, default=60.0,
                    help="CPU time the whole reference-arm run aims at")
    ap.add_argument("--part", choices=["all", "gather_bwd", "hash_gather", "gate"], default="all",
                    help="gather_bwd / hash_gather / gate (forward and fused backward): time "
                         "those calls alone (profiling aid)")
    ap.add_argument("--hidden", type=int, default=0,
                    help="with --part gate: another hidden size (e.g. one the generic kernels take)")
    ap.add_argument("--dist-backend", choices=["nccl", "gloo"], default="nccl",
                    help="process-group backend of the multi-GPU all-reduce")
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip the measurements of the other workloads")
    ap.add_argument("--prime-base", type=int, default=0,
                    help="with --part gather_bwd: tables of the primes from this base")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.part == "gather_bwd":
        run_gather_bwd_only(args)
    elif args.part == "hash_gather":
        run_hash_gather_only(args)
    elif args.part == "gate":
        run_gate_only(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
