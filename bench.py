#!/usr/bin/env python
"""Engram forward benchmark on B200.

One step = the whole forward (remap + hash, gather, W_K/W_V projections with
gate partials, gate + causal conv) over one batch of the workload, through
the C ABI.  Default workload: the largest single-GPU prefill, B=8 sequences x
4096 tokens, 16 tables of 2781271 x 128 bf16 (11.4 GB), d_mem 2048, d 2560,
conv width 4.  --workload c2 runs B=4 x 4096 with 16 tables of 1000003 x 64
(d_mem 1024), c4 the decode shape, c5 the host-memory tier.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload c3] [--batch B --table-rows M]

--batch and --table-rows shrink the workload (fewer sequences, smaller prime
tables) for ncu captures that must stay a few GB in size.

Under torchrun every rank runs an independent replica (no collective on the
data path: the forward shards by sequence); timing is the max over ranks.
Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "Engram forward tokens/sec on 1 B200; gather HBM GB/s as % of ~8 TB/s peak"
L2_FLUSH_BYTES = 256 << 20
L2_DESC = (f"flushed before every timed step, outside the events: a {L2_FLUSH_BYTES >> 20} MiB write, then a "
           f"{L2_FLUSH_BYTES >> 20} MiB read that evicts the lines the write left dirty")


class L2Flush:
    """Evicts the step's data from L2 (126 MB) before a timed step.  A write
    of twice L2's size alone leaves L2 full of its own dirty lines, and the
    step's first kernel would pay for writing them back; the read that
    follows leaves clean lines only, as a cache flush-and-invalidate does."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()
SPEC_HBM_GBS = 8000.0


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def describe(wl) -> str:
    return (f"{wl.name}: B={wl.B} T={wl.T} t_begin={wl.t_begin}, V={wl.V}->V'={wl.Vc}, Zipf s={wl.zipf_s}, "
            f"orders {list(wl.orders)} x K={wl.K} ({wl.J} tables of {wl.M} x {wl.D} {wl.dtype}), "
            f"d_mem={wl.d_mem}, d={wl.d}, conv w={wl.w}")


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.index, self.period = index, period_s
        self.samples = []
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(self.period)

    def sample(self):
        if not self.ok:
            return
        try:
            mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
            rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            self.samples.append((mhz, int(rs)))
        except Exception:
            pass

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()
        if not self.samples:
            self.sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"], "samples": 0}
        mhz = sorted(s[0] for s in self.samples)
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(mhz)), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


# ---------------------------------------------------------------- oracle timing (CPU)

def oracle_sample_time(wl, n_tokens: int):
    """Time the oracle (single-threaded, as it stands) on the first n_tokens of
    sequence 0 of the workload.  Untimed preparation: the table rows the sample
    touches are fetched from the seeded generator into compact host tables
    (the sample's indices remapped to them)."""
    import oracle
    sw = wl.replace(B=1, T=n_tokens, t_begin=0)
    inp = synth.Inputs(sw)
    canon, _ = oracle.remap(inp.tok, inp.P)
    idx, _ = oracle.hash_ids(canon, sw.Vc, sw.orders, sw.K, inp.mult, inp.rows)
    U = []
    idx_c = np.empty_like(idx)
    for j in range(sw.J):
        u, inv = np.unique(idx[:, j], return_inverse=True)
        U.append(u)
        idx_c[:, j] = inv
    umax = max(len(u) for u in U)
    compact = np.zeros((sw.J, umax, sw.D), dtype=np.float32)
    for j in range(sw.J):
        compact[j, :len(U[j])] = inp.table_rows(j, U[j])
    rows_c = np.array([len(u) for u in U], dtype=np.uint32)
    h = inp.all_hidden()
    t0 = time.perf_counter()
    canon, _ = oracle.remap(inp.tok, inp.P)
    idx, _ = oracle.hash_ids(canon, sw.Vc, sw.orders, sw.K, inp.mult, inp.rows)
    e = oracle.gather(idx_c, rows_c, compact)
    k = oracle.project(e, inp.Wk)
    v = oracle.project(e, inp.Wv)
    alpha = oracle.gate(h, k, inp.gq, inp.gk, 1e-6)
    vt = alpha[:, None] * v
    u = oracle.conv(vt, inp.conv_w)
    oracle.output(vt, u, h, True)
    return time.perf_counter() - t0


# ---------------------------------------------------------------- DRAM traffic

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture of each kernel on a workload, with the digest of the kernel's
# sources at capture time (their code, comments and blank lines left out):
# once the code changes, the figure no longer describes the kernel and the
# line reports null.  profiles/ holds the capture's summary and the command
# that made it.
CSRC = os.path.join(ROOT, "hashed_gram_embedding_02_b200", "csrc")
KERNEL_SOURCES = {
    "gate_k_tc": ("project_tc.cu", "tc.cuh", "common.cuh", "ptx.cuh"),
    "vconv_tc": ("project_tc.cu", "tc.cuh", "common.cuh", "ptx.cuh"),
    "gate_kv_decode": ("decode_tc.cu", "tc.cuh", "common.cuh", "ptx.cuh"),
    "conv_decode": ("decode_tc.cu", "tc.cuh", "common.cuh", "ptx.cuh"),
    "retrieve": ("retrieve.cu", "common.cuh"),
}
CAPTURED_TRAFFIC = {
    # (workload, kernel): (source digest, bytes per launch)
    # c2 at full size, mean of the five timed steps' launches (profiles/launches_c2.md)
    ("c2", "vconv_tc"): ("c854b247a509134b", 123174144 + 28366950),
    ("c2", "gate_k_tc"): ("c854b247a509134b", 122753075 + 507085),
    ("c2", "retrieve"): ("cd4c38c473a10c27", 28943667 + 190822),
    # c3 kernels on 2 sequences and 499979-row tables (profiles/dram_c3_small.md)
    ("c3-B2-M499979", "vconv_tc"): ("59d2794a31cc0db6", 86297856 + 2050304),
    ("c3-B2-M499979", "gate_k_tc"): ("59d2794a31cc0db6", 86043136 + 130048),
    ("c3-B2-M499979", "retrieve"): ("8c46903b0c8d286e", 29667072 + 480512),
    # c3 and c4 at full size, mean of the five timed steps' launches
    # (profiles/launches_c3.md, profiles/launches_c4.md)
    ("c3", "vconv_tc"): ("c854b247a509134b", 314464102 + 128461363),
    ("c3", "gate_k_tc"): ("c854b247a509134b", 312547584 + 7371162),
    ("c3", "retrieve"): ("cd4c38c473a10c27", 115575347 + 80895590),
    ("c4", "retrieve"): ("cd4c38c473a10c27", 1209139 + 2867),
    ("c4", "gate_kv_decode"): ("6bc5ef79605ad072", 23401165 + 0),
    ("c4", "conv_decode"): ("6bc5ef79605ad072", 11986534 + 0),
}


def _code_only(text: str) -> str:
    """The source without comments and blank lines: editing a comment does
    not change the compiled kernel, so it keeps the capture valid."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def source_digest(files, read=None) -> str:
    """Digest of the kernel's sources (code only).  `read(name)` returns a
    file's text; by default the file under csrc/."""
    if read is None:
        def read(name):
            with open(os.path.join(CSRC, name), encoding="utf-8") as fh:
                return fh.read()
    h = hashlib.sha256()
    for f in files:
        h.update(_code_only(read(f)).encode())
    return h.hexdigest()[:16]


def captured_traffic(workload: str, kernel: str):
    """Captured DRAM bytes per launch, or None when there is no capture of
    this kernel's current sources on this workload."""
    rec = CAPTURED_TRAFFIC.get((workload, kernel))
    if rec is None or kernel not in KERNEL_SOURCES:
        return None
    return rec[1] if source_digest(KERNEL_SOURCES[kernel]) == rec[0] else None


# ---------------------------------------------------------------- ranks

def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest of every rank's x (device-timed milliseconds): the job is
    as slow as its slowest replica.  A collective on the timing scalar only,
    never on the data path."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_workload(wl, rank: int, world: int):
    """Each replica processes its own batch of the same shape (weak scaling)."""
    return wl.replace(seed=wl.seed + 1000 * rank) if world > 1 else wl


def job_tokens_per_s(tokens_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms / 1e3)


# ---------------------------------------------------------------- reference arm

def selected_workload(args):
    """The workload named on the command line, with --batch / --table-rows applied."""
    wl = synth.WORKLOADS[args.workload]
    if args.batch:
        wl = wl.replace(name=f"{wl.name}-B{args.batch}", B=args.batch)
    if args.table_rows:
        if not synth._is_prime(args.table_rows):
            raise SystemExit(f"--table-rows {args.table_rows} is not prime")
        wl = wl.replace(name=f"{wl.name}-M{args.table_rows}", M=args.table_rows)
    if getattr(args, "fp8", False):
        wl = wl.replace(name=f"{wl.name}-fp8", dtype="fp8")
    return wl


def host_cpu():
    """The host's CPU model and logical core count (reported beside the oracle's rate)."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "host_cores": os.cpu_count()}


def run_reference(args, rank, world):
    if rank != 0:
        return
    wl = selected_workload(args)
    n = args.ref_tokens
    if n <= 0:
        # size each step so that warm-up + timed steps take about 90 s
        rate = 16 / oracle_sample_time(wl, 16)
        n = int(max(8, min(1024, rate * 90.0 / (args.steps + args.warmup))))
    for _ in range(args.warmup):
        oracle_sample_time(wl, n)
    ts = [oracle_sample_time(wl, n) for _ in range(args.steps)]
    sec = float(np.mean(ts))
    val = n / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(wl), "sample": f"first {n} tokens of sequence 0 per step"},
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"first {n} tokens of sequence 0, single-threaded fp64 C++ oracle",
                         **host_cpu()},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- host-memory tier

def _mem_available() -> int:
    with open("/proc/meminfo") as f:
        for line in f:
            if line.startswith("MemAvailable:"):
                return int(line.split()[1]) * 1024
    raise RuntimeError("MemAvailable not found in /proc/meminfo")


def run_host_tier(args, wl, rank, world, dev):
    """Tables in host memory: per step, hash -> dedupe (GPU) -> stand-in
    layer GEMM [n x 2560] x [2560 x 10240] on the compute stream while the
    host packs the distinct rows and copies them on a side stream -> staged
    gather -> projections, gate and conv.  Every step takes a fresh token
    batch (its own seed), so rows found in the HBM hot-row cache are rows an
    earlier batch admitted, not the same batch again.  Before timing, the
    cache is filled by --cache-warm batches (retrieval only).  The tables are
    shrunk to the largest prime row count that fits in 30 % of the available
    host memory (the stated 200 GB does not fit), and the line states the
    size."""
    import torch
    import torch.distributed as dist

    import hashed_gram_embedding_02_b200 as eb

    budget = int(0.30 * _mem_available()) // max(1, world)
    wl = synth.host_scaled(wl, budget)
    inp = synth.Inputs(wl)
    dd = inp.device_dense(dev)
    t0 = time.time()
    host = inp.host_tables(dev)
    gen_s = time.time() - t0
    h = inp.device_hidden(dev)
    n = wl.n_tok
    cfg = eb.make_config(orders=wl.orders, heads=wl.K, rows=[int(x) for x in inp.rows], mult=inp.mult,
                         row_dim=wl.D, hidden=wl.d, conv_width=wl.w, vocab=wl.V, canon_vocab=wl.Vc,
                         dtype=eb.ENGRAM_BF16)
    eng = eb.Engram(cfg, B=wl.B, L=wl.T)
    n_threads = max(1, min(16, (os.cpu_count() or 2) - 2))
    tier = eb.HostTier(eng, host, max_lookups=n * wl.J, n_threads=n_threads)
    fetch_mode = args.host_fetch
    map_s = None
    if fetch_mode == "mapped":
        t0 = time.time()
        try:
            tier.map_tables()
            map_s = time.time() - t0
        except eb.EngramError as err:
            print(f"mapping the host tables failed ({err}); packing and copying instead", file=sys.stderr)
            fetch_mode = "copy"
    cache_rows = args.cache_rows
    if cache_rows > 0:
        tier.enable_cache(cache_rows, min_count=2)
    idx = torch.empty(n, wl.J, dtype=torch.int32, device=dev)
    e = torch.empty(n, wl.d_mem, dtype=torch.bfloat16, device=dev)
    y = torch.empty(n, wl.d, dtype=torch.bfloat16, device=dev)
    ws_bytes = eb.engram_workspace_bytes(eng.ctx, wl.B, wl.T)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    x_layer = torch.randn(n, 2560, dtype=torch.bfloat16, device=dev)
    w_layer = torch.randn(2560, 10240, dtype=torch.bfloat16, device=dev) * 0.02
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()
    side = torch.cuda.Stream(priority=-1)
    stats = []
    cstats = []
    batch_no = [0]

    def next_tokens():
        # a fresh seeded Zipf batch of the same shape for every call
        k = batch_no[0]
        batch_no[0] += 1
        return torch.from_numpy(synth.zipf_tokens(wl.replace(seed=wl.seed + 1000 + k))).to(dev, non_blocking=True)

    def engram_part(with_layer: bool, ev_fetch=None, tok=None, full=True):
        tok = next_tokens() if tok is None else tok
        eb.engram_hash(eng.ctx, tok, dd["P"], wl.B, wl.T, wl.T, 0, idx)
        tier.dedupe(idx, n)
        if with_layer:
            torch.matmul(x_layer, w_layer)                      # the preceding layer's work
        if ev_fetch is not None:
            ev_fetch[0].record(side)
        n_unique = tier.fetch(side)
        if ev_fetch is not None:
            ev_fetch[1].record(side)
        tier.gather(n, e)
        if full:
            eb.engram_gate_conv(eng.ctx, e, h, dd["Wk"], dd["Wv"], dd["gq"], dd["gk"], dd["conv_w"], wl.B, wl.T,
                                None, y, None, 1, ws, ws_bytes)
        return n_unique

    def timed(fn, K):
        out = []
        for _ in range(K):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            out.append((a, b))
        torch.cuda.synchronize()
        return float(np.mean([a.elapsed_time(b) for a, b in out]))

    for _ in range(args.cache_warm if cache_rows > 0 else 0):
        engram_part(False, full=False)
    for _ in range(args.warmup):
        engram_part(True)
    torch.cuda.synchronize()
    st, flags = eng.status()
    if st != eb.ENGRAM_OK:
        raise RuntimeError(f"device status {st} flags {flags:#x} after warm-up")
    K = args.steps
    toks = [next_tokens() for _ in range(K)]
    fetch_ev = []

    def step():
        ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        stats.append(engram_part(True, ev, tok=toks[len(fetch_ev)]))
        if fetch_mode == "copy":
            cstats.append(tier.cache_stats())       # the fetch has waited for the batch's counts
        fetch_ev.append(ev)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        step_ms = timed(step, K)
    step_ms = max_over_ranks(step_ms, world, dev)
    fetch_ms = float(np.mean([a.elapsed_time(b) for a, b in fetch_ev]))
    layer_ms = timed(lambda: torch.matmul(x_layer, w_layer), max(3, K // 2))
    toks_alone = [next_tokens() for _ in range(max(3, K // 2))]
    it_alone = iter(toks_alone)
    alone_ms = timed(lambda: engram_part(False, tok=next(it_alone)), len(toks_alone))
    if fetch_mode == "mapped":
        # the mapped fetch learns its counts only when the batch is done: take
        # them from a few more fresh batches, untimed, one at a time
        for _ in range(max(3, min(K, 16))):
            stats_ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            engram_part(True, stats_ev)
            torch.cuda.synchronize()
            cstats.append(tier.cache_stats())
        stats = [c["fetched_rows"] for c in cstats]
    tstats = tier.stats()
    uniq = float(np.mean(stats))
    fetch_bytes = uniq * wl.D * 2
    cache = None
    if cache_rows > 0:
        cached_rows = float(np.mean([c["cached_rows"] for c in cstats]))
        cached_lookups = float(np.mean([c["cached_lookups"] for c in cstats]))
        lookups = float(np.mean([c["lookups"] for c in cstats]))
        cache = {"capacity_rows": cache_rows, "capacity_gb": cache_rows * wl.D * 2 / 1e9, "admit_min_count": 2,
                 "warm_batches": args.cache_warm, "resident_rows_last": cstats[-1]["resident"],
                 "lookup_hit_rate": cached_lookups / lookups,
                 "distinct_rows_per_step": uniq + cached_rows, "cached_rows_per_step": cached_rows,
                 "row_hit_rate": cached_rows / (uniq + cached_rows),
                 "pcie_bytes_saved_per_step": cached_rows * wl.D * 2,
                 "pcie_mb_per_step_without_cache": (uniq + cached_rows) * wl.D * 2 / 1e6}
    # pinned host -> device copy peak of this machine, for the roofline
    probe_h = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
    probe_d = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    h2d_ms = timed(lambda: probe_d.copy_(probe_h, non_blocking=True), 5)
    h2d_peak = (256 << 20) / (h2d_ms / 1e3) / 1e9
    achieved = fetch_bytes / (fetch_ms / 1e3) / 1e9
    st, flags = eng.status()
    if st != eb.ENGRAM_OK:
        raise RuntimeError(f"device status {st} flags {flags:#x} after timing")
    tier.close()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": job_tokens_per_s(n, world, step_ms), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: seeded Zipf tokens (a fresh batch every step), counter-based N(0,s^2) tables (host "
                "memory)/hidden/weights",
        "config": {"workload": describe(wl), "B": wl.B, "seq_len": wl.T, "tokens_per_step": n * world,
                   "host_tables_gb": wl.J * wl.M * wl.D * 2 / 1e9,
                   "table_sizing": f"rows per table = largest prime fitting 30% of MemAvailable ({budget / 1e9:.1f} GB)",
                   "step": "hash, dedupe (against the HBM hot-row cache), stand-in layer GEMM 32768x2560x10240 "
                           "(cuBLAS) overlapping the row fetch on a side stream, staged gather, cache admission, "
                           "projections+gate+conv",
                   "host_fetch": (f"mapped: a GPU kernel reads the distinct rows from the page-locked, mapped host "
                                  f"tables (registered once in {map_s:.1f} s)" if fetch_mode == "mapped" else
                                  "copy: host threads pack the distinct rows into pinned staging, cudaMemcpyAsync"),
                   "parallelism": f"replicas x{world} (no collective)",
                   "l2": L2_DESC},
        "roofline": {"kernel": ("host fetch (GPU reads of mapped host memory)" if fetch_mode == "mapped"
                                else "host fetch (pack + PCIe copy)"), "bound": "pcie", "achieved": achieved,
                     "peak": h2d_peak, "unit": "GB/s", "frac": achieved / h2d_peak, "traffic": None,
                     "peak_source": "pinned 256 MiB H2D copy measured in this run",
                     "algorithmic": f"fetched distinct rows x {wl.D * 2} B = {fetch_bytes / 1e6:.1f} MB per step"},
        "host_tier": {"lookups": n * wl.J, "fetched_rows": uniq, "fetch_mb": fetch_bytes / 1e6,
                      "fetch_ms": fetch_ms, "last_fetch": tstats, "pack_threads": n_threads,
                      "layer_gemm_ms": layer_ms, "engram_alone_ms": alone_ms, "step_ms": step_ms,
                      "overhead_over_layer": (step_ms - layer_ms) / layer_ms, "table_generation_s": gen_s},
        "hot_row_cache": cache,
        # per step: hash, dedupe insert, dedupe slot, staged gather, cache
        # admission (with the cache), key pass, value pass (the stand-in GEMM
        # and the memsets are not this library's)
        "cpu_baseline": None, "e2e": None,
        "gpu_launches": (7 if cache_rows > 0 else 6) * K + (K if fetch_mode == "mapped" else 0),
        "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


def table_grad_bytes(n: int, J: int, D: int, es: int, U: int) -> dict:
    """Algorithmic bytes of one table update from dL/de: what the step must
    read and write at least once.  n tokens, J tables of D-wide rows in
    `es`-byte elements, U distinct rows touched.
      grad_reduce: every lookup's slice of dL/de read once (n*J*D*es), each
        distinct row's fp32 sum written once (U*D*4);
      table_sgd: the sums and row ids read (U*D*4 + U*8), the touched table
        rows read and written (2*U*D*es);
      step: the two, plus the indices read (n*J*4) and the row ids written
        (U*8) by the dedupe."""
    reduce_b = n * J * D * es + U * D * 4
    sgd_b = U * D * 4 + U * 8 + 2 * U * D * es
    return {"grad_reduce": reduce_b, "table_sgd": sgd_b, "step": reduce_b + sgd_b + n * J * 4 + U * 8}


def run_table_grad(args, wl, rank, world, dev):
    """The tables' training update from dL/de: per step, engram_table_grad
    (dedupe, scan, place, ordered per-row sums) then engram_table_sgd on the
    resident tables, with the batch's indices and a seeded dL/de resident in
    HBM.  The row count is read back once after the warm-up, never inside a
    step (the update takes it from device memory)."""
    import torch
    import torch.distributed as dist

    import hashed_gram_embedding_02_b200 as eb

    if wl.dtype != "bf16":
        raise SystemExit("--table-grad times bf16 workloads")
    inp = synth.Inputs(wl)
    dd = inp.device_dense(dev)
    tables = inp.device_tables(dev)
    n, J, D, es = wl.n_tok, wl.J, wl.D, 2
    cfg = eb.make_config(orders=wl.orders, heads=wl.K, rows=[int(x) for x in inp.rows], mult=inp.mult,
                         row_dim=D, hidden=wl.d, conv_width=wl.w, vocab=wl.V, canon_vocab=wl.Vc,
                         dtype=eb.ENGRAM_BF16)
    eng = eb.Engram(cfg)
    idx = torch.empty(n, J, dtype=torch.int32, device=dev)
    tok = torch.from_numpy(inp.tok).to(dev)
    eb.engram_hash(eng.ctx, tok, dd["P"], wl.B, wl.T, wl.T, 0, idx)
    g = torch.Generator(device=dev).manual_seed(wl.seed + 77)
    d_e = (torch.randn(n, wl.d_mem, device=dev, generator=g) * 1e-2).to(torch.bfloat16)
    cap = n * J
    rows = torch.empty(cap, dtype=torch.int64, device=dev)
    grad = torch.empty(cap, D, dtype=torch.float32, device=dev)
    cnt = torch.zeros(1, dtype=torch.int64, device=dev)
    ws_bytes = eb.engram_table_grad_workspace_bytes(eng.ctx, n)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    lr = 1e-3
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def step():
        eb.engram_table_grad(eng.ctx, idx, n, d_e, rows, grad, cnt, ws, ws_bytes)
        eb.engram_table_sgd(eng.ctx, rows, grad, cnt, cap, tables, lr)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    st, flags = eng.status()
    if st != eb.ENGRAM_OK:
        raise RuntimeError(f"device status {st} flags {flags:#x} after warm-up")
    U = int(cnt.item())
    K = args.steps
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev = []
    with ClockSampler(dev.index) as clocks:
        for _ in range(K):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            step()
            b.record(stream)
            ev.append((a, b))
        torch.cuda.synchronize()
    step_ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in ev])), world, dev)

    # per-kernel durations from the library's events, in separate profiled steps
    eb.engram_profile_enable(eng.ctx, True)
    rec = []
    for i in range(K + args.warmup):
        flush()
        eb.engram_table_grad(eng.ctx, idx, n, d_e, rows, grad, cnt, ws, ws_bytes)
        p1 = eb.engram_profile_read(eng.ctx)
        eb.engram_table_sgd(eng.ctx, rows, grad, cnt, cap, tables, lr)
        p2 = eb.engram_profile_read(eng.ctx)
        if i >= args.warmup:
            rec.append(p1 + p2)
    eb.engram_profile_enable(eng.ctx, False)
    names = [nm for nm, _ in rec[0]]
    kms = {nm: float(np.mean([r[j][1] for r in rec])) for j, nm in enumerate(names)}
    st, flags = eng.status()
    if st != eb.ENGRAM_OK:
        raise RuntimeError(f"device status {st} flags {flags:#x} after timing")
    if rank != 0:
        return
    hbm, _, _, peak_src = _peaks()
    nbytes = table_grad_bytes(n, J, D, es, U)
    # the reduce is two launches (short segments by lane groups, long ones a
    # CTA each) over one set of algorithmic bytes: its roofline takes both
    kms_r = {nm: ms for nm, ms in kms.items() if nm != "grad_reduce_long"}
    kms_r["grad_reduce"] = kms.get("grad_reduce", 0.0) + kms.get("grad_reduce_long", 0.0)
    kernels = {nm: {"ms": ms} for nm, ms in kms.items()}
    for nm, ms in kms_r.items():
        if nm in nbytes and ms > 0:
            gbs = nbytes[nm] / (ms / 1e3) / 1e9
            kernels.setdefault(nm, {})
            kernels[nm].update(bound="hbm", achieved=gbs, unit="GB/s", frac=gbs / hbm,
                               **({"ms_both_launches": ms} if nm == "grad_reduce" else {}))
    dom = max(kms_r, key=kms_r.get)
    timed_dom = dom if dom in nbytes else max((nm for nm in kms_r if nm in nbytes), key=kms_r.get)
    dk = kernels[timed_dom]
    step_gbs = nbytes["step"] / (step_ms / 1e3) / 1e9
    # launches per step: dedupe 2, scan 3 blocks + the adds, place 1, reduce 2 (short and long segments), sgd 1
    nb1 = (cap + 4095) // 4096
    nb2 = (nb1 + 4095) // 4096
    per_step = 2 + 3 + (1 if nb2 > 1 else 0) + (1 if nb1 > 1 else 0) + 1 + 2 + 1
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        m = min(n, max(1, args.cpu_tokens))
        idx_np = idx[:m].cpu().numpy().view(np.uint32)
        de_np = d_e[:m].float().cpu().numpy().astype(np.float64)
        t0 = time.perf_counter()
        oracle.table_grad(idx_np, inp.rows, de_np, D)
        cpu_s = time.perf_counter() - t0
        cpu = {"value": m / cpu_s, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"the gradient of the first {m} tokens' lookups ({cpu_s:.2f} s), numpy fp64 "
                         "(np.unique + np.add.at), no table update", **host_cpu()}
    line = {
        "metric": "Engram table backward (sparse gradient from dL/de + SGD update) tokens/sec on 1 B200",
        "value": job_tokens_per_s(n, world, step_ms), "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic: the workload's seeded Zipf tokens hashed on the device, dL/de ~ N(0, 1e-4) bf16",
        "config": {"workload": describe(wl), "B": wl.B, "seq_len": wl.T, "tokens_per_step": n * world,
                   "lookups": cap, "distinct_rows": U, "parallelism": f"replicas x{world} (no collective)",
                   "l2": L2_DESC, "launch": "eager"},
        "roofline": {"kernel": timed_dom + (" (+ grad_reduce_long)" if timed_dom == "grad_reduce" else ""),
                     "bound": "hbm", "achieved": dk.get("achieved"), "peak": hbm,
                     "unit": "GB/s", "frac": dk.get("frac"), "traffic": None,
                     "peak_source": f"{peak_src} HBM copy",
                     "algorithmic": f"{nbytes[timed_dom] / 1e6:.1f} MB per launch"},
        "step_bytes": {"algorithmic_mb": nbytes["step"] / 1e6, "achieved_gbs": step_gbs, "frac": step_gbs / hbm},
        "kernels": kernels, "kernels_ms": kms, "dominant_kernel": dom,
        "cpu_baseline": cpu, "e2e": None, "gpu_launches": per_step * K, "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


def e2e_host(args, eng, inp, dd, tables, h, state, wl, tdt, es, n, K, flush, stream, world, dev):
    """The same step end to end through the C ABI with HOST buffers:
    engram_forward_host copies the ids and h in from pinned host memory and Y
    back out, chunk by chunk, overlapped with the compute; all of it inside
    the events.  Timed as eager calls and as replays of a CUDA graph that
    captured one call (its copies are graph nodes that run again on every
    replay, from and to the same pinned buffers); `value` is the graph
    replay unless the capture failed, as for the device-time figure."""
    import torch
    tok_h = torch.from_numpy(inp.tok).pin_memory()
    h_h = h.cpu().pin_memory()
    y_h = torch.empty(n, wl.d, dtype=tdt).pin_memory()
    Ke = max(3, min(K, 50))

    def call():
        eng.forward_host(tok_h, dd["P"], tables, h_h, dd["Wk"], dd["Wv"], dd["conv_w"], y_h, t_begin=wl.t_begin,
                         gq=dd["gq"], gk=dd["gk"], conv_state=state, add_residual=True)

    def timed(run):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(Ke)]
        for i in range(Ke + 3):
            flush()
            if i >= 3:
                ev[i - 3][0].record(stream)
            run()
            if i >= 3:
                ev[i - 3][1].record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in ev])), world, dev)

    eager_ms = timed(call)
    graph_ms, path = None, "eager calls"
    if not args.no_graph:
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                call()
            torch.cuda.synchronize()
            graph_ms, path = timed(g.replay), "replays of a CUDA graph of one call"
        except Exception as exc:                      # capture unsupported: the eager figure stands
            torch.cuda.synchronize()
            path = f"eager calls (graph capture failed: {type(exc).__name__})"
    e2e_ms = graph_ms if graph_ms is not None else eager_ms
    ids_copied = wl.B * (wl.T - max(0, wl.t_begin - (max(wl.orders) - 1)))
    e2e = {"value": job_tokens_per_s(n, world, e2e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": int(ids_copied * 4 + h_h.numel() * es),
           "d2h_bytes_per_step": int(y_h.numel() * es), "ms_per_step": e2e_ms,
           "eager": {"value": job_tokens_per_s(n, world, eager_ms), "ms_per_step": eager_ms},
           "path": "engram_forward_host: pinned host ids + h in, Y out to pinned host, chunked and overlapped; "
                   + path}
    return e2e


# ---------------------------------------------------------------- our arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="c3", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--batch", type=int, default=0, help="override B (0: the workload's)")
    ap.add_argument("--table-rows", type=int, default=0, help="override the rows per table (a prime; 0: the workload's)")
    ap.add_argument("--cpu-tokens", type=int, default=4096,
                    help="oracle sample for cpu_baseline (default: one full 4096-token sequence)")
    ap.add_argument("--ref-tokens", type=int, default=0,
                    help="oracle sample per reference step (0: sized so the run takes about 90 s)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager launches instead of a CUDA graph replay")
    ap.add_argument("--table-grad", action="store_true",
                    help="time the tables' training update (engram_table_grad + engram_table_sgd) instead of the "
                         "forward")
    ap.add_argument("--branches", type=int, default=1,
                    help="multi-branch module: M residual branches (own W_K, h, gate and Y each; shared tables, "
                         "W_V and conv)")
    ap.add_argument("--fp8", action="store_true",
                    help="tables, W_K and W_V as FP8 E4M3 codes: the projections as FP8 tcgen05 GEMMs")
    ap.add_argument("--sharded", action="store_true",
                    help="split the tables over the ranks (rank r holds shard r); each rank's retrieval reads "
                         "the other ranks' rows over NVLink (CUDA IPC mappings)")
    ap.add_argument("--cache-rows", type=int, default=1 << 22,
                    help="host-memory workload: rows of the HBM hot-row cache (0: none)")
    ap.add_argument("--host-fetch", default="copy", choices=["mapped", "copy"],
                    help="host-memory workload: rows fetched by a GPU kernel reading the mapped host tables, or "
                         "packed by host threads and copied")
    ap.add_argument("--cache-warm", type=int, default=32,
                    help="host-memory workload: batches that fill the hot-row cache before timing")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch
    import torch.distributed as dist

    import hashed_gram_embedding_02_b200 as eb

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    wl = selected_workload(args)
    wl = replica_workload(wl, rank, world)
    if wl.host_tables:
        run_host_tier(args, wl, rank, world, dev)
        if world > 1:
            dist.destroy_process_group()
        return
    if args.table_grad:
        run_table_grad(args, wl, rank, world, dev)
        if world > 1:
            dist.destroy_process_group()
        return
    inp = synth.Inputs(wl)
    dd = inp.device_dense(dev)
    h = inp.device_hidden(dev)
    tdt = torch.float32 if wl.dtype == "f32" else torch.bfloat16      # h and Y
    es = wl.elem_bytes                                                 # tables, e
    cfg = eb.make_config(orders=wl.orders, heads=wl.K, rows=[int(x) for x in inp.rows], mult=inp.mult,
                         row_dim=wl.D, hidden=wl.d, conv_width=wl.w, vocab=wl.V, canon_vocab=wl.Vc,
                         dtype={"bf16": eb.ENGRAM_BF16, "f32": eb.ENGRAM_F32, "fp8": eb.ENGRAM_FP8}[wl.dtype])
    eng = eb.Engram(cfg, B=wl.B, L=wl.T - wl.t_begin)
    n = wl.n_tok
    sharded = None
    tables = None
    if args.sharded:
        # every rank's tables are the same seeded values (the workload's own
        # seed, before the per-replica seeds), split by global row
        tab_inp = synth.Inputs(selected_workload(args))

        def all_gather(obj):
            every = [None] * world
            dist.all_gather_object(every, obj)
            return every
        sharded = eb.ShardedTables(eng, world, rank, wl.D, tdt, dev,
                                   lambda first, cnt, out: tab_inp.device_table_range(first, cnt, out),
                                   all_gather=all_gather)
    else:
        tables = inp.device_tables(dev)
    M = args.branches
    mb = M > 1 or wl.dtype == "fp8"          # the multi-branch entry point (FP8 takes its scales)
    if mb:
        if args.sharded:
            raise SystemExit("--branches / --fp8 and --sharded are separate modes")
        branches = [synth.branch_inputs(inp, m) for m in range(M)]
        bdd = [dd] + [b.device_dense(dev) for b in branches[1:]]
        h = torch.stack([h] + [b.device_hidden(dev) for b in branches[1:]]).contiguous()
        Wk_mb = torch.stack([x["Wk"] for x in bdd]).contiguous()
        ks_mb = torch.stack([x["k_scale"] for x in bdd]).contiguous() if wl.dtype == "fp8" else None
        gq_mb = torch.stack([x["gq"] for x in bdd]).contiguous()
        gk_mb = torch.stack([x["gk"] for x in bdd]).contiguous()
        y = torch.empty(M, n, wl.d, dtype=tdt, device=dev)
    else:
        y = torch.empty(n, wl.d, dtype=tdt, device=dev)
    state = (torch.zeros(M, wl.B, wl.w - 1, wl.d, dtype=torch.float32, device=dev).squeeze(0)
             if wl.t_begin > 0 else None)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()

    def step():
        if mb:
            eng.forward_multibranch(dd["tok"], dd["P"], tables, h, Wk_mb, dd["Wv"], dd["conv_w"], y,
                                    t_begin=wl.t_begin, gq=gq_mb, gk=gk_mb, k_scale=ks_mb, v_scale=dd["v_scale"],
                                    conv_state=state, add_residual=True)
        elif sharded is not None:
            eng.forward_sharded(dd["tok"], dd["P"], sharded.ptrs, h, dd["Wk"], dd["Wv"], dd["conv_w"], y,
                                t_begin=wl.t_begin, gq=dd["gq"], gk=dd["gk"], conv_state=state, add_residual=True)
        else:
            eng.forward(dd["tok"], dd["P"], tables, h, dd["Wk"], dd["Wv"], dd["conv_w"], y, t_begin=wl.t_begin,
                        gq=dd["gq"], gk=dd["gk"], conv_state=state, add_residual=True)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, flags = eng.status()
    if st != eb.ENGRAM_OK:
        raise RuntimeError(f"device status {st} flags {flags:#x} after warm-up")

    # ---- one forward captured as a CUDA graph: the timed loop replays it, so
    # the host's launch work (argument checks, tensor maps, four launches)
    # stays out of the device time of short steps such as decode
    graph, launch = None, "eager"
    if not args.no_graph:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step()
            torch.cuda.synchronize()
            launch = "CUDA graph of one forward (captured after the warm-up), replayed each step"
        except Exception as exc:                      # capture unsupported: time eager launches
            graph, launch = None, f"eager (graph capture failed: {type(exc).__name__})"
            torch.cuda.synchronize()
    run = graph.replay if graph is not None else step
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()

    # ---- timed: K whole steps, L2 flushed before each (outside the events)
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(K):
            flush()
            ev[i][0].record(stream)
            run()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(float(np.mean([a.elapsed_time(b) for a, b in ev])), world, dev)
    value = job_tokens_per_s(n, world, ms)

    # ---- per-kernel durations: the library's own CUDA events around each
    # kernel of engram_forward (same workload, same stream, L2 flushed).
    # The profiled forward is captured as a graph too (its events become
    # event-record nodes), so the host's launch work does not fall between
    # the events of a short kernel
    eb.engram_profile_enable(eng.ctx, True)
    prof_run, prof_launch = step, "eager"
    if graph is not None:
        try:
            pgraph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(pgraph):
                step()
            torch.cuda.synchronize()
            prof_run, prof_launch = pgraph.replay, "graph"
        except Exception:
            torch.cuda.synchronize()
    def profile_steps(run):
        out = []
        for i in range(K + args.warmup):
            flush()
            run()
            prof = eb.engram_profile_read(eng.ctx)
            if i >= args.warmup:
                out.append(prof)
        return out

    rec = profile_steps(prof_run)
    if prof_launch == "graph" and any(t <= 0.0 for r in rec for _, t in r):
        # events that a graph replay recorded without a usable interval: time
        # eager launches instead
        eb.engram_profile_enable(eng.ctx, False)
        eb.engram_profile_enable(eng.ctx, True)
        prof_launch = "eager (graph-recorded events gave no interval)"
        rec = profile_steps(step)
    eb.engram_profile_enable(eng.ctx, False)
    names = [nm for nm, _ in rec[0]]
    kms = {nm: float(np.mean([r[j][1] for r in rec])) for j, nm in enumerate(names)}
    per_step_launches = len(names)

    hbm, tf_burst, tf_sust, peak_src = _peaks()
    if wl.dtype == "fp8":
        # FP8 contraction: the bf16 peak times the nominal dense ratio 4.5 / 2.25
        tf_burst, tf_sust, peak_src = 2.0 * tf_burst, 2.0 * tf_sust, peak_src + " bf16 x 2 (FP8/bf16 nominal)"
    G = (wl.d + 127) // 128
    L = wl.T - wl.t_begin
    pass_flops = 2.0 * n * wl.d_mem * wl.d                      # one of the two projection passes
    work = {
        # name: (bound, algorithmic units per launch, unit)
        # remap + n-grams + hash + gather in one kernel: ids in, indices out,
        # table rows in, e_cat out
        "retrieve": ("hbm", n * (4.0 + wl.J * 4) + wl.B * 4.0 * min(wl.T, 3) + 2.0 * n * wl.d_mem * es, "bytes"),
        "retrieve_sharded": ("hbm", n * (4.0 + wl.J * 4) + wl.B * 4.0 * min(wl.T, 3) + 2.0 * n * wl.d_mem * es,
                             "bytes"),
        "gate_k_tc": ("tensor", M * pass_flops, "flop"),
        "vconv_tc": ("tensor", pass_flops, "flop"),
        # decode (one position per sequence): both contractions in one kernel,
        # then the conv over v: v and alpha in, the history read and
        # rewritten, h in, Y out
        "gate_kv_decode": ("tensor", 2 * pass_flops, "flop"),
        "conv_decode": ("hbm", n * wl.d * (4.0 + 24.0 + 2.0 + 2.0) + n * 4.0 + wl.d * 16.0, "bytes"),
        "state_merge": ("hbm", wl.B * (wl.w - 1) * wl.d * 8.0, "bytes"),
    }
    kern = {}
    for nm, t in kms.items():
        if nm not in work:
            continue
        bound, units, u = work[nm]
        rate = units / (t / 1e3)
        if bound == "tensor":
            kern[nm] = {"ms": t, "bound": "tensor", "achieved": rate / 1e12, "unit": "TFLOP/s",
                        "frac": rate / 1e12 / tf_burst}
        else:
            kern[nm] = {"ms": t, "bound": "hbm", "achieved": rate / 1e9, "unit": "GB/s", "frac": rate / 1e9 / hbm}
        kern[nm]["traffic"] = captured_traffic(wl.name, nm)
    dominant = max(kms, key=kms.get)
    dk = kern.get(dominant, {})
    roofline = {"kernel": dominant, "bound": dk.get("bound"), "achieved": dk.get("achieved"),
                "peak": tf_burst if dk.get("bound") == "tensor" else hbm, "unit": dk.get("unit"),
                "frac": dk.get("frac"), "traffic": dk.get("traffic"),
                # context: the same rate against the sustained (power-capped) figure
                "frac_of_sustained": (dk.get("achieved") / tf_sust) if dk.get("bound") == "tensor" else None,
                "peak_source": f"{peak_src} " + ("bf16 burst" if dk.get("bound") == "tensor" else "HBM copy"),
                "algorithmic": (f"{work[dominant][1]:.4g} FLOP per launch (2*n*d_mem*d per projection)"
                                if dk.get("bound") == "tensor" else f"{work.get(dominant, (0, 0))[1]:.4g} bytes per launch")}
    rname = "retrieve_sharded" if sharded is not None else "retrieve"
    gather_gbs = kern[rname]["achieved"] if rname in kern else None
    gather_bytes = work["retrieve"][1]

    # ---- end to end through the C ABI with HOST buffers: engram_forward_host
    # copies the ids and h in from pinned host memory and Y back out, chunk by
    # chunk, overlapped with the compute; all of it inside the events
    e2e = None
    if sharded is None and not mb:
        e2e = e2e_host(args, eng, inp, dd, tables, h, state, wl, tdt, es, n, K, flush, stream, world, dev)
    elif sharded is not None:
        barrier()                  # every rank is done reading the others' shards
        sharded.close()

    st, flags = eng.status()
    if st != eb.ENGRAM_OK:
        raise RuntimeError(f"device status {st} flags {flags:#x} after timing")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec = oracle_sample_time(wl, args.cpu_tokens)
        cpu = {"value": args.cpu_tokens / sec, "unit": "tokens/s", "cores": 1, "kind": "oracle",
               "sample": f"first {args.cpu_tokens} tokens of sequence 0 ({sec:.1f} s), single-threaded fp64 C++",
               **host_cpu()}

    if world > 1:
        barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8-e4m3 (h, Y bf16)" if wl.dtype == "fp8" else wl.dtype,
        "data": "synthetic: seeded Zipf tokens, counter-based N(0,s^2) tables/hidden/weights",
        "config": {"workload": describe(wl) + (f", {M} branches" if M > 1 else ""), "B": wl.B, "seq_len": wl.T,
                   "tokens_per_step": n * world,
                   "parallelism": (f"tables sharded over {world} GPUs, rows read over NVLink by the retrieval"
                                   if sharded is not None else f"replicas x{world} (no collective)"),
                   "l2": L2_DESC,
                   "launch": launch, "kernel_events": f"per-kernel events, {prof_launch} launches"},
        "roofline": roofline,
        "gather": {"kernel": "retrieve (remap + n-grams + hash + gather)", "achieved_gbs": gather_gbs,
                   "frac_of_8000": gather_gbs / SPEC_HBM_GBS, "frac_of_measured": gather_gbs / hbm,
                   "bytes_per_launch": gather_bytes},
        "kernels": kern, "kernels_ms": kms,
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": per_step_launches * K, "clocks": clocks.summary(),
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
