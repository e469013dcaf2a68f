#!/usr/bin/env python3
"""Bench: paged INT8 KV decode attention on B200 (one JSON line on rank 0).

A step is one pass of the whole hot path over one decode batch:
kv8_quantize_append of the batch's new K/V tokens, then
kv8_paged_decode_attention (one split-K kernel whose last chunk per
sequence and KV head merges the partials) over every sequence's paged INT8
cache.  The default workload is the Llama-3.1-8B layer
shape at batch 64 with 32768-token contexts (4.43 GB of codes and scales,
larger than L2, read once per step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kv8|reference]

Multi-GPU (torchrun, one rank per GPU): sequences are independent, so every
rank runs its own full batch with no data-path collective (weak scaling);
the step time is the max over ranks and ``value`` counts every rank's tokens.

``--impl reference`` times the CPU oracle (the plain C fp64 implementation)
on a bounded sample of the same workload, on rank 0 only.
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
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = ("paged KV8 decode attention tokens/s and achieved HBM GB/s "
          "(% of B200 peak)")
UNIT = "tokens/s"
BYTES_PER_TOKEN_HEAD = 2 * 128 + 2 * 4  # K+V codes and their fp32 scales
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0


# --------------------------------------------------------------------- util
def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def algorithmic_bytes(w: W.Workload) -> dict:
    """Bytes one decode launch must move: codes + scales of every (token,
    KV head) attended, q, out and the block-table entries used."""
    kv = w.token_heads() * BYTES_PER_TOKEN_HEAD
    q = w.batch * w.num_q_heads * w.head_dim * 2
    out = q
    tables = sum(math.ceil(int(t) / w.block_size) for t in w.context_lens) * 4
    return {"kv": kv, "q": q, "out": out, "tables": tables,
            "total": kv + q + out + tables}


def unique_kv_bytes(w: W.Workload) -> int:
    """Codes + scales of the distinct (physical block, KV head) pages the
    launch attends: a block shared by several sequences (a common prefix)
    counts once, with the most tokens any sequence uses of it."""
    used = {}
    for b in range(w.batch):
        t = int(w.context_lens[b])
        for j in range(math.ceil(t / w.block_size)):
            blk = int(w.block_tables[b, j])
            used[blk] = max(used.get(blk, 0), min(w.block_size, t - j * w.block_size))
    return sum(used.values()) * w.num_kv_heads * BYTES_PER_TOKEN_HEAD


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# the translation units a decode launch is built from: the kernel and the
# host code that sizes and launches it (plus the files they include)
DECODE_ROOTS = ("kv8_decode.cu", "kv8_api.cu")


# the KIVI decode's translation unit (its kernels and their entry points)
KIVI_ROOTS = ("kv8_kivi.cu",)


def decode_sources(roots=DECODE_ROOTS) -> list:
    """csrc files a launch is compiled from: `roots` and, recursively, the
    csrc files they #include."""
    csrc = os.path.join(ROOT, "paged_int8_kv_b200", "csrc")
    seen, todo = set(), list(roots)
    while todo:
        fn = todo.pop()
        if fn in seen or not os.path.exists(os.path.join(csrc, fn)):
            continue
        seen.add(fn)
        with open(os.path.join(csrc, fn)) as f:
            for line in f:
                line = line.strip()
                if line.startswith("#include \""):
                    name = line.split('"')[1]
                    if "/" not in name:  # the public header is not csrc
                        todo.append(name)
    return sorted(seen)


def kernel_source_hash(roots=DECODE_ROOTS) -> str:
    """Hash of a launch's sources: a committed DRAM-traffic record counts
    only while it matches (other kernels' files do not enter)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_int8_kv_b200", "csrc")
    for fn in decode_sources(roots):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, roots=DECODE_ROOTS):
    """DRAM bytes per launch from a committed ncu capture, if it was taken
    on the current source of the launch built from `roots` (else None)."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    rec = d.get(workload)
    if not rec or rec.get("source_hash") != kernel_source_hash(roots):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict | None:
        if self.proc is None:
            return None
        try:
            self.proc.terminate()
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                if self.uuid and self.uuid not in parts[1]:
                    continue
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4)
                          if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def max_over_ranks(vals, dist=None, device=None):
    """Element-wise max of per-rank timings (every rank gets the result)."""
    if dist is None:
        return list(vals)
    import torch
    t = torch.tensor(list(vals), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(units_per_rank: int, world: int, ms_per_step: float) -> float:
    """Units all ranks processed per second, over the slowest rank's time."""
    return units_per_rank * world / (ms_per_step * 1e-3)


# ------------------------------------------------------------- CPU oracle
def oracle_sample_seconds(w: W.Workload, seqs, threads: int = 1) -> tuple[float, str]:
    """Time the oracle's decode step (append of the new token + attention
    for every query head) on sequences ``seqs``; cache build excluded.

    With ``threads`` > 1 the attention calls, one per (sequence, KV head),
    run on a pool of that many threads (the oracle is plain single-threaded
    C; its calls release the interpreter lock, so the pool spreads them over
    the host cores)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    prep = []
    for b in seqs:
        k, v = w.sequence_kv(b)
        n = k.shape[0]
        nblk = max(1, math.ceil(n / w.block_size))
        shape = (nblk, w.num_kv_heads, w.block_size, w.head_dim)
        kc = np.full(shape, 127, np.int8)
        vc = np.full(shape, 127, np.int8)
        ks = np.full(shape[:3], np.nan, np.float32)
        vs = np.full(shape[:3], np.nan, np.float32)
        slots = np.arange(n, dtype=np.int64)
        oracle.quantize_append(k[:-1], slots[:-1], kc, ks)
        oracle.quantize_append(v[:-1], slots[:-1], vc, vs)
        prep.append((b, k, v, slots, kc, vc, ks, vs))
    g = w.group
    tasks = [(i, kvh) for i in range(len(prep)) for kvh in range(w.num_kv_heads)]

    def attend(task):
        i, kvh = task
        b, k, v, slots, kc, vc, ks, vs = prep[i]
        table = np.arange(kc.shape[0], dtype=np.int32)[None, :]
        oracle.decode_attention(w.q()[b:b + 1], kc, vc, ks, vs, table,
                                w.context_lens[b:b + 1],
                                pairs=[(0, h) for h in range(kvh * g, (kvh + 1) * g)])

    t0 = time.perf_counter()
    for b, k, v, slots, kc, vc, ks, vs in prep:
        oracle.quantize_append(k[-1:], slots[-1:], kc, ks)
        oracle.quantize_append(v[-1:], slots[-1:], vc, vs)
    if threads > 1:
        with ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(attend, tasks))
    else:
        for t in tasks:
            attend(t)
    total = time.perf_counter() - t0
    desc = (f"{len(seqs)} of {w.batch} sequences of {w.name}: append 1 token "
            f"+ attention for all {w.num_q_heads} query heads over "
            f"{int(w.context_lens[list(seqs)].sum())} tokens (fp64, "
            f"{threads} thread{'s' if threads > 1 else ''})")
    return total, desc


def oracle_kivi_sample_seconds(w: W.Workload, seqs, threads: int = 1) -> tuple[float, str]:
    """Time the oracle's KIVI decode step (append of the new token + attention
    for every query head) on sequences ``seqs``, each in a private cache
    holding its other tokens (cache build excluded); with ``threads`` > 1 the
    sequences run on a pool of that many threads (the C oracle releases the
    interpreter lock).  Returns (seconds, description)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    prep = []
    for b in seqs:
        k, v = w.sequence_kv(b)
        n = k.shape[0]
        nblk = max(1, math.ceil(n / w.block_size))
        table = np.arange(nblk, dtype=np.int32)[None, :]
        c = oracle.KiviCache(nblk, w.num_kv_heads, 1)
        if n > 1:
            oracle.kivi_append(c, k[:-1], v[:-1], np.array([0, n - 1]),
                               np.array([n - 1]), table)
        prep.append((b, k, v, n, table, c))

    def one(item):
        b, k, v, n, table, c = item
        if n:
            oracle.kivi_append(c, k[-1:], v[-1:], np.array([0, 1]), np.array([n]), table)
        oracle.kivi_decode_attention(w.q()[b:b + 1], c, table, np.array([n]))

    used = max(1, min(threads, len(prep)))
    t0 = time.perf_counter()
    if used > 1:
        with ThreadPoolExecutor(max_workers=used) as ex:
            list(ex.map(one, prep))
    else:
        for item in prep:
            one(item)
    total = time.perf_counter() - t0
    desc = (f"{len(prep)} sequences of {w.name} (KIVI), one decode step each "
            f"(append of the new token + all {w.num_q_heads} heads' attention), "
            f"{used} thread{'s' if used > 1 else ''}")
    return total, desc


def oracle_int4_sample_seconds(w: W.Workload, seqs, threads: int = 1) -> tuple[float, str]:
    """oracle_kivi_sample_seconds for the INT4 cache: per sequence, the
    quantise-append of its new token and the attention of all its heads."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    prep = []
    for b in seqs:
        k, v = w.sequence_kv(b)
        n = k.shape[0]
        nblk = max(1, math.ceil(n / w.block_size))
        shape = (nblk, w.num_kv_heads, w.block_size, w.head_dim // 2)
        kc, vc = np.zeros(shape, np.uint8), np.zeros(shape, np.uint8)
        ks, vs = np.zeros(shape[:3], np.float32), np.zeros(shape[:3], np.float32)
        slots = np.arange(n, dtype=np.int64)
        oracle.quantize_append_int4(k[:-1], slots[:-1], kc, ks)
        oracle.quantize_append_int4(v[:-1], slots[:-1], vc, vs)
        prep.append((b, k, v, n, slots, kc, vc, ks, vs))

    def one(item):
        b, k, v, n, slots, kc, vc, ks, vs = item
        oracle.quantize_append_int4(k[-1:], slots[-1:], kc, ks)
        oracle.quantize_append_int4(v[-1:], slots[-1:], vc, vs)
        table = np.arange(kc.shape[0], dtype=np.int32)[None, :]
        oracle.decode_attention_int4(w.q()[b:b + 1], kc, vc, ks, vs, table, np.array([n]))

    used = max(1, min(threads, len(prep)))
    t0 = time.perf_counter()
    if used > 1:
        with ThreadPoolExecutor(max_workers=used) as ex:
            list(ex.map(one, prep))
    else:
        for item in prep:
            one(item)
    total = time.perf_counter() - t0
    desc = (f"{len(prep)} sequences of {w.name} (INT4), one decode step each "
            f"(quantise-append of the new token + all {w.num_q_heads} heads' "
            f"attention), {used} thread{'s' if used > 1 else ''}")
    return total, desc


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, w: W.Workload, rank: int):
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    cores = host_cores()
    nseq = max(1, args.ref_seqs)
    seqs = list(range(min(nseq, w.batch)))
    for _ in range(args.warmup):
        oracle_sample_seconds(w, seqs[:1], cores)
    times = []
    desc = ""
    for i in range(args.steps):
        s, desc = oracle_sample_seconds(w, [seqs[i % len(seqs)]], cores)
        times.append(s)
    sec = sum(times) / len(times)
    value = 1.0 / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, args, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores,
                         "kind": "oracle", "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def bench_config(w: W.Workload, args, world: int) -> dict:
    return {"workload": w.name, "batch": w.batch,
            "context_lens": (int(w.context_lens.min()), int(w.context_lens.max())),
            "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "block_size": w.block_size,
            "chunk_tokens": args.chunk, "num_blocks": w.num_blocks,
            "parallelism": (f"{world} ranks, one GPU each, every rank its own "
                            "batch (sequences independent)" if world > 1 else
                            "1 GPU"),
            "l2": "no flush: the cache read each step is larger than L2"
                  if algorithmic_bytes(w)["total"] > 126e6 * 4 else
                  "L2 flushed between steps"}


# -------------------------------------------------------------- GPU bench
class DeviceWorkload:
    """One workload's cache and decode inputs on the GPU."""

    def __init__(self, w: W.Workload, dev, chunk: int):
        import torch
        from paged_int8_kv_b200.runtime import PagedKV8Cache, fill_from_host
        self.w = w
        self.chunk = chunk
        self.cache = PagedKV8Cache(w.num_blocks, w.num_kv_heads, device=dev)
        fill_from_host(self.cache, w.fill_segments())
        kn, vn, sl = w.step_tokens()
        self.host_step = (kn, vn, sl)
        self.k_new = torch.from_numpy(kn).view(torch.bfloat16).to(dev)
        self.v_new = torch.from_numpy(vn).view(torch.bfloat16).to(dev)
        self.slots = torch.from_numpy(sl).to(dev)
        self.q = torch.from_numpy(w.q()).view(torch.bfloat16).to(dev)
        self.bt = torch.from_numpy(w.block_tables).to(dev)
        self.cl = torch.from_numpy(w.context_lens).to(dev)
        self.out = torch.empty(self.q.shape, dtype=torch.bfloat16, device=dev)
        self.ws = self.cache.workspace(w.batch, w.num_q_heads,
                                       w.max_context_len, chunk)
        # groups sharing a prefix: decoded through the shared-prefix entry
        # point (the shared pages scored once per group)
        self.prefix = None
        if w.prefix_group is not None and w.prefix_len > 0:
            ng = int(w.prefix_group.max()) + 1
            self.prefix = (
                torch.from_numpy(w.prefix_group.astype(np.int32)).to(dev),
                torch.full((ng,), w.prefix_len, dtype=torch.int32, device=dev),
                int(np.bincount(w.prefix_group[w.prefix_group >= 0]).max()),
                w.prefix_len)
        self.use_prefix = self.prefix is not None

    def append(self, k=None, v=None, s=None):
        self.cache.append(self.k_new if k is None else k,
                          self.v_new if v is None else v,
                          self.slots if s is None else s)

    def decode(self, form, q=None, bt=None, cl=None):
        import paged_int8_kv_b200 as pk
        c = self.cache
        if self.use_prefix:
            pg, pl, gmax, plen = self.prefix
            pk.kv8_paged_decode_attention_prefix(
                self.q if q is None else q, c.k_cache, c.v_cache, c.k_scales,
                c.v_scales, self.bt if bt is None else bt,
                self.cl if cl is None else cl, self.out,
                self.w.max_context_len, pg, pl, gmax, plen,
                chunk_tokens=self.chunk, workspace=self.ws)
            return
        pk.kv8_paged_decode_attention_form(
            self.q if q is None else q, c.k_cache, c.v_cache, c.k_scales,
            c.v_scales, self.bt if bt is None else bt,
            self.cl if cl is None else cl, self.out, self.w.max_context_len,
            chunk_tokens=self.chunk, workspace=self.ws, form=form)

    def fused(self, form) -> bool:
        """Whether a step goes through the one-launch entry point (the
        automatic form without shared prefixes)."""
        return form == 0 and not self.use_prefix

    def step_fused(self, q=None, k=None, v=None, bt=None, cl=None):
        import paged_int8_kv_b200 as pk
        c = self.cache
        pk.kv8_paged_decode_attention_append(
            self.q if q is None else q, self.k_new if k is None else k,
            self.v_new if v is None else v, c.k_cache, c.v_cache, c.k_scales,
            c.v_scales, self.bt if bt is None else bt,
            self.cl if cl is None else cl, self.out, self.w.max_context_len,
            chunk_tokens=self.chunk, workspace=self.ws)

    def step(self, form):
        if self.fused(form):
            self.step_fused()
            return
        self.append()
        self.decode(form)


def pick_chunk(w: W.Workload, requested: int) -> int:
    """The split a workload is timed with: the config's own chunk when it
    names one (``requested`` > 0), else the library's suggestion for this
    device (kv8_decode_chunk_tokens)."""
    if requested > 0:
        return requested
    import paged_int8_kv_b200 as pk
    return pk.kv8_decode_chunk_tokens(w.batch, w.num_kv_heads, w.max_context_len)


def time_decode_calls(dw: DeviceWorkload, form: int, calls: int, warmup: int,
                      flush) -> list[float]:
    """Per-call device time (ms) of the decode entry point, CUDA events on
    the launching stream, the L2 flushed before each call when ``flush`` is
    a buffer larger than L2."""
    import torch
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        dw.decode(form)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(calls)]
    for i in range(calls):
        if flush is not None:
            flush_l2(flush)
        ev[i][0].record(stream)
        dw.decode(form)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def time_decode_graph(dw: DeviceWorkload, form: int, calls: int, warmup: int,
                      flush) -> list[float]:
    """Per-call device time (ms) of the decode call captured once in a CUDA
    graph and replayed: the same kernels and arguments as the direct call,
    without the host's argument checks and tensor-map encoding between the
    timing events (a serving loop replays such a graph per step).  The L2 is
    flushed before each replay when ``flush`` is a buffer larger than L2."""
    import torch
    for _ in range(warmup):
        dw.decode(form)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        dw.decode(form)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(calls)]
    for i in range(calls):
        if flush is not None:
            flush_l2(flush)
        ev[i][0].record(stream)
        g.replay()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    del g
    return [a.elapsed_time(b) for a, b in ev]


def flush_l2(buf) -> None:
    """Evict L2 by reading a buffer larger than it (a read leaves no dirty
    lines behind, so the timed call pays no write-back of the flush)."""
    import torch
    buf.view(torch.int64).amax()


def rate_record(w: W.Workload, dec_ms: float, peak: float) -> dict:
    ab = algorithmic_bytes(w)
    gbs = ab["total"] / (dec_ms * 1e-3) / 1e9
    rec = {"decode_us": dec_ms * 1e3,
           "tokens_per_s": w.batch / (dec_ms * 1e-3),
           "kv_tokens_per_s": float(w.context_lens.sum()) / (dec_ms * 1e-3),
           "algorithmic_bytes": ab["total"], "hbm_gbs": gbs,
           "frac_of_measured": gbs / peak,
           "frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS}
    uniq = unique_kv_bytes(w)
    if uniq < ab["kv"]:
        ub = uniq + ab["total"] - ab["kv"]
        rec["unique_bytes"] = ub
        rec["hbm_gbs_unique_bytes"] = ub / (dec_ms * 1e-3) / 1e9
        rec["frac_of_measured_unique_bytes"] = rec["hbm_gbs_unique_bytes"] / peak
    return rec


PER_WORKLOAD = ("tiny", "llama8b_b32", "pruned_compact", "prefix_shared_70b")


def run_per_workload(args, dev, peak: float) -> dict:
    """Decode µs, tokens/s and GB/s of every other configured workload,
    timed one decode call at a time (median of ``--calls`` calls, L2
    flushed before each call: these caches fit in or near L2)."""
    import torch
    flush = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)
    res = {}
    for name in PER_WORKLOAD:
        w = W.NAMED[name]()
        dw = DeviceWorkload(w, dev, pick_chunk(w, 0))
        dw.append()
        ms = time_decode_graph(dw, args.kernel, args.calls, 10, flush)
        api = time_decode_calls(dw, args.kernel, args.calls, 10, flush)
        rec = rate_record(w, statistics.median(ms), peak)
        rec.update({"workload": w.name, "chunk_tokens": dw.chunk,
                    "calls": len(ms), "l2": "flushed before each call",
                    "stat": "median", "timing": "CUDA graph replay of the call",
                    "decode_us_direct_call": statistics.median(api) * 1e3})
        if dw.use_prefix:
            # the same batch through the plain entry point, for comparison
            rec["entry_point"] = "kv8_paged_decode_attention_prefix"
            dw.use_prefix = False
            plain = time_decode_graph(dw, args.kernel, args.calls, 10, flush)
            rec["plain_decode_us"] = statistics.median(plain) * 1e3
        res[name] = rec
        del dw
        torch.cuda.empty_cache()
    del flush
    return res


def run_kv8(args, w: W.Workload, rank: int, world: int, dist):
    import torch
    import paged_int8_kv_b200 as pk

    dev = torch.device("cuda", _env_int("LOCAL_RANK", 0))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    form = args.kernel
    dw = DeviceWorkload(w, dev, pick_chunk(w, args.chunk))
    args.chunk = dw.chunk
    flush = None
    ab = algorithmic_bytes(w)
    if ab["total"] <= 4 * 126e6:
        flush = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)
    # per step: one decode kernel with the append fused in (automatic form),
    # else the quantize-append kernel and the decode kernel; a split launch
    # also enqueues a small memset of its merge tickets
    fused = dw.fused(form)
    launches_per_step = 1 if fused else 2
    if fused:  # the step's new K/V read and their codes and scales written
        nt = w.batch * w.num_kv_heads * 2
        ab = dict(ab, append=nt * (w.head_dim * 2 + w.head_dim + 4),
                  total=ab["total"] + nt * (w.head_dim * 2 + w.head_dim + 4))
    memsets_per_step = 1 if dw.ws is not None else 0

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        dw.step(form)
    torch.cuda.synchronize()

    # ---- device-resident timed region
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    barrier()
    torch.cuda.synchronize()
    # clocks: the sampler starts under the same load (untimed steps for about
    # a second) so that its samples cover the timed region and the load
    # leading into it
    sampler.start()
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < 1.0:
        for _ in range(20):
            dw.step(form)
        torch.cuda.synchronize()
    barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush_l2(flush)
        ev[i][0].record(stream)
        if fused:
            dw.step_fused()
        else:
            dw.append()
            dec[i][0].record(stream)
            dw.decode(form)
            dec[i][1].record(stream)
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    # the decode kernel's time: the whole step when the append is fused in
    dec_ms = step_ms if fused else [a.elapsed_time(b) for a, b in dec]
    ms = sum(step_ms) / len(step_ms)
    if flush is None:
        ms = t_start.elapsed_time(t_end) / args.steps
    dms = sum(dec_ms) / len(dec_ms)

    # ---- for comparison: the same steps as two calls (quantize-append, then
    # the decode call), device-resident like the above
    two_ms = two_dec_ms = None
    if fused:
        tev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for _ in range(args.warmup):
            dw.append()
            dw.decode(form)
        torch.cuda.synchronize()
        barrier()
        for i in range(args.steps):
            if flush is not None:
                flush_l2(flush)
            tev[i][0].record(stream)
            dw.append()
            tev[i][1].record(stream)
            dw.decode(form)
            tev[i][2].record(stream)
        torch.cuda.synchronize()
        two_ms = statistics.mean(a.elapsed_time(c) for a, _, c in tev)
        two_dec_ms = statistics.mean(b.elapsed_time(c) for _, b, c in tev)
        barrier()

    # ---- end to end through the public API: host buffers in, result out
    kn, vn, sl = dw.host_step
    pin = lambda a: torch.from_numpy(a).pin_memory()  # noqa: E731
    h_k, h_v, h_s = pin(kn), pin(vn), pin(sl)
    h_q, h_bt, h_cl = pin(w.q()), pin(w.block_tables), pin(w.context_lens)
    h_out = torch.empty(dw.q.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size()
              for t in ((h_k, h_v, h_q, h_bt, h_cl) if fused else
                        (h_k, h_v, h_s, h_q, h_bt, h_cl)))
    d2h = h_out.numel() * h_out.element_size()
    d_k, d_v, d_s = torch.empty_like(dw.k_new), torch.empty_like(dw.v_new), torch.empty_like(dw.slots)
    d_q, d_bt, d_cl = torch.empty_like(dw.q), torch.empty_like(dw.bt), torch.empty_like(dw.cl)

    def e2e_step():
        d_k.view(torch.int16).copy_(h_k.view(torch.int16), non_blocking=True)
        d_v.view(torch.int16).copy_(h_v.view(torch.int16), non_blocking=True)
        d_s.copy_(h_s, non_blocking=True)
        d_q.view(torch.int16).copy_(h_q.view(torch.int16), non_blocking=True)
        d_bt.copy_(h_bt, non_blocking=True)
        d_cl.copy_(h_cl, non_blocking=True)
        if fused:
            dw.step_fused(d_q, d_k, d_v, d_bt, d_cl)
        else:
            dw.append(d_k, d_v, d_s)
            dw.decode(form, d_q, d_bt, d_cl)
        h_out.copy_(dw.out, non_blocking=True)

    # the same lead-in as the device-timed region: about a second of the same
    # steps under load while the clock sampler runs, so that both numbers
    # are taken at the clocks a sustained run settles to
    e2e_sampler = ClockSampler(uuid)
    e2e_sampler.start()
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < 1.0:
        for _ in range(10):
            e2e_step()
        torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        if flush is not None:
            flush_l2(flush)
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.steps
    barrier()
    e2e_clocks = e2e_sampler.stop()

    # ---- max over ranks
    ms, dms, e2e_ms = max_over_ranks([ms, dms, e2e_ms], dist, dev)
    if two_ms is not None:
        two_ms, two_dec_ms = max_over_ranks([two_ms, two_dec_ms], dist, dev)

    status = pk.kv8_read_device_status(clear=True)
    peak, peak_kind = measured_peaks()
    del dw, flush
    torch.cuda.empty_cache()
    # the other workloads, one GPU each rank (rank 0 reports them)
    per = None
    if not args.no_per_workload:
        per = run_per_workload(args, dev, peak)
    if rank != 0:
        return 0

    value = whole_job_rate(w.batch, world, ms)
    achieved = ab["total"] / (dms * 1e-3) / 1e9
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        seqs = list(range(min(args.cpu_seqs, w.batch)))
        cores = host_cores()
        sec, desc = oracle_sample_seconds(w, seqs, cores)
        sec1, desc1 = oracle_sample_seconds(w, seqs, 1)
        cpu = {"value": len(seqs) / sec, "unit": UNIT, "cores": cores,
               "kind": "oracle", "sample": desc,
               "single_thread": {"value": len(seqs) / sec1, "unit": UNIT,
                                 "cores": 1, "sample": desc1}}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "kv_dtype": "int8", "out_dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q/K/V, shuffled blocks)",
        "config": bench_config(w, args, world),
        "decode_form": form,
        "hbm_gbs": achieved,
        **({"hbm_gbs_unique_bytes": (uniq + ab["total"] - ab["kv"]) / (dms * 1e-3) / 1e9,
            "unique_bytes": uniq + ab["total"] - ab["kv"]}
           if (uniq := unique_kv_bytes(w)) < ab["kv"] else {}),
        "hbm_frac_of_measured": achieved / peak,
        "hbm_frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
        "decode_us": dms * 1e3,
        "decode_us_x_sm_mhz": (dms * 1e3 * clocks["sm_mhz"]
                               if clocks and clocks.get("sm_mhz") else None),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                                    if peak_kind == "measured" else "fallback 6650 GB/s",
                     "kernel": ("decode kernel (fused append, split-K pages, fused "
                                "chunk merge), timed as the whole "
                                "kv8_paged_decode_attention_append step" if fused else
                                "decode kernel (split-K pages + fused chunk merge), "
                                "timed as the kv8_paged_decode_attention call"),
                     "algorithmic_bytes": ab["total"],
                     "traffic": recorded_traffic(w.name)},
        "e2e": {"value": whole_job_rate(w.batch, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms, "clocks": e2e_clocks},
        "step_entry_point": ("kv8_paged_decode_attention_append (append fused "
                             "into the decode kernel)" if fused else
                             "kv8_quantize_append + the decode call"),
        "two_call_step": (
            {"ms_per_step": two_ms, "decode_us": two_dec_ms * 1e3,
             "value": whole_job_rate(w.batch, world, two_ms), "unit": UNIT,
             "entry_points": "kv8_quantize_append, kv8_paged_decode_attention"}
            if two_ms is not None else None),
        "gpu_launches": launches_per_step * args.steps,
        "memsets": memsets_per_step * args.steps,
        "clocks": clocks,
        "device_status": status,
        "per_workload": per,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def extend_flops(lens, new, num_q_heads: int, head_dim: int = 128) -> int:
    """Algorithmic flops of a causal extend: every new row of every query
    head against every token it sees, 2*d for q.k and 2*d for p.v."""
    total = 0
    for t, n in zip(lens, new):
        keys = sum(t - n + i + 1 for i in range(n))
        total += 4 * head_dim * keys * num_q_heads
    return total


def run_extend(args, rank: int, world: int, dist):
    """Extend (chunked-prefill) attention: batch 4 sequences of the
    Llama-3.1-8B head shape, 32768 cached tokens each, of which the last
    2048 are the new query rows; one kv8_paged_extend_attention call per
    step, inputs resident (1.1 GB of cache, larger than L2)."""
    import torch
    import paged_int8_kv_b200 as pk
    dev = torch.device("cuda", _env_int("LOCAL_RANK", 0))
    torch.cuda.set_device(dev)
    B, T, NEW = 4, 32768, 2048
    w = W.make_workload("llama8b_extend_b4_ctx32k_new2k", 1006, [T] * B, 32, 8,
                        description="batch 4, context 32768, 2048 new rows each")
    dw = DeviceWorkload(w, dev, 0)
    qs = np.arange(0, (B + 1) * NEW, NEW, dtype=np.int32)
    rng = np.random.default_rng([1006, 9])
    qh = W.f32_to_bf16_bits(rng.standard_normal((B * NEW, 32, 128), dtype=np.float32))
    q = torch.from_numpy(qh).view(torch.bfloat16).to(dev)
    qsd = torch.from_numpy(qs).to(dev)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    c = dw.cache

    def call():
        pk.kv8_paged_extend_attention(q, c.k_cache, c.v_cache, c.k_scales,
                                      c.v_scales, dw.bt, dw.cl, qsd, out, NEW)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    stream = torch.cuda.current_stream()
    for a, b in ev:
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    ms = statistics.median([a.elapsed_time(b) for a, b in ev])
    ms = max_over_ranks([ms], dist, dev)[0]
    status = pk.kv8_read_device_status(clear=True)
    fl = extend_flops([T] * B, [NEW] * B, 32)
    peak = None
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak = float(json.load(f)["bf16_tflops"])
    except Exception:
        peak = 1590.0
    tflops = fl / (ms * 1e-3) / 1e12
    if rank == 0:
        print(json.dumps({
            "metric": "paged KV8 extend attention new tokens/s and tensor TFLOP/s",
            "value": whole_job_rate(B * NEW, world, ms), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16 operands, f32 accumulation",
            "data": "synthetic (seeded N(0,1))",
            "config": {"workload": w.name, "batch": B, "context": T,
                       "new_rows": NEW, "q_heads": 32, "kv_heads": 8},
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak,
                         "unit": "TFLOP/s", "frac": tflops / peak,
                         "algorithmic_flops": fl,
                         "peak_source": "MEASURED_PEAKS.json bf16_tflops (fp16 "
                                        "runs at the bf16 rate)"},
            "device_status": status}), flush=True)
    return 0


INT4_BYTES_PER_TOKEN_HEAD = 2 * 64 + 2 * 4  # packed K+V nibbles, fp32 scales


def run_int4(args, w: W.Workload, rank: int, world: int, dist):
    """The INT4 cache variant on the timed workload: one step = the step's
    INT4 quantise-append plus one kv8_int4_paged_decode_attention call,
    inputs resident (the 32K workload's INT4 cache, 2.2 GB, is larger than
    L2)."""
    import torch
    import paged_int8_kv_b200 as pk
    dev = torch.device("cuda", _env_int("LOCAL_RANK", 0))
    torch.cuda.set_device(dev)
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim // 2)
    kc = torch.zeros(shape, dtype=torch.uint8, device=dev)
    vc = torch.zeros(shape, dtype=torch.uint8, device=dev)
    ks = torch.zeros(shape[:3], dtype=torch.float32, device=dev)
    vs = torch.zeros(shape[:3], dtype=torch.float32, device=dev)

    def to_dev(a, bf16=True):
        t = torch.from_numpy(a).pin_memory().to(dev, non_blocking=True)
        return t.view(torch.bfloat16) if bf16 else t
    for k, v, sl in w.fill_segments():
        if sl.shape[0]:
            pk.kv8_int4_quantize_append(to_dev(k), to_dev(v), to_dev(sl, False),
                                        kc, vc, ks, vs)
    kn, vn, sl = w.step_tokens()
    k_new, v_new, slots = to_dev(kn), to_dev(vn), to_dev(sl, False)
    q = to_dev(w.q())
    bt = torch.from_numpy(w.block_tables).to(dev)
    cl = torch.from_numpy(w.context_lens).to(dev)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    chunk = pick_chunk(w, args.chunk)
    nbytes = pk.kv8_decode_workspace_bytes(w.batch, w.num_q_heads, w.head_dim,
                                           w.max_context_len, chunk)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def decode():
        pk.kv8_int4_paged_decode_attention(q, kc, vc, ks, vs, bt, cl, out,
                                           w.max_context_len,
                                           chunk_tokens=chunk, workspace=ws)

    def step():
        pk.kv8_int4_quantize_append(k_new, v_new, slots, kc, vc, ks, vs)
        decode()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks([t0.elapsed_time(t1) / args.steps], dist, dev)[0]
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for a, b in ev:
        a.record(stream)
        decode()
        b.record(stream)
    torch.cuda.synchronize()
    dec_ms = statistics.median([a.elapsed_time(b) for a, b in ev])
    status = pk.kv8_read_device_status(clear=True)
    ab = algorithmic_bytes(w)
    kv = w.token_heads() * INT4_BYTES_PER_TOKEN_HEAD
    total = kv + ab["total"] - ab["kv"]
    peak, src = measured_peaks()
    gbs = total / (dec_ms * 1e-3) / 1e9
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        seqs = list(range(min(args.cpu_seqs, w.batch)))
        cores = host_cores()
        sec, desc = oracle_int4_sample_seconds(w, seqs, cores)
        cpu = {"value": len(seqs) / sec, "unit": "tokens/s",
               "cores": max(1, min(cores, len(seqs))), "kind": "oracle",
               "sample": desc}
    if rank == 0:
        print(json.dumps({
            "metric": "paged INT4-KV decode attention tokens/s and achieved HBM GB/s",
            "value": whole_job_rate(w.batch, world, ms), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u4 codes, s8/u8 integer mma, f32 softmax",
            "data": "synthetic (seeded N(0,1))",
            "config": {"workload": w.name + "_int4", "batch": w.batch,
                       "context_tokens": int(w.context_lens.sum()),
                       "chunk_tokens": chunk, "l2": "inputs larger than L2"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak,
                         "unit": "GB/s", "frac": gbs / peak,
                         "traffic": None, "peak_source": src,
                         "algorithmic_bytes": total,
                         "decode_us": dec_ms * 1e3},
            "cpu_baseline": cpu,
            "device_status": status}), flush=True)
    return 0


KIVI_PAGE_BYTES = 2176  # one (block, KV head) page record of the KIVI cache


def kivi_algorithmic_bytes(w: W.Workload) -> dict:
    """Bytes one KIVI decode launch must move: the page record of every full
    page attended, the bf16 K and V rows of each partial page (read from the
    tail), q, out and the block-table entries used."""
    full = sum(int(t) // w.block_size for t in w.context_lens)
    rows = sum(int(t) % w.block_size for t in w.context_lens)
    kv = (full * KIVI_PAGE_BYTES + rows * 2 * w.head_dim * 2) * w.num_kv_heads
    ab = algorithmic_bytes(w)
    return {"kv": kv, "total": kv + ab["total"] - ab["kv"]}


def run_kivi(args, w: W.Workload, rank: int, world: int, dist):
    """The KIVI cache variant on the timed workload: one step = the step's
    kv8_kivi_append (one token per sequence; a token that completes its page
    quantises it) plus one kv8_kivi_paged_decode_attention call, inputs
    resident (the 32K workload's page records, 2.3 GB, are larger than L2)."""
    import torch
    import paged_int8_kv_b200 as pk
    dev = torch.device("cuda", _env_int("LOCAL_RANK", 0))
    torch.cuda.set_device(dev)
    cache = torch.zeros((w.num_blocks, w.num_kv_heads, KIVI_PAGE_BYTES),
                        dtype=torch.uint8, device=dev)
    tail = torch.zeros((w.batch, w.num_kv_heads, 2, w.block_size, w.head_dim),
                       dtype=torch.bfloat16, device=dev)
    bt = torch.from_numpy(w.block_tables).to(dev)

    def to_dev(a, bf16=False):
        t = torch.from_numpy(np.ascontiguousarray(a)).pin_memory().to(dev, non_blocking=True)
        return t.view(torch.bfloat16) if bf16 else t

    def call_args(c):
        k, v, cu, cl = c
        return (to_dev(k, True), to_dev(v, True), to_dev(cu), to_dev(cl), bt,
                cache, tail, max(int(np.diff(cu).max(initial=0)), 1))
    for c in w.kivi_fill_calls():
        pk.kv8_kivi_append(*call_args(c))
        torch.cuda.synchronize()  # the pinned host rows are reused
    step_args = call_args(w.kivi_step_call())
    q = to_dev(w.q(), True)
    cl = torch.from_numpy(w.context_lens).to(dev)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    chunk = pick_chunk(w, args.chunk)
    nbytes = pk.kv8_decode_workspace_bytes(w.batch, w.num_q_heads, w.head_dim,
                                           w.max_context_len, chunk)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def decode():
        pk.kv8_kivi_paged_decode_attention(q, cache, tail, bt, cl, out,
                                           w.max_context_len,
                                           chunk_tokens=chunk, workspace=ws)

    def step():
        pk.kv8_kivi_append(*step_args)
        decode()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks([t0.elapsed_time(t1) / args.steps], dist, dev)[0]
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for a, b in ev:
        a.record(stream)
        decode()
        b.record(stream)
    torch.cuda.synchronize()
    dec_ms = statistics.median([a.elapsed_time(b) for a, b in ev])
    status = pk.kv8_read_device_status(clear=True)
    total = kivi_algorithmic_bytes(w)["total"]
    peak, src = measured_peaks()
    gbs = total / (dec_ms * 1e-3) / 1e9
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        seqs = list(range(min(args.cpu_seqs, w.batch)))
        cores = host_cores()
        sec, desc = oracle_kivi_sample_seconds(w, seqs, cores)
        cpu = {"value": len(seqs) / sec, "unit": "tokens/s",
               "cores": max(1, min(cores, len(seqs))), "kind": "oracle",
               "sample": desc}
    if rank == 0:
        print(json.dumps({
            "metric": "paged KIVI-KV decode attention tokens/s and achieved HBM GB/s",
            "value": whole_job_rate(w.batch, world, ms), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u2 codes, f32 CUDA-core arithmetic",
            "data": "synthetic (seeded N(0,1))",
            "config": {"workload": w.name + "_kivi", "batch": w.batch,
                       "context_tokens": int(w.context_lens.sum()),
                       "chunk_tokens": chunk, "l2": "inputs larger than L2"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak,
                         "unit": "GB/s", "frac": gbs / peak,
                         "traffic": recorded_traffic(w.name + "_kivi", KIVI_ROOTS),
                         "peak_source": src,
                         "algorithmic_bytes": total,
                         "decode_us": dec_ms * 1e3},
            "cpu_baseline": cpu,
            "device_status": status}), flush=True)
    return 0


def run_dry_cpu(args, rank: int, world: int, dist):
    """The launch and rank logic alone, on CPU ranks over gloo: every rank
    times a trivial host step, the max over ranks is taken, rank 0 prints a
    line marked as a dry run (no measurement: value is null)."""
    for _ in range(args.warmup):
        time.sleep(0.001)
    if dist is not None:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time.sleep(0.001)
    ms = (time.perf_counter() - t0) * 1e3 / args.steps
    ms = max_over_ranks([ms], dist, None)[0]
    if rank == 0:
        print(json.dumps({"dry_run": True, "metric": METRIC, "value": None,
                          "unit": UNIT, "n_gpus": world, "steps": args.steps,
                          "warmup": args.warmup, "ms_per_step_host": ms,
                          "ranks_seen": world}), flush=True)
    return 0


def _free_port() -> int:
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def spawn_ranks(n: int) -> int:
    """Re-launch this command as n ranks, one process per GPU (the same
    launch the multi-GPU driver uses), and return its exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1",
           "--master-port", str(_free_port()), os.path.abspath(__file__),
           *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kv8", choices=["kv8", "reference"])
    ap.add_argument("--workload", default="llama8b_b64_32k", choices=sorted(W.NAMED))
    ap.add_argument("--chunk", type=int, default=512,
                    help="chunk_tokens of the timed workload (0: the library's "
                         "suggestion for this device)")
    ap.add_argument("--kernel", type=int, default=0,
                    help="decode form: 0 auto, 1 CUDA-core, 2 mma.sync tensor-core, 3 tcgen05")
    ap.add_argument("--calls", type=int, default=50,
                    help="timed decode calls per workload in per_workload")
    ap.add_argument("--cpu-seqs", type=int, default=8)
    ap.add_argument("--ref-seqs", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-workload", action="store_true")
    ap.add_argument("--extend", action="store_true",
                    help="time extend (chunked-prefill) attention instead")
    ap.add_argument("--int4", action="store_true",
                    help="time the INT4 cache variant on --workload instead")
    ap.add_argument("--kivi", action="store_true",
                    help="time the KIVI cache variant on --workload instead")
    ap.add_argument("--dry-run-cpu", action="store_true",
                    help="rank/launch logic only, on CPU over gloo (no GPU work, "
                         "no measurement)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = _env_int("WORLD_SIZE", 1)
    rank = _env_int("RANK", 0)
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        return spawn_ranks(args.gpus)
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}",
              file=sys.stderr)
        return 2
    if args.impl == "reference":
        return run_reference(args, W.NAMED[args.workload](), rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        if args.dry_run_cpu:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        else:
            import torch
            torch.cuda.set_device(_env_int("LOCAL_RANK", 0))
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if args.dry_run_cpu:
            return run_dry_cpu(args, rank, world, dist)
        if args.extend:
            return run_extend(args, rank, world, dist)
        if args.int4:
            return run_int4(args, W.NAMED[args.workload](), rank, world, dist)
        if args.kivi:
            return run_kivi(args, W.NAMED[args.workload](), rank, world, dist)
        return run_kv8(args, W.NAMED[args.workload](), rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
