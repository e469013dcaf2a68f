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


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_int8_kv_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, fn), "rb") as f:
                h.update(fn.encode())
                h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per decode launch from a committed ncu capture, if it was
    taken on the current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    rec = d.get(workload)
    if not rec or rec.get("source_hash") != kernel_source_hash():
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
def oracle_sample_seconds(w: W.Workload, seqs) -> tuple[float, str]:
    """Time the oracle's decode step (append of the new token + attention
    for every query head) on sequences ``seqs``; cache build excluded."""
    import oracle
    total = 0.0
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
        table = np.arange(nblk, dtype=np.int32)[None, :]
        t0 = time.perf_counter()
        oracle.quantize_append(k[-1:], slots[-1:], kc, ks)
        oracle.quantize_append(v[-1:], slots[-1:], vc, vs)
        oracle.decode_attention(w.q()[b:b + 1], kc, vc, ks, vs, table,
                                w.context_lens[b:b + 1])
        total += time.perf_counter() - t0
    desc = (f"{len(seqs)} of {w.batch} sequences of {w.name}: append 1 token "
            f"+ attention for all {w.num_q_heads} query heads over "
            f"{int(w.context_lens[list(seqs)].sum())} tokens (fp64, 1 thread)")
    return total, desc


def run_reference(args, w: W.Workload, rank: int):
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    nseq = max(1, args.ref_seqs)
    seqs = list(range(nseq))
    for _ in range(args.warmup):
        oracle_sample_seconds(w, seqs[:1])
    times = []
    desc = ""
    for i in range(args.steps):
        s, desc = oracle_sample_seconds(w, [seqs[i % nseq]])
        times.append(s)
    sec = sum(times) / len(times)
    value = 1.0 / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1,
                         "kind": "oracle",
                         "sample": "per step: " + desc.replace("1 of", "1 of")},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def bench_config(w: W.Workload, args) -> dict:
    return {"workload": w.name, "batch": w.batch,
            "context_lens": (int(w.context_lens.min()), int(w.context_lens.max())),
            "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "block_size": w.block_size,
            "chunk_tokens": args.chunk, "num_blocks": w.num_blocks,
            "parallelism": f"replica x{args.gpus} (sequences independent)",
            "l2": "no flush: the cache read each step is larger than L2"
                  if algorithmic_bytes(w)["total"] > 126e6 * 4 else
                  "L2 flushed between steps"}


# -------------------------------------------------------------- GPU bench
def run_kv8(args, w: W.Workload, rank: int, world: int, dist):
    import torch
    import paged_int8_kv_b200 as pk
    from paged_int8_kv_b200.runtime import PagedKV8Cache, fill_from_host

    dev = torch.device("cuda", _env_int("LOCAL_RANK", 0))
    torch.cuda.set_device(dev)
    pk.kv8_set_decode_kernel(args.kernel)
    stream = torch.cuda.current_stream()

    cache = PagedKV8Cache(w.num_blocks, w.num_kv_heads, device=dev)
    fill_from_host(cache, w.fill_segments())
    kn, vn, sl = w.step_tokens()
    k_new = torch.from_numpy(kn).view(torch.bfloat16).to(dev)
    v_new = torch.from_numpy(vn).view(torch.bfloat16).to(dev)
    slots = torch.from_numpy(sl).to(dev)
    q = torch.from_numpy(w.q()).view(torch.bfloat16).to(dev)
    bt = torch.from_numpy(w.block_tables).to(dev)
    cl = torch.from_numpy(w.context_lens).to(dev)
    out = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    maxlen = w.max_context_len
    ws = cache.workspace(w.batch, w.num_q_heads, maxlen, args.chunk)
    flush = None
    ab = algorithmic_bytes(w)
    if ab["total"] <= 4 * 126e6:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    # per step: the quantize-append kernel and the decode kernel (a split
    # launch also enqueues a small memset of its merge tickets)
    launches_per_step = 2
    memsets_per_step = 1 if ws is not None else 0

    def step():
        cache.append(k_new, v_new, slots)
        pk.kv8_paged_decode_attention(q, cache.k_cache, cache.v_cache,
                                      cache.k_scales, cache.v_scales, bt, cl,
                                      out, maxlen, chunk_tokens=args.chunk,
                                      workspace=ws)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
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
            step()
        torch.cuda.synchronize()
    barrier()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        cache.append(k_new, v_new, slots)
        dec[i][0].record(stream)
        pk.kv8_paged_decode_attention(q, cache.k_cache, cache.v_cache,
                                      cache.k_scales, cache.v_scales, bt, cl,
                                      out, maxlen, chunk_tokens=args.chunk,
                                      workspace=ws)
        dec[i][1].record(stream)
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    dec_ms = [a.elapsed_time(b) for a, b in dec]
    ms = sum(step_ms) / len(step_ms)
    if flush is None:
        ms = t_start.elapsed_time(t_end) / args.steps
    dms = sum(dec_ms) / len(dec_ms)

    # ---- end to end through the public API: host buffers in, result out
    pin = lambda a: torch.from_numpy(a).pin_memory()  # noqa: E731
    h_k, h_v, h_s = pin(kn), pin(vn), pin(sl)
    h_q, h_bt, h_cl = pin(w.q()), pin(w.block_tables), pin(w.context_lens)
    h_out = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (h_k, h_v, h_s, h_q, h_bt, h_cl))
    d2h = h_out.numel() * h_out.element_size()
    d_k, d_v, d_s = torch.empty_like(k_new), torch.empty_like(v_new), torch.empty_like(slots)
    d_q, d_bt, d_cl = torch.empty_like(q), torch.empty_like(bt), torch.empty_like(cl)

    def e2e_step():
        d_k.view(torch.int16).copy_(h_k.view(torch.int16), non_blocking=True)
        d_v.view(torch.int16).copy_(h_v.view(torch.int16), non_blocking=True)
        d_s.copy_(h_s, non_blocking=True)
        d_q.view(torch.int16).copy_(h_q.view(torch.int16), non_blocking=True)
        d_bt.copy_(h_bt, non_blocking=True)
        d_cl.copy_(h_cl, non_blocking=True)
        cache.append(d_k, d_v, d_s)
        pk.kv8_paged_decode_attention(d_q, cache.k_cache, cache.v_cache,
                                      cache.k_scales, cache.v_scales, d_bt,
                                      d_cl, out, maxlen, chunk_tokens=args.chunk,
                                      workspace=ws)
        h_out.copy_(out, non_blocking=True)

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
            flush.fill_(1)
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.steps
    barrier()
    e2e_clocks = e2e_sampler.stop()

    # ---- max over ranks
    ms, dms, e2e_ms = max_over_ranks([ms, dms, e2e_ms], dist, dev)

    status = pk.kv8_read_device_status(clear=True)
    if rank != 0:
        return 0

    tokens = w.batch * world
    value = whole_job_rate(w.batch, world, ms)
    peak, peak_kind = measured_peaks()
    achieved = ab["total"] / (dms * 1e-3) / 1e9
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        seqs = list(range(min(args.cpu_seqs, w.batch)))
        sec, desc = oracle_sample_seconds(w, seqs)
        cpu = {"value": len(seqs) / sec, "unit": UNIT, "cores": 1,
               "kind": "oracle", "sample": desc}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "kv_dtype": "int8", "out_dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q/K/V, shuffled blocks)",
        "config": bench_config(w, args),
        "hbm_gbs": achieved,
        **({"hbm_gbs_unique_bytes": (uniq + ab["total"] - ab["kv"]) / (dms * 1e-3) / 1e9,
            "unique_bytes": uniq + ab["total"] - ab["kv"]}
           if (uniq := unique_kv_bytes(w)) < ab["kv"] else {}),
        "hbm_frac_of_measured": achieved / peak,
        "hbm_frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
        "decode_us": dms * 1e3,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                                    if peak_kind == "measured" else "fallback 6650 GB/s",
                     "kernel": "decode_kernel (split-K pages + fused chunk merge), "
                               "timed as the kv8_paged_decode_attention call",
                     "algorithmic_bytes": ab["total"],
                     "traffic": recorded_traffic(w.name)},
        "e2e": {"value": whole_job_rate(w.batch, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms, "clocks": e2e_clocks},
        "gpu_launches": launches_per_step * args.steps,
        "memsets": memsets_per_step * args.steps,
        "clocks": clocks,
        "device_status": status,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kv8", choices=["kv8", "reference"])
    ap.add_argument("--workload", default="llama8b_b64_32k", choices=sorted(W.NAMED))
    ap.add_argument("--chunk", type=int, default=512)
    ap.add_argument("--kernel", type=int, default=0, help="0 auto, 1 CUDA-core, 2 mma.sync tensor-core, 3 tcgen05")
    ap.add_argument("--cpu-seqs", type=int, default=4)
    ap.add_argument("--ref-seqs", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = W.NAMED[args.workload]()

    world = _env_int("WORLD_SIZE", 1)
    rank = _env_int("RANK", 0)
    if args.impl == "reference":
        return run_reference(args, w, rank)
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(_env_int("LOCAL_RANK", 0))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        return run_kv8(args, w, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
