"""Benchmark: paged decode attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--kernel auto|simt|mma] [--partition P]

A step is one pass of the decode hot path over one batch: the new token of
every sequence is appended to the paged cache (kv_cache_append, at the slot of
its last position) and paged decode attention runs over every sequence's full
context (partition kernel + log-sum-exp reduce).  Default workload: the
Llama-2-13B-shaped layer (64 sequences, 40 heads MHA, head_dim 128, fp16 KV,
block 16, context lengths uniform in [128, 2048], shuffled pool 1.2x).

Metric: algorithmic bytes of the step (K and V of every context token, q and
out, table entries, lengths, the appended tokens' reads and writes) per second.
Inputs are larger than L2 (about 1.4 GB of K/V per step), so no flush runs
between steps.  Time is measured with CUDA events on the launching stream,
bracketed by a barrier and a synchronize, max over ranks.  One JSON line is
printed by rank 0.  For N > 1 every rank runs its own replica of the workload
(sequences are independent: weak scaling, no data-path collective).

--impl reference times the CPU oracle (float64, all host cores) on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import (CONFIGS, ELEM_BYTES, algorithmic_bytes, make_decode_inputs,  # noqa: E402
                       make_e4m3_pages)

METRIC = "paged decode attention KV-read GB/s (% of B200 HBM peak) and tokens/s"
FALLBACK_HBM_GBS = 6650.0
RATED_HBM_GBS = 8000.0      # B200's rated HBM3e bandwidth (the copy peak above is measured)


# --------------------------------------------------------------------------
# helpers

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(values, world: int, device: str = "cuda"):
    """Element-wise max of per-rank values over the process group (timings
    are reported as the slowest rank's)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            return json.load(open(p))
        except Exception:
            return None
    return None


def step_bytes(cfg, lens, window: int = 0, kv_dtype: str | None = None,
               per_page_scales: bool = False) -> int:
    """Decode algorithmic bytes + the append: read k, v of each new token,
    write them (as E4M3 codes with kv_dtype "e4m3"), read the slot."""
    e = ELEM_BYTES[cfg.dtype]
    ec = ELEM_BYTES[kv_dtype or cfg.dtype]
    append = len(lens) * (2 * cfg.num_kv_heads * cfg.head_dim * (e + ec) + 8)
    return algorithmic_bytes(cfg, lens, window, kv_dtype, per_page_scales) + append


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.idx = device_index
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


KERNEL_SOURCES = {
    "simt": ("decode_common.cuh", "decode_simt.cuh", "device_common.cuh"),
    "mma": ("decode_common.cuh", "decode_mma.cuh", "device_common.cuh"),
    "simt_e4m3": ("decode_common.cuh", "decode_simt.cuh", "device_common.cuh"),
    "mma_e4m3": ("decode_common.cuh", "decode_mma.cuh", "decode_mma_e4m3.cuh",
                 "device_common.cuh"),
}


SCHEDULE_NAMES = {"items": "work list, longest partition first",
                  "order": "longest sequence first", "none": "batch order"}


def kernel_source_digest(variant: str) -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_346_b200", "csrc")
    for f in KERNEL_SOURCES[variant]:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def resolve_variant(cfg, kernel: str, kv: str = "same") -> str:
    """The decode kernel the library's automatic choice takes for cfg."""
    if kv.startswith("e4m3"):
        if kernel == "mma" or (kernel == "auto" and cfg.group <= 16):
            return "mma_e4m3"
        return "simt_e4m3"
    if kernel != "auto":
        return kernel
    return "mma" if cfg.dtype != "f32" and 4 <= cfg.group <= 16 else "simt"


def recorded_traffic(workload: str, variant: str, partition: int | None = None,
                     kv: str = "same"):
    """DRAM bytes per decode call from a committed ncu summary, if it was
    taken on the current kernel sources (else None).  Summaries of runs with a
    scale per E4M3 page carry the suffix _page."""
    suffix = "_page" if kv == "e4m3-page" else ""
    p = os.path.join(ROOT, "profiles", f"decode_{variant}_{workload}{suffix}.md")
    if not os.path.exists(p):
        return None
    rec = {}
    for line in open(p):
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            rec[k.strip()] = v.strip().strip("`")
    if rec.get("kernel_sources_sha256_16") != kernel_source_digest(variant):
        return None
    if partition is not None and rec.get("partition_size") not in (None, str(partition)):
        return None
    try:
        return int(rec["dram_bytes_per_decode_call"])
    except (KeyError, ValueError):
        return None


# --------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline field)

def oracle_rate(inp, budget_s: float, seed: int = 0, pages=None, window: int = 0,
                per_page: bool = False):
    """Time the float64 oracle on whole sequences (all heads), in a seeded
    order, passing over the batch again until about budget_s of wall time;
    returns (bytes/s, seconds, sample description, threads).  pages: E4M3
    pages (workloads.QuantisedPages) to decode instead of inp's caches."""
    import oracle
    cfg = inp.cfg
    kvd = "e4m3" if pages is not None else None

    def run_rows(rows, threads):
        if pages is None:
            return oracle.paged_decode_inputs(inp, rows=rows, threads=threads, window=window)
        return oracle.paged_decode(inp.q, pages.k_cache, pages.v_cache, inp.block_tables,
                                   inp.context_lens, scale=cfg.scale, dtype=cfg.dtype,
                                   kv_dtype="e4m3", k_scale=pages.k_scale,
                                   v_scale=pages.v_scale, rows=rows, threads=threads,
                                   window=window)
    threads = oracle.max_threads()
    order = np.random.default_rng(seed).permutation(cfg.num_seqs)
    nseq, ntok, nbytes, t_total = 0, 0, 0, 0.0
    while True:
        for b in order:
            rows = np.array([[b, h] for h in range(cfg.num_q_heads)], dtype=np.int32)
            t0 = time.perf_counter()
            run_rows(rows, threads)
            t_total += time.perf_counter() - t0
            nseq += 1
            ntok += int(inp.context_lens[b])
            nbytes += algorithmic_bytes(cfg, inp.context_lens[[b]], window, kvd, per_page)
            if t_total >= budget_s:
                break
        if t_total >= budget_s:
            break
    desc = (f"{nseq} sequence decodes (all {cfg.num_q_heads} heads, {ntok} context tokens; "
            f"passes over the {cfg.num_seqs}-sequence batch of {cfg.name}"
            f"{', E4M3 pages' if pages is not None else ''})")
    return nbytes / t_total, t_total, desc, threads


def run_reference(args, cfg):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    inp = make_decode_inputs(cfg, seed=args.seed, shuffle=args.tables == "shuffled")
    import oracle
    e4m3 = args.kv in ("e4m3", "e4m3-page")
    per_page = args.kv == "e4m3-page"
    pages = make_e4m3_pages(inp, seed=args.seed, per_page=per_page) if e4m3 else None
    kvd = "e4m3" if e4m3 else None
    W = args.window
    threads = oracle.max_threads()

    def run_rows(rows):
        if pages is None:
            return oracle.paged_decode_inputs(inp, rows=rows, threads=threads, window=W)
        return oracle.paged_decode(inp.q, pages.k_cache, pages.v_cache, inp.block_tables,
                                   inp.context_lens, scale=cfg.scale, dtype=cfg.dtype,
                                   kv_dtype="e4m3", k_scale=pages.k_scale,
                                   v_scale=pages.v_scale, rows=rows, threads=threads, window=W)

    # calibrate on a few sequences, then size each step's sample so the whole
    # run stays within about --ref-budget seconds
    cal = np.arange(min(4, cfg.num_seqs))
    t0 = time.perf_counter()
    run_rows(np.array([[b, h] for b in cal for h in range(cfg.num_q_heads)], dtype=np.int32))
    rate = algorithmic_bytes(cfg, inp.context_lens[cal], W, kvd, per_page) / max(
        time.perf_counter() - t0, 1e-6)
    steps_total = args.steps + args.warmup
    budget = args.ref_budget / max(steps_total, 1)
    seq_bytes = algorithmic_bytes(cfg, inp.context_lens, W, kvd, per_page) / cfg.num_seqs
    nseq = int(max(1, min(cfg.num_seqs, math.floor(rate * budget / seq_bytes))))
    g = np.random.default_rng(args.seed)
    times = []
    nbytes = []
    for i in range(steps_total):
        seqs = g.choice(cfg.num_seqs, size=nseq, replace=False)
        rows = np.array([[b, h] for b in seqs for h in range(cfg.num_q_heads)], dtype=np.int32)
        t0 = time.perf_counter()
        run_rows(rows)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
            nbytes.append(algorithmic_bytes(cfg, inp.context_lens[seqs], W, kvd, per_page))
    value = sum(nbytes) / sum(times) / 1e9
    sample = (f"{nseq} of {cfg.num_seqs} sequences per step (all {cfg.num_q_heads} heads), "
              f"float64 C oracle, {threads} threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(times) / len(times), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfg, inp.context_lens, args.gpus, args.tables, W, args.kv),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------
# GPU arm

def workload_config(cfg, lens, world: int, tables: str, window: int, kv: str) -> dict:
    """The workload a line measures (the same dict on both arms)."""
    per_page = kv == "e4m3-page"
    kv_pages = (("e4m3 (per-page fp32 scales)" if per_page else "e4m3 (per-head fp32 scales)")
                if kv.startswith("e4m3") else cfg.dtype)
    kvd = "e4m3" if kv.startswith("e4m3") else None
    dec = algorithmic_bytes(cfg, lens, window, kvd, per_page)
    return {"workload": cfg.name, "global_batch": cfg.num_seqs * world,
            "seq_len": round(float(np.mean(lens)), 1), "num_q_heads": cfg.num_q_heads,
            "num_kv_heads": cfg.num_kv_heads, "head_dim": cfg.head_dim,
            "block_size": cfg.block_size, "block_tables": tables, "sliding_window": window,
            "kv_pages": kv_pages, "q_out": cfg.dtype, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (%.2f GB of K/V per step)" % (dec / 1e9)}


class Workload:
    """One decode workload on the device: seeded inputs, the step (append of
    each sequence's new token + decode) and its byte counts."""

    def __init__(self, args, cfg, kv: str, rank: int, partition: int, window: int):
        import torch

        import paged_kv_cache_346_b200 as pkv
        self.cfg, self.kv = cfg, kv
        self.kern = {"auto": pkv.PKV_KERNEL_AUTO, "simt": pkv.PKV_KERNEL_SIMT,
                     "mma": pkv.PKV_KERNEL_MMA}[args.kernel]
        inp = make_decode_inputs(cfg, seed=args.seed + rank, shuffle=args.tables == "shuffled")
        self.inp = inp
        self.e4m3 = e4m3 = kv in ("e4m3", "e4m3-page")
        self.per_page = per_page = kv == "e4m3-page"
        if e4m3 and cfg.dtype == "f32":
            raise SystemExit("E4M3 pages take fp16/bf16 q")

        def dev(a):
            if cfg.dtype == "bf16" and a.dtype == np.uint16:
                return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
            return torch.from_numpy(np.ascontiguousarray(a)).cuda()
        self.dev = dev

        self.pages = None
        if e4m3:
            self.pages = pages = make_e4m3_pages(inp, seed=args.seed + rank, per_page=per_page)
            self.q = dev(inp.q)
            self.kc = dev(pages.k_cache).view(torch.float8_e4m3fn)
            self.vc = dev(pages.v_cache).view(torch.float8_e4m3fn)
            self.ks, self.vs = dev(pages.k_scale), dev(pages.v_scale)
        else:
            self.q, self.kc, self.vc = dev(inp.q), dev(inp.k_cache), dev(inp.v_cache)
            self.ks = self.vs = None
        self.bt, self.cl = dev(inp.block_tables), dev(inp.context_lens)
        B, H, D, bs = cfg.num_seqs, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
        self.lens = lens = inp.context_lens.astype(np.int64)
        last = lens - 1
        slots_np = (inp.block_tables[np.arange(B), last // bs].astype(np.int64) * bs + last % bs)
        self.slots = dev(slots_np)
        # the new token of each sequence: the K/V already at its last position
        # (so every step rewrites identical bits and the workload stays fixed)
        # (with E4M3 pages: those values dequantised to q's type; re-quantising
        # them reaches a fixed point after the first step)
        sb_idx = torch.from_numpy(slots_np // bs).cuda()
        so_idx = torch.from_numpy(slots_np % bs).cuda()
        if e4m3:
            ksel = self.ks[sb_idx] if per_page else self.ks[None, :]   # [B or 1, Hkv]
            vsel = self.vs[sb_idx] if per_page else self.vs[None, :]
            self.knew = (self.kc.view(torch.uint8)[sb_idx, :, so_idx, :].view(
                torch.float8_e4m3fn).float() * ksel[:, :, None]).to(self.q.dtype).contiguous()
            self.vnew = (self.vc.view(torch.uint8)[sb_idx, :, so_idx, :].view(
                torch.float8_e4m3fn).float() * vsel[:, :, None]).to(self.q.dtype).contiguous()
        else:
            self.knew = self.kc.view(-1, H, bs, D)[sb_idx, :, so_idx, :].contiguous()
            self.vnew = self.vc.view(-1, H, bs, D)[sb_idx, :, so_idx, :].contiguous()
        self.out = torch.empty_like(self.q)
        self.mcl = mcl = inp.max_context_len
        self.W = W = window
        span = min(mcl, W + bs - 1) if W > 0 else mcl
        self.Pused = partition or pkv.pkv_decode_default_partition(B, H, span)
        # the schedule, from host lengths: a work list of (sequence, partition)
        # pairs longest first (cut with the resolved partition size), or the
        # sequences longest first over the partition grid, or batch order
        self.order = self.items = None
        if args.schedule == "items":
            self.items = dev(pkv.pkv_decode_schedule_items(inp.context_lens, bs, self.Pused, W))
            partition = self.Pused
        elif args.schedule == "order":
            self.order = dev(pkv.pkv_decode_schedule_order(inp.context_lens))
        self.P = P = partition
        ws_bytes = pkv.pkv_decode_workspace_size(B, cfg.num_q_heads, H, D, span, P)
        self.ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
        self.launches_per_step = 1 + 1 + (1 if math.ceil(span / self.Pused) > 1 else 0)
        kvd = "e4m3" if e4m3 else None
        self.step_bytes = step_bytes(cfg, lens, W, kvd, per_page)
        self.dec_bytes = algorithmic_bytes(cfg, lens, W, kvd, per_page)
        self.variant = resolve_variant(cfg, args.kernel, kv)
        self.pkv = pkv

    def decode(self, stream):
        pkv, c = self.pkv, self.cfg
        if self.e4m3:
            pkv.pkv_paged_attention_decode_e4m3(
                self.out, self.q, self.kc, self.vc, self.ks, self.vs, self.bt, self.cl, c.scale,
                c.block_size, self.mcl, partition_size=self.P, workspace=self.ws,
                seq_order=self.order, items=self.items, sliding_window=self.W, kernel=self.kern,
                stream=stream)
        else:
            pkv.pkv_paged_attention_decode(
                self.out, self.q, self.kc, self.vc, self.bt, self.cl, c.scale, c.block_size,
                self.mcl, partition_size=self.P, workspace=self.ws, seq_order=self.order,
                items=self.items, sliding_window=self.W, kernel=self.kern, stream=stream)

    def append(self, stream):
        if self.e4m3:
            self.pkv.pkv_kv_cache_append_e4m3(self.kc, self.vc, self.knew, self.vnew, self.ks,
                                              self.vs, self.slots, stream=stream)
        else:
            self.pkv.pkv_kv_cache_append(self.kc, self.vc, self.knew, self.vnew, self.slots,
                                         stream=stream)


def time_blocks(w: Workload, steps: int, warmup: int, min_device_s: float, barrier, local,
                max_blocks: int = 400):
    """Warm up, then time blocks of exactly `steps` steps (append + decode;
    each block bracketed by a barrier and a synchronize, CUDA events on the
    launching stream at the block's ends only, so nothing sits between a
    step's two launches) until at least min_device_s / 2 of device time (and
    3 blocks); then the same number of blocks of `steps` decode calls alone
    with events around every call, for the decode's own time.  NVML clocks
    are sampled throughout.  -> (block ms list, mean decode ms per block
    list, clocks)"""
    import torch
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        w.append(stream)
        w.decode(stream)
    torch.cuda.synchronize()
    ev_dec = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    blocks, dec = [], []
    with ClockSampler(local) as clocks:
        while True:
            barrier()
            torch.cuda.synchronize()
            t_start.record(stream)
            for i in range(steps):
                w.append(stream)
                w.decode(stream)
            t_end.record(stream)
            torch.cuda.synchronize()
            barrier()
            blocks.append(t_start.elapsed_time(t_end))
            if (len(blocks) >= 3 and sum(blocks) * 1e-3 >= min_device_s / 2) or \
                    len(blocks) >= max_blocks:
                break
        for _ in range(len(blocks)):
            barrier()
            torch.cuda.synchronize()
            for i in range(steps):
                ev_dec[i][0].record(stream)
                w.decode(stream)
                ev_dec[i][1].record(stream)
            torch.cuda.synchronize()
            barrier()
            dec.append(statistics.mean(a.elapsed_time(b) for a, b in ev_dec))
    flags = w.pkv.pkv_device_status(clear=True)
    if flags:
        raise SystemExit(f"device status flags {flags:#x} during the benchmark")
    return blocks, dec, clocks.summary()


def median_block(blocks, dec):
    """The median step block and the median decode time."""
    return statistics.median(blocks), statistics.median(dec)


def hbm_peak():
    peaks = measured_peaks()
    if peaks and "hbm_gbs" in peaks:
        return float(peaks["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    return FALLBACK_HBM_GBS, "fallback"


def roofline_of(w: Workload, dec_ms: float, args) -> dict:
    peak, src = hbm_peak()
    achieved = w.dec_bytes / (dec_ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "paged decode (partition kernel + LSE reduce)",
            "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "peak_source": src,
            "frac_of_rated_8tbs": round(achieved / RATED_HBM_GBS, 4),
            "decode_ms": round(dec_ms, 5), "bytes_per_launch": int(w.dec_bytes),
            "variant": w.variant,
            "traffic": recorded_traffic(w.cfg.name, w.variant, w.Pused, w.kv)}


def run_ours(args, cfg):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    w = Workload(args, cfg, args.kv, rank, args.partition, args.window)
    pkv = w.pkv
    B, H, D, bs = cfg.num_seqs, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    stream = torch.cuda.current_stream()

    # ---- device-resident timing: blocks of --steps steps, the median block
    blocks, decs, clocks = time_blocks(w, args.steps, args.warmup, args.min_time, barrier, local)
    ms, dec_ms = median_block(blocks, decs)

    # ---- end to end through the public API: every step copies its inputs
    # (q, the new tokens' K/V, slots, tables, lengths, schedule) from
    # pinned host memory and reads its output back.  The inputs of a step are
    # packed in one pinned buffer (one upload), and the C ABI is called with
    # argument lists prepared once, so the host keeps ahead of the GPU.  Two
    # input and two output buffers and two copy streams let step i+1's upload
    # and step i-1's readback run under step i's kernels; events order every
    # reuse.
    q, kc, vc, out, ws = w.q, w.kc, w.vc, w.out, w.ws
    fields = [("q", q), ("knew", w.knew), ("vnew", w.vnew), ("slots", w.slots), ("bt", w.bt),
              ("cl", w.cl)]
    if w.order is not None:
        fields.append(("order", w.order))
    if w.items is not None:
        fields.append(("items", w.items))
    offs, total = {}, 0
    for name, t in fields:
        offs[name] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_in = torch.empty(total, dtype=torch.uint8).pin_memory()
    for name, t in fields:
        nb_ = t.numel() * t.element_size()
        h_in[offs[name]:offs[name] + nb_].copy_(t.reshape(-1).view(torch.uint8).cpu())
    d_in = [torch.empty(total, dtype=torch.uint8, device="cuda") for _ in range(2)]
    d_out = [torch.empty_like(out) for _ in range(2)]
    h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for _, t in fields)
    d2h = h_out[0].numel() * h_out[0].element_size()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_done + ev_out:
        e.record(stream)
    c_stream = ctypes.c_void_p(stream.cuda_stream)
    dt_code = pkv.torch_dtype_code(q.dtype)
    N_blocks = kc.shape[0]
    P, W, mcl = w.P, w.W, w.mcl
    calls = []
    for j in range(2):
        ptr = {name: ctypes.c_void_p(d_in[j].data_ptr() + offs[name]) for name, _ in fields}
        kp, vp = ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(vc.data_ptr())
        if w.e4m3:
            ksp, vsp = ctypes.c_void_p(w.ks.data_ptr()), ctypes.c_void_p(w.vs.data_ptr())
            spb = 1 if w.per_page else 0
            append_args = (kp, vp, ptr["knew"], ptr["vnew"], ksp, vsp, spb, ptr["slots"], B, H, D,
                           bs, N_blocks, dt_code, c_stream)
            sched = ((ptr["items"], w.items.shape[0]) if w.items is not None
                     else (ptr.get("order"),))
            decode_args = (ctypes.c_void_p(d_out[j].data_ptr()), ptr["q"], kp, vp, ksp, vsp,
                           spb, ptr["bt"], ptr["cl"], *sched, B, cfg.num_q_heads,
                           H, D, bs, w.bt.shape[1], N_blocks, mcl, cfg.scale, W, dt_code, P,
                           ctypes.c_void_p(ws.data_ptr()), ws.numel(), w.kern, c_stream)
        else:
            append_args = (kp, vp, ptr["knew"], ptr["vnew"], ptr["slots"], B, H, D, bs,
                           N_blocks, dt_code, c_stream)
            sched = ((ptr["items"], w.items.shape[0]) if w.items is not None
                     else (ptr.get("order"),))
            decode_args = (ctypes.c_void_p(d_out[j].data_ptr()), ptr["q"], kp, vp, ptr["bt"],
                           ptr["cl"], *sched, B, cfg.num_q_heads, H, D, bs,
                           w.bt.shape[1], N_blocks, mcl, cfg.scale, W, dt_code, P,
                           ctypes.c_void_p(ws.data_ptr()), ws.numel(), w.kern, c_stream)
        calls.append((append_args, decode_args))
    c_append = pkv.lib.pkv_kv_cache_append_e4m3 if w.e4m3 else pkv.lib.pkv_kv_cache_append
    if w.items is not None:
        c_decode = (pkv.lib.pkv_paged_attention_decode_e4m3_items if w.e4m3
                    else pkv.lib.pkv_paged_attention_decode_items)
    else:
        c_decode = (pkv.lib.pkv_paged_attention_decode_e4m3 if w.e4m3
                    else pkv.lib.pkv_paged_attention_decode)

    def e2e_step(i):
        j = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_done[j])          # the kernels of step i-2 are done with d_in[j]
            d_in[j].copy_(h_in, non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        stream.wait_event(ev_out[j])             # d_out[j] of step i-2 has been read back
        a_args, d_args = calls[j]
        if c_append(*a_args) or c_decode(*d_args):
            raise SystemExit("C-ABI call failed in the e2e loop")
        ev_done[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[j])
            h_out[j].copy_(d_out[j], non_blocking=True)
            ev_out[j].record(s_out)

    e2e_steps = max(4, min(args.steps * 20, 1000))
    for i in range(max(args.warmup, 3)):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_stream(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_event(ev_out[(e2e_steps - 1) % 2])
    stream.wait_event(ev_out[(e2e_steps - 2) % 2])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    assert torch.equal(h_out[0], out.cpu()) and torch.equal(h_out[1], out.cpu())
    del d_in, d_out, h_in, h_out

    # ---- the other workloads the targets name, measured the same way
    also = []
    for spec in ([] if args.also == "none" else args.also.split(",")):
        name, _, kv = spec.partition(":")
        kv = kv or "same"
        if name == cfg.name and kv == args.kv:
            continue
        w2 = Workload(args, CONFIGS[name], kv, rank, CONFIGS[name].partition_size, 0)
        b2, d2, c2 = time_blocks(w2, args.steps, args.warmup, args.min_time, barrier, local)
        m2, dm2 = median_block(b2, d2)
        m2, dm2 = max_over_ranks([m2, dm2], world)
        also.append((w2, b2, m2, dm2, c2))
        del w2

    # ---- max over ranks
    ms, dec_ms, e2e_ms = max_over_ranks([ms, dec_ms, e2e_ms], world)

    if rank == 0:
        per_step_ms = ms / args.steps
        value = world * w.step_bytes / (per_step_ms * 1e-3) / 1e9
        peak, _ = hbm_peak()
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per_step_ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3" if w.e4m3 else cfg.dtype, "data": "synthetic",
            "config": workload_config(cfg, w.lens, world, args.tables, w.W, args.kv),
            "impl_config": {"partition_size": w.Pused, "kernel": args.kernel,
                            "schedule": SCHEDULE_NAMES[args.schedule]},
            "timing": {"blocks": len(blocks), "steps_per_block": args.steps,
                       "block_ms_median": round(ms, 4), "block_ms_min": round(min(blocks), 4),
                       "block_ms_max": round(max(blocks), 4),
                       "device_s_timed": round(sum(blocks) * 1e-3, 3),
                       "note": "median of the timed blocks; each block is --steps steps "
                               "bracketed by a barrier and a synchronize; the decode time "
                               "(roofline) comes from as many blocks of decode calls alone"},
            "tokens_per_s": round(world * B / (per_step_ms * 1e-3), 1),
            "pct_of_hbm_peak": round(100 * value / world / peak, 2),
            "pct_of_rated_hbm_8tbs": round(100 * value / world / RATED_HBM_GBS, 2),
            "e2e": {"value": round(world * w.step_bytes / (e2e_ms * 1e-3) / 1e9, 2),
                    "unit": "GB/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "ms_per_step": round(e2e_ms, 4)},
            "gpu_launches": w.launches_per_step * args.steps,
            "roofline": roofline_of(w, dec_ms, args),
            "clocks": clocks,
        }
        if also:
            line["also"] = []
            for w2, b2, m2, dm2, c2 in also:
                st = m2 / args.steps
                v2 = world * w2.step_bytes / (st * 1e-3) / 1e9
                line["also"].append({
                    "config": workload_config(w2.cfg, w2.lens, world, args.tables, 0, w2.kv),
                    "impl_config": {"partition_size": w2.Pused, "kernel": args.kernel,
                                    "schedule": SCHEDULE_NAMES[args.schedule]},
                    "value": round(v2, 2), "unit": "GB/s", "ms_per_step": round(st, 5),
                    "tokens_per_s": round(world * w2.cfg.num_seqs / (st * 1e-3), 1),
                    "pct_of_hbm_peak": round(100 * v2 / world / peak, 2),
                    "blocks": len(b2), "device_s_timed": round(sum(b2) * 1e-3, 3),
                    "roofline": roofline_of(w2, dm2, args), "clocks": c2})
        if world == 1 and not args.no_cpu_baseline:
            rate, secs, desc, threads = oracle_rate(w.inp, args.cpu_budget, seed=args.seed,
                                                    pages=w.pages, window=w.W,
                                                    per_page=w.per_page)
            line["cpu_baseline"] = {"value": round(rate / 1e9, 4), "unit": "GB/s",
                                    "cores": threads, "kind": "oracle",
                                    "sample": desc + f", {secs:.1f} s"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_cow(args):
    """Parallel sampling with copy-on-write prefix sharing: 32 prompts x 8
    samples share 1024 + r tokens (r in [1, 15], so the last shared block is
    partly filled).  Two timed phases, each replaying the same device work:
    (i) the fork step -- every sample appends its first token, the allocator
    hands out 7 block copies per prompt, and the step runs copy_blocks,
    kv_cache_append and the decode; (ii) a steady step once every sample has
    a private tail of U[1, 512] tokens -- append + decode, no copies.  The
    decode is the shared-prefix decode (each prompt's shared blocks read once
    for its samples); the regular decode of the same step is timed beside it
    ("regular_decode")."""
    import torch

    import paged_kv_cache_346_b200 as pkv
    from workloads import COW_SAMPLING, draw_cow_recipe

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    c = COW_SAMPLING
    rec = draw_cow_recipe(seed=args.seed)
    P, S = rec.num_prompts, rec.samples
    B, H, D, bs = P * S, c["num_kv_heads"], c["head_dim"], c["block_size"]
    e = 2
    N = sum(-(-int(L) // bs) for L in rec.shared_lens) + B * (3 + -(-c["tail_hi"] // bs))
    alloc = pkv.BlockAllocator(N, bs)
    for p in range(P):
        assert alloc.add_seq(1_000_000 + p, int(rec.shared_lens[p])) == 0
        for s_ in range(S):
            assert alloc.fork(1_000_000 + p, p * S + s_) == 0
        assert alloc.free_seq(1_000_000 + p) == 0
    g = torch.Generator(device="cuda").manual_seed(args.seed)
    kc = torch.randn((N, H, bs, D), generator=g, device="cuda", dtype=torch.float32).half()
    vc = torch.randn((N, H, bs, D), generator=g, device="cuda", dtype=torch.float32).half()
    seqs = np.arange(B)
    scale = 1.0 / math.sqrt(D)
    stream = torch.cuda.current_stream()

    def phase(pairs_np, slots_np, tables_np, lens_np):
        q = torch.randn((B, H, D), generator=g, device="cuda", dtype=torch.float32).half()
        knew = torch.randn((B, H, D), generator=g, device="cuda", dtype=torch.float32).half()
        vnew = torch.randn((B, H, D), generator=g, device="cuda", dtype=torch.float32).half()
        pairs = torch.from_numpy(pairs_np).cuda()
        slots = torch.from_numpy(slots_np).cuda()
        tables = torch.from_numpy(tables_np).cuda()
        lens = torch.from_numpy(lens_np).cuda()
        out = torch.empty_like(q)
        L = int(lens_np.max())
        ws = torch.empty(max(16, pkv.pkv_decode_workspace_size(B, H, H, D, L)),
                         dtype=torch.uint8, device="cuda")
        # the shared prompt blocks of each prompt's samples, found from the
        # host tables (the allocator's), for the shared-prefix decode
        spl_np, mem_np = pkv.pkv_decode_prefix_groups(tables_np, lens_np, bs)
        spl, mem = torch.from_numpy(spl_np).cuda(), torch.from_numpy(mem_np).cuda()
        mpl = int(spl_np.max())
        ws_g = torch.empty(max(16, pkv.pkv_decode_prefix_groups_workspace_size(B, H, H, D, L,
                                                                              mpl)),
                           dtype=torch.uint8, device="cuda")
        npairs = len(pairs_np)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(3)]

        def decode(grouped):
            if grouped:
                pkv.pkv_paged_attention_decode_prefix_groups(out, q, kc, vc, tables, lens, spl,
                                                             mem, scale, bs, L, mpl,
                                                             workspace=ws_g, stream=stream)
            else:
                pkv.pkv_paged_attention_decode(out, q, kc, vc, tables, lens, scale, bs, L,
                                               workspace=ws, stream=stream)

        def step(grouped, timed=False):
            if timed:
                ev[0][0].record(stream)
            if npairs:
                pkv.pkv_copy_blocks(kc, vc, pairs, stream=stream)
            if timed:
                ev[0][1].record(stream)
                ev[1][0].record(stream)
            pkv.pkv_kv_cache_append(kc, vc, knew, vnew, slots, stream=stream)
            if timed:
                ev[1][1].record(stream)
                ev[2][0].record(stream)
            decode(grouped)
            if timed:
                ev[2][1].record(stream)

        def timed_steps(grouped):
            for _ in range(args.warmup):
                step(grouped)
            torch.cuda.synchronize()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record(stream)
            for _ in range(args.steps):
                step(grouped, timed=True)
            t1.record(stream)
            torch.cuda.synchronize()
            # per-kernel times of the last step (events were re-recorded each step)
            return t0.elapsed_time(t1) / args.steps, [a.elapsed_time(b) for a, b in ev]

        ms_r, parts_r = timed_steps(False)
        out_r = out.clone()
        ms, parts = timed_steps(True)
        # the two decodes differ only in summation order
        diff = float((out.float() - out_r.float()).abs().max())
        # bytes: logical = every sequence's K/V as read; unique = distinct
        # physical (block, slot) entries the decode reads
        kv_tok = 2 * H * D * e
        logical = int(lens_np.astype(np.int64).sum()) * kv_tok
        filled = {}
        for i in range(B):
            Li = int(lens_np[i])
            for j in range(-(-Li // bs)):
                blk = int(tables_np[i, j])
                filled[blk] = max(filled.get(blk, 0), min(bs, Li - j * bs))
        unique = sum(filled.values()) * kv_tok
        qo = 2 * B * H * D * e
        tab = int(sum(-(-int(x) // bs) for x in lens_np)) * 4 + 4 * B
        copy = npairs * 4 * H * bs * D * e
        append = B * (4 * H * D * e + 8)
        return {
            "ms_per_step": round(ms, 5),
            "copy_pairs": npairs,
            "prefix_groups": int(len(mem_np)),
            "shared_prefix_tokens_mean": round(float(spl_np.mean()), 1),
            "kernel_ms_last_step": {"copy_blocks": round(parts[0], 5),
                                    "kv_append": round(parts[1], 5),
                                    "decode": round(parts[2], 5)},
            "regular_decode": {"ms_per_step": round(ms_r, 5), "decode_ms": round(parts_r[2], 5),
                               "decode_unique_GBps": round((unique + qo + tab) /
                                                           (parts_r[2] * 1e-3) / 1e9, 1)},
            "max_abs_diff_vs_regular": diff,
            "logical_bytes": logical + qo + tab + copy + append,
            "unique_bytes": unique + qo + tab + copy + append,
            "effective_GBps": round((logical + qo + tab + copy + append) / (ms * 1e-3) / 1e9, 1),
            "unique_GBps": round((unique + qo + tab + copy + append) / (ms * 1e-3) / 1e9, 1),
            "decode_unique_GBps": round((unique + qo + tab) / (parts[2] * 1e-3) / 1e9, 1),
            "mean_context": round(float(lens_np.mean()), 1),
        }

    # (i) fork step
    st, slots, pairs, done = alloc.append_slots(seqs)
    assert st == 0 and done == B
    tables, lens = alloc.build_block_tables(seqs, N)
    maxb = int(max(-(-int(x) // bs) for x in lens))
    fork = phase(pairs, slots, np.ascontiguousarray(tables[:, :maxb]), lens)
    # (ii) grow private tails on the host, then one steady step
    for i in range(B):
        for _ in range(int(rec.tail_lens[i]) - 1):
            r = alloc.append_slot(int(seqs[i]))
            assert r[0] == 0 and r[2] < 0
    st, slots, pairs, done = alloc.append_slots(seqs)
    assert st == 0 and len(pairs) == 0
    tables, lens = alloc.build_block_tables(seqs, N)
    maxb = int(max(-(-int(x) // bs) for x in lens))
    steady = phase(pairs, slots, np.ascontiguousarray(tables[:, :maxb]), lens)
    stats = alloc.stats()
    flags = pkv.pkv_device_status(clear=True)
    if flags:
        raise SystemExit(f"device status flags {flags:#x}")
    if rank == 0:
        peaks = measured_peaks() or {}
        line = {
            "metric": METRIC + " (copy-on-write sampling)", "value": steady["effective_GBps"],
            "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic",
            "config": {"workload": "cow_sampling", "prompts": P, "samples": S,
                       "shared_tokens_mean": float(rec.shared_lens.mean()),
                       "heads": H, "head_dim": D, "block_size": bs},
            "fork_step": fork, "steady_step": steady,
            "allocator": stats, "hbm_peak_GBps": peaks.get("hbm_gbs"),
        }
        print(json.dumps(line), flush=True)
    return 0


def run_swap(args):
    """Swapping: whole pages of the Llama-2-13B-shaped layer (40 heads x 16
    tokens x 128 dims fp16 = 160 KB per page, K and V) moved between the
    device pool and a page-locked host pool by pkv_swap_blocks, in a seeded
    random scatter, both directions; next to it the host link's rate for one
    contiguous copy of the same bytes (torch copy_, the copy engines)."""
    import torch

    import paged_kv_cache_346_b200 as pkv

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    H, bs, D = 40, 16, 128
    n = 2048                                       # pages per direction (K and V each)
    N_dev, N_host = 3 * n, 2 * n
    g = torch.Generator(device="cuda").manual_seed(args.seed)
    dk = torch.randn((N_dev, H, bs, D), generator=g, device="cuda").half()
    dv = torch.randn((N_dev, H, bs, D), generator=g, device="cuda").half()
    hk = torch.empty((N_host, H, bs, D), dtype=torch.float16).pin_memory()
    hv = torch.empty((N_host, H, bs, D), dtype=torch.float16).pin_memory()
    rng_ = np.random.default_rng(args.seed)
    out_pairs = np.stack([rng_.choice(N_dev, n, replace=False),
                          rng_.choice(N_host, n, replace=False)], 1).astype(np.int32)
    in_pairs = np.stack([out_pairs[:, 1], rng_.choice(N_dev, n, replace=False)], 1).astype(np.int32)
    p_out, p_in = torch.from_numpy(out_pairs).cuda(), torch.from_numpy(in_pairs).cuda()
    stream = torch.cuda.current_stream()
    page = H * bs * D * 2
    nbytes = 2 * n * page                          # K and V pages moved per call

    def timed(fn, reps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    reps = max(3, min(args.steps, 20))
    t_out = timed(lambda: pkv.pkv_swap_blocks(hk, hv, dk, dv, p_out, stream=stream), reps)
    t_in = timed(lambda: pkv.pkv_swap_blocks(dk, dv, hk, hv, p_in, stream=stream), reps)
    flat_h = hk.view(-1)[: n * page // 2]
    flat_d = dk.view(-1)[: n * page // 2]
    t_d2h = timed(lambda: flat_h.copy_(flat_d, non_blocking=True), reps)
    t_h2d = timed(lambda: flat_d.copy_(flat_h, non_blocking=True), reps)
    flags = pkv.pkv_device_status(clear=True)
    if rank == 0:
        line = {
            "metric": "swap GB/s (pages between the device pool and page-locked host memory)",
            "value": round(nbytes / (t_in * 1e-3) / 1e9, 2), "unit": "GB/s",
            "n_gpus": 1, "steps": reps, "warmup": args.warmup, "higher_is_better": True,
            "data": "synthetic", "dtype": "f16",
            "config": {"workload": "swap", "pages": n, "page_bytes": page,
                       "bytes_per_call": nbytes},
            "swap_in_GBps": round(nbytes / (t_in * 1e-3) / 1e9, 2),
            "swap_out_GBps": round(nbytes / (t_out * 1e-3) / 1e9, 2),
            "swap_in_ms": round(t_in, 4), "swap_out_ms": round(t_out, 4),
            "contiguous_h2d_GBps": round((n * page) / (t_h2d * 1e-3) / 1e9, 2),
            "contiguous_d2h_GBps": round((n * page) / (t_d2h * 1e-3) / 1e9, 2),
            "device_status": flags,
        }
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama2_13b_layer",
                    choices=sorted(CONFIGS) + ["cow_sampling", "swap"])
    ap.add_argument("--kernel", choices=["auto", "simt", "mma"], default="auto")
    ap.add_argument("--partition", type=int, default=None,
                    help="tokens per partition (default: automatic under --window, else the "
                         "workload's, else automatic)")
    ap.add_argument("--seed", type=int, default=2)
    ap.add_argument("--window", type=int, default=0,
                    help="sliding window in tokens (0: attend to the whole context)")
    ap.add_argument("--kv", choices=["same", "e4m3", "e4m3-page"], default="same",
                    help="page element type: the workload's, or FP8 E4M3 codes with "
                         "per-head (e4m3) or per-page (e4m3-page) scales")
    ap.add_argument("--tables", choices=["shuffled", "identity"], default="shuffled",
                    help="physical block ids: a seeded permutation of the pool, or the "
                         "identity (each sequence's pages contiguous in memory)")
    ap.add_argument("--schedule", choices=["items", "order", "none"], default="items",
                    help="items: a work list of (sequence, partition) pairs, longest "
                         "partition first; order: sequences longest first over the partition "
                         "grid; none: batch order")
    ap.add_argument("--no-order", dest="schedule", action="store_const", const="none",
                    help="the same as --schedule none")
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of oracle work for the cpu_baseline field")
    ap.add_argument("--ref-budget", type=float, default=90.0,
                    help="seconds of oracle work for --impl reference")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--min-time", type=float, default=0.5,
                    help="time blocks of --steps steps until at least this many seconds of "
                         "device time (and 3 blocks); the median block is reported")
    ap.add_argument("--also", default="gqa_bs16,gqa_bs32,gqa_bs16:e4m3,llama2_13b_layer:e4m3",
                    help="further workloads[:kv] measured the same way and reported under "
                         "\"also\" (none: only the main one)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps
    if args.workload == "cow_sampling":
        return run_cow(args)
    if args.workload == "swap":
        return run_swap(args)
    cfg = CONFIGS[args.workload]
    if args.partition is None:
        # a workload's partition size is set for its whole contexts; behind a
        # window the span is far shorter, so the library chooses
        args.partition = 0 if args.window else cfg.partition_size
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
