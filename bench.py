"""Benchmark: one decode step of the paged KV-cache hot path per iteration.

A step = (copy-on-write block copies when the workload has them) + the cache write
of the step's new tokens + paged decode attention, on seeded synthetic inputs that
are resident in HBM.  The decode is launched over the (sequence, partition) units that
exist, planned from the host's copy of the lengths (pa_decode_planned; `--no-plan`: the
full grid).  The copies are done by the decode's own CTAs (pa_decode_cow;
`--cow separate`: a pa_copy_blocks launch before the step), and such workloads' lines
carry `cow_compare`, both forms timed alternately in the same run.  Default workload: the Llama-2-7B-shaped decode step (64
sequences, 32 q heads = 32 kv heads, head_dim 128, block size 16, bf16, context
lengths uniform in [128, 2048], shuffled physical blocks).

Prints ONE JSON line on rank 0.  `value` = algorithmic bytes of all ranks' steps /
max-over-ranks device time (GB/s); `e2e` = the same through the public API with
pinned host inputs copied in and the output copied out inside the timed region;
`roofline` = pa_decode's achieved bandwidth against the measured HBM copy rate;
`cpu_baseline` = the fp64 CPU oracle on the host cores.

`--impl reference` times that oracle alone (rank 0) in the same JSON format.

Other operations of the library, one JSON line each (`--op`):
  swap         preemption swap of a group of the workload's sequences to a pinned host
               pool and back (GB/s over the host link, against a pinned memcpy);
  prefill      causal multi-query attention of a prefill workload (--workload prefill_*;
               algorithmic TFLOP/s against the measured bf16 tensor rate);
  kv_write     the cache write alone (GB/s, L2 flushed before every call);
  copy_blocks  the copy-on-write block copy alone (the prefix workload).
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "paged decode attn KV-read GB/s (% of B200 HBM peak); decode seq-steps/s"
FALLBACK_HBM_GBS = 6650.0
WORKLOADS = {
    "llama2_7b": ("llama2_7b", {}, "Llama-2-7B-shaped decode step: 64 seqs, 32 q heads / 32 kv "
                  "heads, head_dim 128, block_size 16, bf16, context_lens U[128,2048], "
                  "pool = blocks needed + 10% spare, shuffled"),
    "gqa_llama3_8b": ("gqa_llama3_8b", {"block_size": 16}, "GQA Llama-3-8B-shaped decode: 256 "
                      "seqs, 32/8 heads, head_dim 128, bs 16, bf16, lognormal lens (median 1024)"),
    "gqa_llama3_8b_bs32": ("gqa_llama3_8b", {"block_size": 32}, "GQA Llama-3-8B-shaped decode at "
                           "block_size 32"),
    "long_8_1": ("long_8_1", {"block_size": 16}, "long-context split-K decode: 8 seqs, 8/1 heads, "
                 "head_dim 128, bs 16, lens U[32768,131072]"),
    "long_32_8": ("long_32_8", {"block_size": 16}, "long-context split-K decode: 8 seqs, 32/8 "
                  "heads, head_dim 128, bs 16, lens U[32768,131072]"),
    "long_8_1_bs512": ("long_8_1", {"block_size": 512}, "long-context split-K decode: 8 seqs, "
                       "8/1 heads, head_dim 128, bs 512, lens U[32768,131072]"),
    "long_32_8_bs512": ("long_32_8", {"block_size": 512}, "long-context split-K decode: 8 seqs, "
                        "32/8 heads, head_dim 128, bs 512, lens U[32768,131072]"),
    "prefix_cow": ("prefix_cow", {}, "prefix sharing + copy-on-write: 64 groups x 8 samples, "
                   "1000-token shared prefix, 32/8 heads, bs 16"),
    "window_4096_gqa": ("window_4096_gqa", {}, "sliding-window decode (W = 4096): 64 seqs, 32/8 "
                        "heads, head_dim 128, bs 16, lens U[8192,32768], only the pages of each "
                        "window held (earlier table entries -1)"),
}


# ----------------------------------------------------------------------------- bytes

def decode_bytes(case) -> int:
    """Algorithmic bytes of one pa_decode: K and V of every attended (sequence, kv head,
    token) once -- all L tokens, or the last W under a sliding window -- q and out once,
    the block-table entries of the attended pages, context lengths."""
    eb = 2
    L = case.context_lens.astype(np.int64)
    lo = np.maximum(L - case.window, 0) if case.window > 0 else np.zeros_like(L)
    kv = int((L - lo).sum()) * 2 * case.num_kv_heads * case.head_dim * eb
    qo = 2 * case.num_seqs * case.num_q_heads * case.head_dim * eb
    pages = (L + case.block_size - 1) // case.block_size - lo // case.block_size
    tables = int(pages.sum()) * 4 * case.num_kv_heads
    return kv + qo + tables + 4 * case.num_seqs


def write_bytes(case) -> int:
    T = case.slot_mapping.shape[0]
    return 2 * 2 * T * case.num_kv_heads * case.head_dim * 2 + 8 * T


def copy_bytes(case) -> int:
    P = case.copy_pairs.shape[0]
    return 2 * 2 * P * case.num_kv_heads * case.block_size * case.head_dim * 2 + 16 * P


def cow_bytes(case) -> int:
    """The copies pa_decode_cow makes: the named rows of every kv head, read and written
    in both caches, plus the per-sequence triples."""
    rows = int(case.cow[case.cow[:, 0] >= 0, 2].sum()) if case.cow.shape[0] else 0
    return 2 * 2 * rows * case.num_kv_heads * case.head_dim * 2 + 12 * case.cow.shape[0]


# ----------------------------------------------------------------------------- helpers

def bf16_peaks():
    """((burst TFLOP/s, kind), (sustained TFLOP/s, kind)): the measured cuBLAS bf16
    rates, else the profiling recipe's figures for this pool (1.59 PFLOP/s burst, about
    1.4 sustained under the 1 kW cap)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            j = json.load(f)
        burst = (float(j["bf16_tflops"]), "measured")
    except Exception:
        return (1590.0, "fallback"), (1400.0, "fallback")
    try:
        return burst, (float(j["bf16_tflops_sustained"]), "measured")
    except Exception:
        return burst, (1400.0, "fallback")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_sources_sha(names=("pa_common.cuh", "pa_decode.cuh")) -> str:
    """Identity of a kernel's sources (the kernel an ncu traffic figure was taken from);
    the decode partition kernel by default."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_441_b200", "csrc")
    for name in names:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_from_profile(workload: str, file: str = "decode_traffic.json",
                         names=("pa_common.cuh", "pa_decode.cuh")):
    """Per-launch DRAM bytes of a kernel from its committed ncu summary, or None when
    the kernel's sources changed since it was captured."""
    path = os.path.join(ROOT, "profiles", file)
    try:
        with open(path) as f:
            j = json.load(f)
    except Exception:
        return None
    if j.get("sources_sha") != kernel_sources_sha(names):
        return None
    entry = j.get("workloads", {}).get(workload)
    return None if entry is None else entry.get("dram_bytes_per_call")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed loop runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def workload_config(case, desc, ws):
    """The keys that identify a decode workload, the same in both arms' JSON lines."""
    return {"workload": desc, "num_seqs": case.num_seqs, "num_q_heads": case.num_q_heads,
            "num_kv_heads": case.num_kv_heads, "head_dim": case.head_dim,
            "block_size": case.block_size, "num_blocks": case.num_blocks,
            "kv_tokens": int(case.context_lens.sum()), "max_context_len": case.max_context_len,
            "sliding_window": case.window, "parallelism": f"dp{ws} (independent replicas)"}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, ws: int, device=None) -> float:
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, ws: int, device=None) -> float:
    if ws == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ----------------------------------------------------------------------------- CPU oracle

def oracle_step_time(case, sel=None, nthreads=0):
    """Wall time of the oracle's decode on `sel` (all (s, h) if None) over the
    already-written cache, plus the KV bytes that sample reads."""
    import oracle
    t = time.perf_counter()
    oracle.decode(case.q, case._kc_written, case._vc_written, case.block_tables,
                  case.context_lens, case.scale, case.dtype, sel=sel, nthreads=nthreads,
                  sliding_window=case.window)
    dt = time.perf_counter() - t
    return dt


def prepare_oracle(case):
    import oracle
    kc, vc = case.k_cache.copy(), case.v_cache.copy()
    if case.copy_pairs.shape[0]:
        oracle.copy_blocks(kc, vc, case.copy_pairs)
    oracle.kv_write(case.key, case.value, case.slot_mapping, kc, vc)
    case._kc_written, case._vc_written = kc, vc


def sel_bytes(case, sel) -> int:
    L = case.context_lens.astype(np.int64)
    G = case.num_q_heads // case.num_kv_heads
    # the oracle reads K and V once per (s, q head); count the distinct kv rows like the
    # GPU metric does: per (s, kv head) covered by the sample
    kvh = {(int(s), int(h) // G) for s, h in sel}
    span = np.minimum(L, case.window) if case.window > 0 else L
    kv = sum(int(span[s]) for s, _ in kvh) * 2 * case.head_dim * 2
    return kv + 2 * len(sel) * case.head_dim * 2


def cpu_baseline(case, budget_s=10.0):
    import oracle
    prepare_oracle(case)
    nthreads = oracle.max_threads()
    all_sel = np.array([(s, h) for s in range(case.num_seqs) for h in range(case.num_q_heads)],
                       np.int32)
    reps, total, t_all = 0, 0.0, 0.0
    while t_all < budget_s or reps == 0:
        dt = oracle_step_time(case, sel=all_sel, nthreads=nthreads)
        t_all += dt
        reps += 1
        if reps >= 50:
            break
    gbs = decode_bytes(case) * reps / t_all / 1e9
    # the same oracle on one thread, over a seeded sample of (seq, q head) pairs sized to
    # about a third of the budget
    rng = np.random.default_rng(0)
    probe = all_sel[rng.permutation(len(all_sel))[:8]]
    per_pair = oracle_step_time(case, sel=probe, nthreads=1) / len(probe)
    n1 = int(max(1, min(len(all_sel), budget_s / 3 / max(per_pair, 1e-9))))
    sel1 = all_sel[rng.permutation(len(all_sel))[:n1]]
    t1 = oracle_step_time(case, sel=sel1, nthreads=1)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": nthreads, "kind": "oracle",
            "sample": f"full workload decode (all {case.num_seqs} seqs x {case.num_q_heads} "
                      f"q heads), fp64 C oracle with OpenMP, repeated {reps}x in {t_all:.1f} s",
            "seq_steps_per_s": round(case.num_seqs * reps / t_all, 3),
            "single_thread": {"value": round(sel_bytes(case, sel1) / t1 / 1e9, 4),
                              "unit": "GB/s", "cores": 1,
                              "sample": f"{n1} of {len(all_sel)} (seq, q head) pairs, seeded, "
                                        f"{t1:.1f} s"}}


# ----------------------------------------------------------------------------- GPU arm

# The Llama-shaped decode workloads on which pa_decode is held to >= 70% of 8 TB/s; the
# default run times each of them beside the headline workload (one GPU).
PER_CONFIG = ["llama2_7b", "gqa_llama3_8b", "gqa_llama3_8b_bs32", "long_8_1", "long_8_1_bs512",
              "long_32_8", "long_32_8_bs512"]
ROOF_GROUP = 10        # consecutive calls between two events
ROOF_MIN_GROUPS = 20   # at least 200 calls ...
ROOF_MIN_S = 0.5       # ... and at least half a second of device time
FLUSH_CALLS = 50       # L2-flushed pass: median of this many single calls
FLUSH_BYTES = 256 << 20
PF_BURSTS = 10         # prefill burst pass: bursts of 10 calls ...
PF_BURST_IDLE_S = 0.05  # ... each after this idle pause (the clock recovers from the cap)


class DecodeStep:
    """A decode workload resident on the device and its step: copy-on-write copies (when
    the workload has them), the cache write and paged decode.  The write is fused into the
    decode (pa_decode_append) when every sequence appends exactly one token and nothing is
    copied; copies are done by the decode's own CTAs (pa_decode_cow, cow="folded") or by
    a pa_copy_blocks launch before the write (cow="separate")."""

    def __init__(self, torch, pa, case, device, partition_size, cow="folded", plan=True):
        self.case, self.pa = case, pa
        dt = case.dtype

        def d16(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(
                torch.bfloat16 if dt == "bf16" else torch.float16)

        def di(a):
            return torch.from_numpy(np.ascontiguousarray(a)).to(device)

        self.q, self.kc, self.vc = d16(case.q), d16(case.k_cache), d16(case.v_cache)
        self.key, self.val = d16(case.key), d16(case.value)
        self.sm, self.bt, self.cl = di(case.slot_mapping), di(case.block_tables), di(case.context_lens)
        self.pairs = di(case.copy_pairs.reshape(-1, 2).astype(np.int64))
        self.out = torch.empty_like(self.q)
        self.ps = partition_size
        W, mcl, win = case.max_blocks_per_seq, case.max_context_len, case.window
        need = pa.decode_workspace_bytes(case.num_seqs, case.num_q_heads, case.num_kv_heads,
                                         case.head_dim, case.block_size, W, mcl, partition_size,
                                         win)
        self.workspace = torch.zeros(max(need, 256), dtype=torch.uint8, device=device)
        ptoks = pa.decode_partition_tokens(case.num_seqs, case.num_q_heads, case.num_kv_heads,
                                           case.head_dim, case.block_size, W, mcl,
                                           partition_size, win)
        span = min(mcl, W * case.block_size, win + 15 if win > 0 else mcl)
        nparts = 0 if ptoks == 0 else -(-span // ptoks)
        self.has_pairs = case.copy_pairs.shape[0] > 0
        self.cow_folded = (self.has_pairs and cow == "folded" and partition_size >= 0
                           and case.cow.shape[0] == case.num_seqs)
        self.cow = di(case.cow) if self.cow_folded else None
        self.fused = ((not self.has_pairs) and case.key.shape[0] == case.num_seqs
                      and partition_size >= 0)
        # launch planned from the host's copy of the lengths (fixed split, no window)
        self.plan = plan and partition_size >= 0 and case.window == 0 and not self.cow_folded
        self.host_lens = np.ascontiguousarray(case.context_lens, np.int32)
        decode_launches = 1 if nparts == 1 else 2
        self.launches_per_step = decode_launches + (
            0 if self.fused else 1 + (1 if self.has_pairs and not self.cow_folded else 0))
        self.split = (f"fixed {ptoks}-token partitions, {nparts} max" if ptoks > 0 else
                      "dynamic: persistent CTAs claim 32-token chunks + LSE merge"
                      if partition_size == -2 else
                      "balanced over persistent warps (stream-K) + LSE merge")
        self.kind = ("pa_decode_planned (cache write fused into decode; the (sequence, "
                     "partition) units that exist, planned from the host lengths)"
                     if self.plan and self.fused
                     else "pa_kv_write + pa_decode_planned" if self.plan and not self.has_pairs
                     else "pa_copy_blocks + pa_kv_write + pa_decode_planned" if self.plan
                     else "pa_decode_append (cache write fused into decode)" if self.fused
                     else "pa_kv_write + pa_decode_cow (copy-on-write rows copied by the "
                          "partition pass)" if self.cow_folded
                     else "pa_copy_blocks + pa_kv_write + pa_decode" if self.has_pairs
                     else "pa_kv_write + pa_decode")
        self.step_bytes = (decode_bytes(case) + write_bytes(case)
                           + (cow_bytes(case) if self.cow_folded else
                              copy_bytes(case) if self.has_pairs else 0))

    def decode(self, b=None):
        """The attention call of the step (with the fused write when the step has it)."""
        c, pa = self.case, self.pa
        b = b or {}
        out, q = b.get("out", self.out), b.get("q", self.q)
        bt, cl = b.get("bt", self.bt), b.get("cl", self.cl)
        if self.plan:
            kv = (dict(key=b.get("key", self.key), value=b.get("val", self.val)) if self.fused
                  else {})
            pa.decode_planned(out, q, self.kc, self.vc, bt, cl, self.host_lens, c.scale,
                              max_context_len=c.max_context_len, partition_size=self.ps,
                              workspace=self.workspace, **kv)
        elif self.fused:
            pa.decode_append(out, q, b.get("key", self.key), b.get("val", self.val), self.kc,
                             self.vc, bt, cl, c.scale, max_context_len=c.max_context_len,
                             partition_size=self.ps, workspace=self.workspace,
                             sliding_window=c.window)
        elif self.cow_folded:
            pa.decode_cow(out, q, self.kc, self.vc, bt, cl, b.get("cow", self.cow), c.scale,
                          max_context_len=c.max_context_len, partition_size=self.ps,
                          workspace=self.workspace, sliding_window=c.window)
        else:
            pa.decode(out, q, self.kc, self.vc, bt, cl, c.scale, max_context_len=c.max_context_len,
                      partition_size=self.ps, workspace=self.workspace, sliding_window=c.window)

    def step(self, b=None):
        b = b or {}
        if not self.fused:
            if self.has_pairs and not self.cow_folded:
                self.pa.copy_blocks(self.kc, self.vc, b.get("pairs", self.pairs))
            self.pa.kv_write(b.get("key", self.key), b.get("val", self.val),
                             b.get("sm", self.sm), self.kc, self.vc)
        self.decode(b)


def time_groups(torch, fn, stream, est_ms, min_s=ROOF_MIN_S):
    """Per-call device time of `fn`: CUDA events on the launching stream around groups of
    ROOF_GROUP consecutive calls (an event between every two launches would stop each
    kernel from being scheduled while the previous one drains), for at least
    ROOF_MIN_GROUPS groups and `min_s` seconds.  Returns (median ms per call over the
    groups, number of calls)."""
    n = max(ROOF_MIN_GROUPS, int(math.ceil(min_s * 1e3 / (ROOF_GROUP * max(est_ms, 1e-3)))))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    for i in range(n):
        ev[i][0].record(stream)
        for _ in range(ROOF_GROUP):
            fn()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) / ROOF_GROUP for a, b in ev), n * ROOF_GROUP


class L2Flush:
    """Leaves L2 cold and clean: writes a FLUSH_BYTES buffer (twice the 126 MB L2), then
    reads another, so the written lines are evicted -- and written back -- before the
    timed call instead of during it."""

    def __init__(self, torch, device):
        self.w = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.r = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.k = 0

    def __call__(self):
        self.k += 1
        self.w.fill_(float(self.k))
        self.r.sum()


def time_flushed(torch, fn, stream, flush):
    """Median device time of FLUSH_CALLS single calls of `fn`, L2 flushed before each."""
    times = []
    for _ in range(FLUSH_CALLS):
        flush()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        b.synchronize()
        times.append(a.elapsed_time(b))
    return statistics.median(times)


def measure_config(torch, pa, name, device, stream, args, peak, flush):
    """One per-config entry: the workload's step on its own, timed like the headline's
    roofline pass (median over groups of consecutive calls) and L2-flushed."""
    wname, kw, desc = WORKLOADS[name]
    from workloads import make_config
    case = make_config(wname, poison=False, **kw)
    ds = DecodeStep(torch, pa, case, device, args.partition_size, plan=not args.no_plan)
    for _ in range(args.warmup):
        ds.step()
    torch.cuda.synchronize()
    sampler = ClockSampler(device.index)
    sampler.start()
    time.sleep(0.2)
    t = time.perf_counter()
    ds.decode()
    torch.cuda.synchronize()
    est = (time.perf_counter() - t) * 1e3
    ms, ncalls = time_groups(torch, ds.decode, stream, est, args.roofline_s)
    clocks = sampler.stop()
    ms_flushed = time_flushed(torch, ds.decode, stream, flush)
    err = pa.device_error(device.index)
    if err:
        raise RuntimeError(f"device error word {err:#x} in the {name} pass")
    db = decode_bytes(case)
    ach, ach_f = db / (ms * 1e-3) / 1e9, db / (ms_flushed * 1e-3) / 1e9
    entry = {"workload": desc, "block_size": case.block_size, "split": ds.split, "call": ds.kind,
             "value": round(ach, 1), "unit": "GB/s", "ms_per_call": round(ms, 6),
             "pct_of_8tbs": round(100 * ach / 8000.0, 2), "meets_70pct_of_8tbs": ach >= 5600.0,
             "roofline": {"achieved": round(ach, 1), "frac": round(ach / peak, 4),
                          "frac_l2_flushed": round(ach_f / peak, 4),
                          "ms_per_call_l2_flushed": round(ms_flushed, 6),
                          "algorithmic_bytes_per_call": db, "calls": ncalls,
                          "traffic": traffic_from_profile(name)},
             "clocks": clocks}
    del ds
    torch.cuda.empty_cache()
    return entry


def run_ours(args):
    import torch
    ws, rank, local = dist_env()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())

    import paged_kv_cache_441_b200 as pa
    from workloads import make_config

    name, kw, desc = WORKLOADS[args.workload]
    if args.seqs:
        kw = dict(kw, num_seqs=args.seqs)
        desc = f"{desc} [profiling subset: first {args.seqs} seqs' distribution]"
    case = make_config(name, poison=False, **kw)
    dt = case.dtype
    ds = DecodeStep(torch, pa, case, device, args.partition_size, cow=args.cow,
                    plan=not args.no_plan)
    q, out = ds.q, ds.out
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        ds.step()
    torch.cuda.synchronize()
    pa.device_error(torch.cuda.current_device())  # clears; warm-up must be clean

    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        ds.step()
    t1.record(stream)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    elapsed_ms = t0.elapsed_time(t1)
    clocks = sampler.stop()

    # Roofline pass: the attention call alone (the fused call when the step has it), a
    # fixed length independent of --steps, with its own clock record; then single calls
    # after an L2 flush.
    roof_sampler = ClockSampler(torch.cuda.current_device())
    roof_sampler.start()
    time.sleep(0.2)
    dec_ms, roof_calls = time_groups(torch, ds.decode, stream, elapsed_ms / max(args.steps, 1),
                                     args.roofline_s)
    roof_clocks = roof_sampler.stop()
    flush = L2Flush(torch, device)
    dec_ms_flushed = time_flushed(torch, ds.decode, stream, flush)
    errbits = pa.device_error(torch.cuda.current_device())
    if errbits:
        raise RuntimeError(f"device error word {errbits:#x} during the timed loop")

    # ---- end to end through the public API: pinned host inputs in, output out
    h_q = torch.from_numpy(case.q.view(np.int16)).view(q.dtype).pin_memory()
    h_key = torch.from_numpy(case.key.view(np.int16)).view(q.dtype).pin_memory()
    h_val = torch.from_numpy(case.value.view(np.int16)).view(q.dtype).pin_memory()
    h_sm = torch.from_numpy(case.slot_mapping).pin_memory()
    h_bt = torch.from_numpy(case.block_tables).pin_memory()
    h_cl = torch.from_numpy(case.context_lens).pin_memory()
    h_pairs = torch.from_numpy(case.copy_pairs.reshape(-1, 2).astype(np.int64)).pin_memory()
    h_cow = torch.from_numpy(case.cow).pin_memory()
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d_bytes = sum(t.numel() * t.element_size() for t in (h_q, h_key, h_val, h_sm, h_bt, h_cl))
    h2d_bytes += (h_cow.numel() * 4 if ds.cow_folded else
                  h_pairs.numel() * 8 if ds.has_pairs else 0)
    d2h_bytes = h_out.numel() * h_out.element_size()
    e2e_steps = max(1, min(args.steps, args.e2e_steps))

    # A serving loop double-buffers the step inputs: while step i computes on one set
    # of device buffers, step i+1's inputs are copied into the other set on a copy
    # stream, and step i's output is read back on that stream as soon as it is ready.
    # Every step still copies all of its own inputs in and its output out.
    copy_stream = torch.cuda.Stream(device=device)
    bufs = [dict(q=torch.empty_like(q), key=torch.empty_like(ds.key), val=torch.empty_like(ds.val),
                 sm=torch.empty_like(ds.sm), bt=torch.empty_like(ds.bt), cl=torch.empty_like(ds.cl),
                 pairs=torch.empty_like(ds.pairs), out=torch.empty_like(out),
                 cow=torch.empty_like(ds.cow) if ds.cow_folded else None) for _ in range(2)]
    h_outs = [h_out, torch.empty(out.shape, dtype=out.dtype).pin_memory()]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_read = [torch.cuda.Event() for _ in range(2)]

    def h2d(i):
        b = bufs[i % 2]
        with torch.cuda.stream(copy_stream):
            if i >= 2:
                copy_stream.wait_event(ev_done[i % 2])  # step i-2 is done with this set
            b["q"].copy_(h_q, non_blocking=True)
            b["key"].copy_(h_key, non_blocking=True)
            b["val"].copy_(h_val, non_blocking=True)
            b["sm"].copy_(h_sm, non_blocking=True)
            b["bt"].copy_(h_bt, non_blocking=True)
            b["cl"].copy_(h_cl, non_blocking=True)
            if ds.cow_folded:
                b["cow"].copy_(h_cow, non_blocking=True)
            elif ds.has_pairs:
                b["pairs"].copy_(h_pairs, non_blocking=True)
            ev_in[i % 2].record(copy_stream)

    def compute(i):
        b = bufs[i % 2]
        stream.wait_event(ev_in[i % 2])
        if i >= 2:
            stream.wait_event(ev_read[i % 2])  # step i-2's output has been read back
        ds.step(b)
        ev_done[i % 2].record(stream)

    def d2h(i):
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(ev_done[i % 2])
            h_outs[i % 2].copy_(bufs[i % 2]["out"], non_blocking=True)
            ev_read[i % 2].record(copy_stream)

    def run_e2e(n):
        h2d(0)
        for i in range(n):
            if i + 1 < n:
                h2d(i + 1)
            compute(i)
            d2h(i)

    run_e2e(args.warmup)
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_stream.wait_event(e0)
    run_e2e(e2e_steps)
    fin = torch.cuda.Event()
    fin.record(copy_stream)
    stream.wait_event(fin)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    # the end-to-end loop computes the same step: bit for bit under a fixed split; the
    # dynamic split's sums vary in the last bits from call to call
    torch.testing.assert_close(h_outs[(e2e_steps - 1) % 2].float(), out.cpu().float(), rtol=0,
                               atol=0 if args.partition_size != -2 else 1e-3)

    # ---- the same step with the copies in their own launch (or folded in), timed in
    # alternation with this one: what folding the copy-on-write into the decode gives
    cow_compare = None
    if ds.has_pairs and ws == 1 and args.partition_size >= 0:
        other = DecodeStep(torch, pa, case, device, args.partition_size,
                           cow="separate" if ds.cow_folded else "folded")
        for _ in range(args.warmup):
            other.step()
        torch.cuda.synchronize()
        est = elapsed_ms / max(args.steps, 1)
        t_this, t_other = [], []
        for _ in range(2):
            t_this.append(time_groups(torch, ds.step, stream, est, args.roofline_s / 2)[0])
            t_other.append(time_groups(torch, other.step, stream, est, args.roofline_s / 2)[0])
        if pa.device_error(device.index):
            raise RuntimeError("device error word set in the copy-on-write comparison")
        folded, separate = ((t_this, t_other) if ds.cow_folded else (t_other, t_this))
        cow_compare = {
            "folded_us_per_step": round(1e3 * statistics.mean(folded), 2),
            "separate_us_per_step": round(1e3 * statistics.mean(separate), 2),
            "folded": "pa_kv_write + pa_decode_cow (rows copied by the CTAs that read them)",
            "separate": "pa_copy_blocks + pa_kv_write + pa_decode",
            "how": "median over groups of consecutive steps, two alternating passes each"}
        del other

    # ---- aggregate over ranks
    max_ms = max_over_ranks(elapsed_ms, ws, device)
    max_e2e_ms = max_over_ranks(e2e_ms, ws, device)
    tot_bytes = sum_over_ranks(float(ds.step_bytes), ws, device)
    ms_per_step = max_ms / args.steps
    value = tot_bytes / (ms_per_step * 1e-3) / 1e9
    e2e_value = tot_bytes / (max_e2e_ms / e2e_steps * 1e-3) / 1e9
    achieved = decode_bytes(case) / (dec_ms * 1e-3) / 1e9
    achieved_flushed = decode_bytes(case) / (dec_ms_flushed * 1e-3) / 1e9
    peak, peak_kind = peaks()
    result = None
    if rank == 0:
        # The other Llama-shaped configs, each timed on its own (one GPU only: the
        # per-rank replicas of a multi-GPU run are the headline workload).
        per_config = None
        if ws == 1 and not args.no_per_config and args.workload in PER_CONFIG:
            head = {"workload": desc, "block_size": case.block_size, "split": ds.split,
                    "call": ds.kind, "value": round(achieved, 1), "unit": "GB/s",
                    "ms_per_call": round(dec_ms, 6),
                    "pct_of_8tbs": round(100 * achieved / 8000.0, 2),
                    "meets_70pct_of_8tbs": achieved >= 5600.0,
                    "roofline": {"achieved": round(achieved, 1), "frac": round(achieved / peak, 4),
                                 "frac_l2_flushed": round(achieved_flushed / peak, 4),
                                 "ms_per_call_l2_flushed": round(dec_ms_flushed, 6),
                                 "algorithmic_bytes_per_call": decode_bytes(case),
                                 "calls": roof_calls,
                                 "traffic": traffic_from_profile(args.workload)},
                    "clocks": roof_clocks}
            per_config = {}
            for cname in PER_CONFIG:
                per_config[cname] = (head if cname == args.workload else
                                     measure_config(torch, pa, cname, device, stream, args, peak,
                                                    flush))
        cpu = None if args.no_cpu_baseline or ws > 1 else cpu_baseline(case, args.cpu_budget)
        result = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "GB/s",
            "n_gpus": ws,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 6),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": dt,
            "data": "synthetic (seeded N(0,1) q/K/V rounded to bf16, shuffled block pool)",
            "config": workload_config(case, desc, ws),
            "plan": {"split": ds.split, "step": ds.kind,
                     "l2": f"inputs larger than L2 ({decode_bytes(case) / 1e9:.2f} GB of K/V "
                           f"read per step vs 126 MB); the timed steps run back to back "
                           f"without a flush; roofline.frac_l2_flushed times single calls "
                           f"after a {FLUSH_BYTES >> 20} MB write + read"},
            **({"cow_compare": cow_compare} if cow_compare else {}),
            "seq_steps_per_s": round(case.num_seqs * ws / (ms_per_step * 1e-3), 1),
            "pct_of_8tbs": round(100 * value / 8000.0, 2),
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d_bytes,
                    "d2h_bytes_per_step": d2h_bytes, "steps": e2e_steps,
                    "how": "pa_* calls on double-buffered device inputs; each step's inputs "
                           "copied from pinned host memory and its output read back on a copy "
                           "stream that overlaps the previous step's compute"},
            "gpu_launches": ds.launches_per_step * args.steps,
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "peak_kind": f"{peak_kind} HBM copy GB/s (burst)",
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "frac_l2_flushed": round(achieved_flushed / peak, 4),
                         "kernel": ("pa_decode_planned (the partition pass over the planned "
                                    "units, cache write fused in) + LSE merge"
                                    if ds.plan and ds.fused else
                                    "pa_decode_append (cache write fused into the partition "
                                    "pass) + LSE merge" if ds.fused else
                                    "pa_decode (partition pass + LSE merge when split)"),
                         "achieved_how": (f"algorithmic bytes / median per-call CUDA-event time "
                                          f"over groups of {ROOF_GROUP} consecutive calls "
                                          f"({roof_calls} calls, >= {args.roofline_s} s, a pass of "
                                          f"its own after the timed steps); frac_l2_flushed: "
                                          f"median of {FLUSH_CALLS} single calls, each after an "
                                          f"L2 flush"),
                         "algorithmic_bytes_per_call": decode_bytes(case),
                         "avg_call_us": round(dec_ms * 1e3, 2),
                         "call_us_l2_flushed": round(dec_ms_flushed * 1e3, 2),
                         "traffic": traffic_from_profile(args.workload),
                         "clocks": roof_clocks},
            "clocks": clocks,
            "per_config": per_config,
            "cpu_baseline": cpu,
        }
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def run_swap(args):
    """Preemption swap of the benchmark workload: the block manager swaps a group of
    sequences out to a pinned host pool and back in; pa_swap_blocks moves the blocks.
    value = bytes that cross the host link per (swap out + swap in) / device time;
    the ceiling is a contiguous pinned cudaMemcpyAsync of the same bytes, each way,
    timed in the same process."""
    import torch
    ws, rank, local = dist_env()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    import paged_kv_cache_441_b200 as pa
    from workloads import make_config

    name, kw, desc = WORKLOADS[args.workload]
    case = make_config(name, poison=False, **kw)
    tdt = torch.bfloat16 if case.dtype == "bf16" else torch.float16
    kc = torch.from_numpy(case.k_cache.view(np.int16)).to(device).view(tdt)
    vc = torch.from_numpy(case.v_cache.view(np.int16)).to(device).view(tdt)
    nb, hkv, bs, d = kc.shape
    lens = case.context_lens.astype(np.int64)
    bm = pa.BlockManager(nb, bs)
    for s in range(case.num_seqs):
        bm.allocate(s, int(lens[s]))
    group = list(range(min(args.swap_seqs, case.num_seqs)))  # the preempted sequences
    ncpu = sum(pa.blocks_needed(int(lens[s]), bs) for s in group)
    bm.set_cpu_pool(ncpu)
    kh = torch.empty((ncpu, hkv, bs, d), dtype=tdt).pin_memory()
    vh = torch.empty((ncpu, hkv, bs, d), dtype=tdt).pin_memory()
    stream = torch.cuda.current_stream()

    def swap_cycle():
        out_pairs = torch.from_numpy(bm.swap_out(group)).to(device)
        pa.swap_blocks(kh, vh, kc, vc, out_pairs)
        in_pairs = torch.from_numpy(bm.swap_in(group)).to(device)
        pa.swap_blocks(kc, vc, kh, vh, in_pairs)

    # kernel-only pass: fixed pair lists, resident on the device
    out_pairs = torch.from_numpy(bm.swap_out(group)).to(device)
    in_pairs = torch.from_numpy(bm.swap_in(group)).to(device)
    moved = 2 * ncpu * hkv * bs * d * kc.element_size()  # K and V, one direction

    def timed(fn, reps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(a.elapsed_time(b), ws, device) / reps

    sampler = ClockSampler(local)
    sampler.start()
    ms_out = timed(lambda: pa.swap_blocks(kh, vh, kc, vc, out_pairs), args.steps)
    ms_in = timed(lambda: pa.swap_blocks(kc, vc, kh, vh, in_pairs), args.steps)
    clocks = sampler.stop()
    ms_e2e = timed(swap_cycle, args.steps)
    flat_h = torch.empty(moved // 2, dtype=torch.int16).pin_memory()
    flat_d = torch.empty(moved // 2, dtype=torch.int16, device=device)
    ms_d2h = timed(lambda: flat_h.copy_(flat_d, non_blocking=True), args.steps)
    ms_h2d = timed(lambda: flat_d.copy_(flat_h, non_blocking=True), args.steps)
    err = pa.device_error(device.index)
    bm.close()
    result = None
    if rank == 0:
        step_ms = ms_out + ms_in
        value = 2 * moved * ws / (step_ms * 1e-3) / 1e9
        peak = 2 * moved / ((ms_d2h + ms_h2d) * 1e-3) / 1e9
        result = {
            "metric": "KV block swap GB/s (device <-> pinned host, out + in)",
            "value": round(value, 2), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(step_ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": case.dtype,
            "data": "synthetic (the benchmark workload's seeded cache)",
            "config": {"workload": f"swap out + swap in of {len(group)} of {case.num_seqs} "
                                   f"sequences of: {desc}",
                       "blocks_per_direction": ncpu, "bytes_per_direction": moved,
                       "l2": "host memory is not cached in L2; no flush"},
            "swap_out_gbs": round(moved / (ms_out * 1e-3) / 1e9, 2),
            "swap_in_gbs": round(moved / (ms_in * 1e-3) / 1e9, 2),
            "e2e": {"value": round(2 * moved * ws / (ms_e2e * 1e-3) / 1e9, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": 8 * 2 * ncpu * 2, "d2h_bytes_per_step": 0,
                    "how": "BlockManager.swap_out / swap_in on the host, the pair lists "
                           "copied to the device, then pa_swap_blocks each way"},
            "gpu_launches": 2 * args.steps,
            "roofline": {"bound": "host_link", "achieved": round(value / ws, 2),
                         "peak": round(peak, 2), "unit": "GB/s",
                         "frac": round(value / ws / peak, 4),
                         "peak_kind": "measured in this run: contiguous pinned cudaMemcpyAsync "
                                      "of the same bytes, device->host and host->device",
                         "memcpy_d2h_gbs": round(moved / (ms_d2h * 1e-3) / 1e9, 2),
                         "memcpy_h2d_gbs": round(moved / (ms_h2d * 1e-3) / 1e9, 2),
                         "kernel": "pa_swap_blocks", "traffic": None},
            "clocks": clocks,
            "device_error": err,
        }
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


PREFILL_WORKLOADS = {
    "prefill_2k_gqa": "prefill of whole prompts: 8 sequences x 2048 tokens, 32/8 heads, "
                      "head_dim 128, bs 16, bf16",
    "prefill_chunk512_gqa": "chunked prefill: 16 sequences each adding 512 tokens to "
                            "1536..3072 earlier ones, 32/8 heads, head_dim 128, bs 16, bf16",
}


def prefill_flops(case) -> int:
    """Algorithmic FLOPs of one pa_prefill: for every (token, query head), q.K over the
    keys it attends (2 d each) and P.V over the same keys (2 d each)."""
    qsl = case.query_start_loc.astype(np.int64)
    keys = 0
    for s in range(case.num_seqs):
        n, L = int(qsl[s + 1] - qsl[s]), int(case.context_lens[s])
        pos = np.arange(L - n, L, dtype=np.int64)
        att = pos + 1 if case.window <= 0 else np.minimum(pos + 1, case.window)
        keys += int(att.sum())
    return 4 * case.head_dim * case.num_q_heads * keys


def prefill_sample_flops(case, sel) -> int:
    qsl = case.query_start_loc.astype(np.int64)
    tot = 0
    for t, _ in sel:
        s = int(np.searchsorted(qsl, t, side="right") - 1)
        n, L = int(qsl[s + 1] - qsl[s]), int(case.context_lens[s])
        p = L - n + (int(t) - int(qsl[s]))
        tot += 4 * case.head_dim * (p + 1 if case.window <= 0 else min(p + 1, case.window))
    return tot


def prefill_oracle_sample(case, budget_s, rng):
    """The fp64 oracle (after the chunk's cache write) on seeded (token, head) samples
    until about budget_s seconds: (TFLOP/s, threads, sample text)."""
    import oracle
    kc, vc = case.k_cache.copy(), case.v_cache.copy()
    oracle.kv_write(case.key, case.value, case.slot_mapping, kc, vc)
    nthreads = oracle.max_threads()
    n, t_all, fl = 256, 0.0, 0
    while t_all < budget_s:
        sel = np.stack([rng.integers(0, case.num_tokens, size=n),
                        rng.integers(0, case.num_q_heads, size=n)], 1).astype(np.int32)
        t = time.perf_counter()
        oracle.prefill(case.q, kc, vc, case.block_tables, case.context_lens,
                       case.query_start_loc, case.scale, case.dtype,
                       sliding_window=case.window, sel=sel, nthreads=nthreads)
        t_all += time.perf_counter() - t
        fl += prefill_sample_flops(case, sel)
    return fl / t_all / 1e12, nthreads, (f"{fl / prefill_flops(case):.4f} of the step's work as "
                                        f"seeded (token, head) samples, {t_all:.1f} s")


def run_prefill(args):
    """Prefill / chunked-prefill step: the chunk's cache write + causal attention."""
    import torch
    ws, rank, local = dist_env()
    if args.impl == "reference":
        if rank != 0:
            return None
        from workloads import make_prefill_config
        case = make_prefill_config(args.workload)
        value, nthreads, sample = prefill_oracle_sample(case, args.reference_budget,
                                                        np.random.default_rng(0))
        return {"impl": "reference", "metric": "prefill attention TFLOP/s", "value": round(value, 6),
                "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(prefill_flops(case) / (value * 1e12) * 1e3, 3),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": {"workload": PREFILL_WORKLOADS[args.workload]},
                "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": nthreads,
                                 "kind": "oracle", "sample": sample},
                "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    device = torch.device("cuda", torch.cuda.current_device())
    import paged_kv_cache_441_b200 as pa
    from workloads import make_prefill_config
    case = make_prefill_config(args.workload, poison=False)
    tdt = torch.bfloat16 if case.dtype == "bf16" else torch.float16

    def d16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(tdt)

    def di(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    q, kc, vc = d16(case.q), d16(case.k_cache), d16(case.v_cache)
    key, val, sm = d16(case.key), d16(case.value), di(case.slot_mapping)
    bt, cl, qsl = di(case.block_tables), di(case.context_lens), di(case.query_start_loc)
    out = torch.empty_like(q)
    win = case.window
    stream = torch.cuda.current_stream()

    def step():
        pa.kv_write(key, val, sm, kc, vc)
        pa.prefill(out, q, kc, vc, bt, cl, qsl, case.scale, sliding_window=win)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    pa.device_error(device.index)
    sampler = ClockSampler(device.index)
    sampler.start()
    time.sleep(0.3)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    elapsed = t0.elapsed_time(t1)
    # roofline pass: pa_prefill alone, events around groups of 10 calls
    group = 10
    ngroups = max(1, args.steps // group)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(ngroups)]
    for i in range(ngroups):
        ev[i][0].record(stream)
        for _ in range(group):
            pa.prefill(out, q, kc, vc, bt, cl, qsl, case.scale, sliding_window=win)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    call_ms = sum(a.elapsed_time(b) for a, b in ev) / (ngroups * group)
    # burst pass: the kernel timed alone at full clock -- bursts of 10 calls, each after
    # an idle pause; under a long back-to-back loop the 1 kW power cap lowers the clock
    burst_ms = []
    for _ in range(PF_BURSTS):
        time.sleep(PF_BURST_IDLE_S)
        torch.cuda.synchronize()
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        for _ in range(group):
            pa.prefill(out, q, kc, vc, bt, cl, qsl, case.scale, sliding_window=win)
        b_.record(stream)
        torch.cuda.synchronize()
        burst_ms.append(a_.elapsed_time(b_) / group)
    burst_call_ms = statistics.median(burst_ms)
    err = pa.device_error(device.index)
    if err:
        raise RuntimeError(f"device error word {err:#x} during the timed loop")

    # end to end: q and the chunk's key/value/slots and metadata in from pinned memory,
    # the output back, every step (serialised on one stream)
    hq_ = torch.from_numpy(case.q.view(np.int16)).view(tdt).pin_memory()
    hk_ = torch.from_numpy(case.key.view(np.int16)).view(tdt).pin_memory()
    hv_ = torch.from_numpy(case.value.view(np.int16)).view(tdt).pin_memory()
    hsm = torch.from_numpy(case.slot_mapping).pin_memory()
    hmeta = [torch.from_numpy(a).pin_memory() for a in (case.block_tables, case.context_lens,
                                                         case.query_start_loc)]
    hout = torch.empty(out.shape, dtype=tdt).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in [hq_, hk_, hv_, hsm] + hmeta)
    d2h = hout.numel() * hout.element_size()
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        q.copy_(hq_, non_blocking=True)
        key.copy_(hk_, non_blocking=True)
        val.copy_(hv_, non_blocking=True)
        sm.copy_(hsm, non_blocking=True)
        for d_, h_ in zip((bt, cl, qsl), hmeta):
            d_.copy_(h_, non_blocking=True)
        step()
        hout.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)

    flops = prefill_flops(case)
    max_ms = max_over_ranks(elapsed, ws, device)
    ms_step = max_ms / args.steps
    value = flops * ws / (ms_step * 1e-3) / 1e12
    e2e_val = flops * ws / (max_over_ranks(e2e_ms, ws, device) / e2e_steps * 1e-3) / 1e12
    achieved = flops / (call_ms * 1e-3) / 1e12
    achieved_burst = flops / (burst_call_ms * 1e-3) / 1e12
    (peak, peak_kind), (peak_s, peak_s_kind) = bf16_peaks()
    result = None
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and ws == 1:
            v, nthreads, sample = prefill_oracle_sample(case, args.cpu_budget,
                                                        np.random.default_rng(1))
            cpu = {"value": round(v, 6), "unit": "TFLOP/s", "cores": nthreads, "kind": "oracle",
                   "sample": sample}
        result = {
            "metric": "prefill attention TFLOP/s", "value": round(value, 2), "unit": "TFLOP/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": case.dtype,
            "data": "synthetic (seeded N(0,1) q/K/V rounded to bf16, shuffled block pool)",
            "config": {"workload": PREFILL_WORKLOADS[args.workload],
                       "num_seqs": case.num_seqs, "num_tokens": case.num_tokens,
                       "num_q_heads": case.num_q_heads, "num_kv_heads": case.num_kv_heads,
                       "head_dim": case.head_dim, "block_size": case.block_size,
                       "sliding_window": win, "step": "pa_kv_write (chunk) + pa_prefill",
                       "parallelism": f"dp{ws} (independent replicas)",
                       "l2": "no flush: the K/V read per call is well under L2; the work is "
                             "tensor-bound"},
            "algorithmic_flops_per_step": flops,
            "e2e": {"value": round(e2e_val, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "gpu_launches": 2 * args.steps,
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak_s,
                         "peak_kind": f"{peak_s_kind} cuBLAS bf16 TFLOP/s (sustained: this pass "
                                      "is a long back-to-back loop under the power cap)",
                         "unit": "TFLOP/s",
                         "frac": round(achieved / peak_s, 4), "kernel": "pa_prefill",
                         "avg_call_us": round(call_ms * 1e3, 2),
                         "achieved_how": "algorithmic FLOPs (both products once; the split "
                                         "P's second product and masked tile work not "
                                         "counted) / mean CUDA-event time per call, events "
                                         "around groups of 10 back-to-back calls after the "
                                         "timed steps",
                         "burst": {"achieved": round(achieved_burst, 2), "peak": peak,
                                   "peak_kind": f"{peak_kind} cuBLAS bf16 TFLOP/s (burst)",
                                   "frac": round(achieved_burst / peak, 4),
                                   "avg_call_us": round(burst_call_ms * 1e3, 2),
                                   "how": f"median over {PF_BURSTS} bursts of 10 calls, each "
                                          f"after {PF_BURST_IDLE_S * 1e3:.0f} ms idle"},
                         "traffic": traffic_from_profile(args.workload, "prefill_traffic.json",
                                                         ("pa_common.cuh", "pa_prefill.cuh"))},
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def run_cache_op(args):
    """pa_kv_write or pa_copy_blocks alone: algorithmic bytes (read + written) / the median
    CUDA-event time of one call, with L2 flushed (256 MB read) before every call."""
    import torch
    import paged_kv_cache_441_b200 as pa
    torch.cuda.set_device(0)
    device = torch.device("cuda", 0)
    from workloads import make_config, make_prefill_config
    if args.workload in PREFILL_WORKLOADS:
        case = make_prefill_config(args.workload, poison=False)
        desc = PREFILL_WORKLOADS[args.workload] + " (the chunk's cache write)"
    else:
        name, kw, desc = WORKLOADS[args.workload]
        case = make_config(name, poison=False, **kw)
    tdt = torch.bfloat16 if case.dtype == "bf16" else torch.float16

    def d16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(tdt)

    kc, vc = d16(case.k_cache), d16(case.v_cache)
    key, val = d16(case.key), d16(case.value)
    sm = torch.from_numpy(case.slot_mapping).to(device)
    pairs = torch.from_numpy(np.ascontiguousarray(
        getattr(case, "copy_pairs", np.zeros((0, 2), np.int64)).reshape(-1, 2).astype(np.int64))).to(device)
    T = int(case.slot_mapping.shape[0])
    hkv, bs, d = case.num_kv_heads, case.block_size, case.head_dim
    if args.op == "kv_write":
        nbytes = 2 * 2 * T * hkv * d * 2 + 8 * T
        fn = lambda: pa.kv_write(key, val, sm, kc, vc)  # noqa: E731
        what = f"{T} tokens x {hkv} kv heads x {d}"
    else:
        if pairs.shape[0] == 0:
            raise SystemExit("--op copy_blocks needs a workload with copy-on-write pairs")
        P = int(pairs.shape[0])
        nbytes = 2 * 2 * P * hkv * bs * d * 2 + 16 * P
        fn = lambda: pa.copy_blocks(kc, vc, pairs)  # noqa: E731
        what = f"{P} block pairs x 2 caches x {hkv * bs * d * 2} B"
    # L2 flush by reading 256 MB: the lines it leaves are clean, so the timed op does not
    # also pay for writing back the flush's own data
    flush = torch.ones(64 << 20, dtype=torch.float32, device=device)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    sampler = ClockSampler(0)
    sampler.start()
    times = []
    for _ in range(args.steps):
        flush.sum()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        times.append(a.elapsed_time(b))
    clocks = sampler.stop()
    err = pa.device_error(0)
    if err:
        raise RuntimeError(f"device error word {err:#x}")
    ms = statistics.median(times)
    value = nbytes / (ms * 1e-3) / 1e9
    # size-matched reference: one contiguous device-to-device copy of the same bytes
    # (nbytes / 2 read, as many written), same flush, same statistic -- at tens of MB the
    # ramp and tail of any copy are a large share of the call
    src_ = torch.empty(nbytes // 2, dtype=torch.uint8, device=device)
    dst_ = torch.empty_like(src_)
    ref_times = []
    for _ in range(args.steps):
        flush.sum()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        dst_.copy_(src_)
        b.record()
        b.synchronize()
        ref_times.append(a.elapsed_time(b))
    ref_ms = statistics.median(ref_times)
    ref_gbs = nbytes / (ref_ms * 1e-3) / 1e9
    del src_, dst_
    # end to end: the op's inputs from pinned host memory, then the op (one stream)
    hk = torch.from_numpy(case.key.view(np.int16)).view(tdt).pin_memory()
    hv = torch.from_numpy(case.value.view(np.int16)).view(tdt).pin_memory()
    hs = torch.from_numpy(case.slot_mapping).pin_memory()
    hp = pairs.cpu().pin_memory()
    e2e_n = max(1, min(args.steps, 50))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_n):
        if args.op == "kv_write":
            key.copy_(hk, non_blocking=True)
            val.copy_(hv, non_blocking=True)
            sm.copy_(hs, non_blocking=True)
        else:
            pairs.copy_(hp, non_blocking=True)
        fn()
    e1.record()
    torch.cuda.synchronize()
    h2d = (hk.numel() * 2 + hv.numel() * 2 + hs.numel() * 8) if args.op == "kv_write" else hp.numel() * 8
    peak, peak_kind = peaks()
    # CPU oracle of the same op on the host cores
    import oracle
    kh, vh = case.k_cache.copy(), case.v_cache.copy()
    t0 = time.perf_counter()
    reps = 0
    while time.perf_counter() - t0 < min(args.cpu_budget, 5.0) or reps == 0:
        if args.op == "kv_write":
            oracle.kv_write(case.key, case.value, case.slot_mapping, kh, vh)
        else:
            oracle.copy_blocks(kh, vh, case.copy_pairs)
        reps += 1
    cpu_s = (time.perf_counter() - t0) / reps
    return {
        "metric": f"pa_{args.op} GB/s (algorithmic bytes read + written)",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": case.dtype, "data": "synthetic",
        "config": {"workload": desc, "op": what, "bytes_per_call": nbytes,
                   "l2": "flushed (256 MB read) before every timed call; median of the calls"},
        "e2e": {"value": round(nbytes * e2e_n / (e0.elapsed_time(e1) * 1e-3) / 1e9, 2),
                "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 0},
        "gpu_launches": args.steps,
        "roofline": {"bound": "hbm", "achieved": round(value, 2), "peak": peak,
                     "peak_kind": f"{peak_kind} HBM copy GB/s", "unit": "GB/s",
                     "frac": round(value / peak, 4), "kernel": f"pa_{args.op}", "traffic": None,
                     "size_matched": {"what": "one contiguous device-to-device copy of the same "
                                              "bytes (torch copy_), same flush and statistic",
                                      "us": round(ref_ms * 1e3, 2), "gbs": round(ref_gbs, 2),
                                      "ratio": round(value / ref_gbs, 4)}},
        "clocks": clocks,
        "cpu_baseline": {"value": round(nbytes / cpu_s / 1e9, 4), "unit": "GB/s", "cores": 1,
                         "kind": "oracle", "sample": f"the whole op, {reps} repetitions"},
    }


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return None
    import oracle
    from workloads import make_config
    name, kw, desc = WORKLOADS[args.workload]
    case = make_config(name, poison=False, **kw)
    prepare_oracle(case)
    nthreads = oracle.max_threads()
    rng = np.random.default_rng(0)
    all_sel = np.array([(s, h) for s in range(case.num_seqs) for h in range(case.num_q_heads)],
                       np.int32)
    # size each step's sample so the whole run stays near `budget` seconds
    probe = all_sel[rng.permutation(len(all_sel))[:64]]
    t_probe = oracle_step_time(case, probe, nthreads) / len(probe)
    per_step = args.reference_budget / max(1, args.steps + args.warmup)
    n = int(max(1, min(len(all_sel), per_step / max(t_probe, 1e-9))))
    sels = [all_sel[rng.permutation(len(all_sel))[:n]] for _ in range(args.steps)]
    for _ in range(args.warmup):
        oracle_step_time(case, sels[0], nthreads)
    tot_t, tot_b = 0.0, 0
    for sel in sels:
        tot_t += oracle_step_time(case, sel, nthreads)
        tot_b += sel_bytes(case, sel)
    value = tot_b / tot_t / 1e9
    sample = (f"{n} of {len(all_sel)} (seq, q head) pairs per step, seeded; fp64 C oracle "
              f"with OpenMP ({nthreads} threads)")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(tot_t / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(case, desc, ws),
            "plan": {"step": "fp64 CPU oracle of the step's attention outputs"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": nthreads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(PREFILL_WORKLOADS),
                    default=None)
    ap.add_argument("--partition-size", type=int, default=0)
    ap.add_argument("--seqs", type=int, default=0,
                    help="profiling only: build the workload with this many sequences")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--roofline-s", type=float, default=ROOF_MIN_S,
                    help="minimum device seconds of each roofline pass (at least "
                         f"{ROOF_MIN_GROUPS * ROOF_GROUP} calls either way)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip timing the other Llama-shaped workloads after the headline one")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--reference-budget", type=float, default=60.0)
    ap.add_argument("--op", choices=["step", "swap", "prefill", "kv_write", "copy_blocks"],
                    default="step",
                    help="swap: time the preemption swap of the workload instead of the step; "
                         "prefill: the prefill / chunked-prefill step (--workload prefill_*)")
    ap.add_argument("--cow", choices=["folded", "separate"], default="folded",
                    help="workloads with copy-on-write: copies done by the decode's own CTAs "
                         "(pa_decode_cow) or by a pa_copy_blocks launch before the step")
    ap.add_argument("--no-plan", action="store_true",
                    help="launch the full (sequence, partition) grid instead of the units "
                         "planned from the host's copy of the context lengths")
    ap.add_argument("--swap-seqs", type=int, default=8,
                    help="swap: number of sequences preempted and restored per step")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload is None:
        args.workload = "prefill_2k_gqa" if args.op == "prefill" else "llama2_7b"
    if args.op in ("kv_write", "copy_blocks"):
        if args.workload is None or (args.op == "copy_blocks" and args.workload == "llama2_7b"):
            args.workload = "prefix_cow" if args.op == "copy_blocks" else args.workload
        res = run_cache_op(args) if args.impl == "ours" else None
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if (args.op == "prefill") != (args.workload in PREFILL_WORKLOADS):
        ap.error("prefill workloads go with --op prefill, the others with --op step/swap")
    if args.op == "prefill":
        res = run_prefill(args)
    elif args.op == "swap":
        res = run_swap(args) if args.impl == "ours" else None
    else:
        res = run_reference(args) if args.impl == "reference" else run_ours(args)
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
