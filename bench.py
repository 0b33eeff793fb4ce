#!/usr/bin/env python3
"""Decode-step benchmark: sparse mixed-precision paged decode attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c1] [--impl kvq|reference]
                    [--path calls|three|two|fused] [--score mean|quad] [--coverage C]
                    [--tier T] [--host-tiers M] [--demote T]

One step = one decode step of one attention layer for the whole batch, all of it in
libkvq kernels: append the new token (quantise + pack + summary), score every page,
select top-k + sink + recent pages, sparse split-K attention + log-sum-exp combine.
``--path calls`` (default) runs it as the four calls kvq_append -> kvq_page_scores ->
kvq_select_topk -> kvq_sparse_decode_attn; ``--path fused`` as the single
kvq_decode_step launch.

Timing: W untimed steps, then K steps replayed from a CUDA graph of the step and timed
on the device with CUDA events on the launching stream around each replay.  Before every
timed step, outside the events, L2 is flushed: a 512 MiB buffer is written (every L2 line
replaced), then a 256 MiB buffer is read, so that the dirty lines of that write are
written back before the step starts and L2 holds no line of the step's data and no
dirty line (a decode loop enters a layer's step with L2 holding other layers' clean
lines, not a backlog of write-backs).  The same steps after the write alone are reported
as ``ms_per_step_write_only_flush``.
Per-kernel durations come from a second graph of the same step with events between the
calls, replayed right after the timed loop.  The whole-step time is bracketed by a barrier + synchronize; with N > 1
(torchrun, one process per GPU, NCCL) every rank runs its own independent batch (weak
scaling: sequences are independent problems, no collective on the data path) and the
max time over ranks is used.  Rank 0 prints one JSON line.

Options: ``--score quad`` scores pages with the quad (Gaussian-MGF) score; ``--coverage``
selects by page-mass coverage; ``--tier T`` stores every prefilled page at tier T;
``--host-tiers M`` keeps the pools of mask M in pinned host memory and ``--host-v-tiers M``
only their V chunks, K staying on the device (the line gains a ``host_link`` object); ``--demote T`` also times kvq_requantize_pages moving the
workload's pages to tier T (a ``demotion`` object).

``--impl reference`` times the CPU oracle (the plain fp64 restatement of the method)
on the host cores on a bounded sample of the same workload and prints the same line.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-step attn tokens/s and achieved HBM GB/s (% of roofline), 1×B200"

DESCR = {
    "c0": "tiny: 1 seq, 8 q / 2 kv heads, D 64, 1024 tokens, fp16, all 16-bit pages, top-8 + page 0 + last page",
    "c1": "Llama-3-8B-shaped layer: batch 8, 32 q / 8 kv heads, D 128, context 32768 (+1 appended token), "
          "bf16 pages, 5% of pages + sink + 4 recent selected per kv head",
    "c2": "c1 shape, tiers 16-bit/int8/int4/int2 = 10/20/30/40%, 10% selected, +1 appended token",
    "c3": "batch 1, 32 q / 8 kv heads, D 128, context 131072 (+1), int4 cold / 16-bit hot pages, "
          "permuted block table, 5% + sink + 16 recent",
    "c4": "ragged Qwen2.5-3B-shaped layer: batch 64, 16 q / 2 kv heads, D 128, contexts log-uniform 2k-64k, "
          "tiers 16-bit/int4/int2/1-bit = 10/30/40/20%, 8% + sink + 4 recent",
}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock / throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "50", "-i", str(self.index)], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        rows = [l.split(", ") for (t, l) in self.lines if t0 <= t <= t1 + 0.06]
        rows = [r for r in rows if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- bytes
def algorithmic_bytes(w, sel: np.ndarray, cnt: np.ndarray, tier_tbl: np.ndarray, quad_rank: int = 0):
    """Bytes the step must move: (attention, scores, select, append) per launch; with the
    quad score the scores also read r' fp16 eigenvalues per page and the append updates
    the open page's sums and eigenvalues."""
    from sparse_mixed_precision_kvq_b200.kvq import kvq_chunk_bytes
    cb = np.array([2 * kvq_chunk_bytes(t, w.D) for t in range(6)], dtype=np.int64)
    attn = 0
    for b in range(w.B):
        for g in range(w.Hkv):
            pages = sel[b, g, :cnt[b, g]]
            attn += int(cb[tier_tbl[b, pages]].sum())
    q_bytes = w.B * w.Hq * w.D * 2
    attn += q_bytes + w.B * w.Hq * w.D * 2 + int(cnt.sum()) * 4          # q, out, page list
    P = np.array([w.pages_after(b) for b in range(w.B)])
    score = int(P.sum()) * w.Hkv * (w.D + quad_rank) * 2 + q_bytes + w.B * w.Hkv * w.max_pages * 4
    select = w.B * w.Hkv * w.max_pages * 4 + int(cnt.sum()) * 4
    append = w.B * w.Hkv * w.D * 2 * 2 if w.append else 0
    if w.append and quad_rank:
        append += w.B * w.Hkv * (w.D * 2 + quad_rank * (4 * 8 + 2))  # key, sums read + written, lambda
    return dict(attn=attn, score=score, select=select, append=append)


# algorithmic bytes of each launch of a path, by the names its timing parts carry
PART_BYTES = {"append": ("append",), "page_scores": ("score",), "select_topk": ("select",),
              "sparse_decode_attn": ("attn",), "append_scores": ("score", "append"),
              "score_select": ("score", "select", "append"), "decode_step": ("attn", "score", "select", "append")}


def kernel_rooflines(names, avg_ms, nbytes, peak: float):
    """Per launch of the step: algorithmic bytes, GB/s over its event-timed duration, and
    the fraction of the HBM peak."""
    out = {}
    for n, ms in zip(names, avg_ms):
        b = sum(nbytes[k] for k in PART_BYTES[n])
        gbs = b / (ms * 1e-3) / 1e9 if ms > 0 else 0.0
        out[n] = {"bytes": int(b), "ms": float(ms), "gbs": gbs, "frac": gbs / peak}
    return out


def kernel_source_hash(kernel_file: str) -> str:
    """First 16 hex digits of the SHA-256 of a kernel's translation unit: the .cu file and
    every header of the package it includes, directly or not, in a fixed order."""
    import re
    csrc = os.path.join(ROOT, "sparse_mixed_precision_kvq_b200", "csrc")
    seen, order = set(), []

    def visit(name):
        if name in seen or not os.path.exists(os.path.join(csrc, name)):
            return
        seen.add(name)
        order.append(name)
        with open(os.path.join(csrc, name)) as f:
            for inc in re.findall(r'^#include "([^"]+)"', f.read(), re.M):
                visit(inc)

    visit(kernel_file)
    h = hashlib.sha256()
    for name in order:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def kernel_traffic(kernel_file: str, workload):
    """ncu DRAM bytes per launch recorded for the current source of a kernel (its file and
    the headers it includes) on `workload` (a plain run of that workload: its own budget
    selection, mean-key scores, device pools), else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if workload is None or not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_file)
    if not e or e.get("source_sha256_16") != kernel_source_hash(kernel_file) or e.get("workload") != workload:
        return None
    return e


# ----------------------------------------------------------------------------- ranks
def rank_workload(config: str, rank: int, batch=None, tier=None):
    """Rank r's batch: the workload's shapes with its own seeds (independent sequences per
    rank: weak scaling, nothing exchanged on the data path).  ``tier`` stores every
    prefilled page at that tier instead of the workload's mix."""
    from sparse_mixed_precision_kvq_b200 import workloads as W
    base = W.make(config)
    over = {} if batch is None else dict(B=batch)
    if tier is not None:
        over.update(tier_fracs={int(tier): 1.0}, hot_f16_planted=False)
    if batch is not None and config != "c4":
        over["lens"] = np.resize(base.lens, batch)
    return W.make(config, seed=base.seed + 1000 * rank, **over)


def max_over_ranks(x: float, device) -> float:
    """The largest x over all ranks of the process group (plain value with one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- GPU arm
PATHS = {"fused": "kvq_decode_step (one persistent launch)",
         "two": "kvq_score_select -> kvq_sparse_decode_attn",
         "three": "kvq_append_scores -> kvq_select_topk -> kvq_sparse_decode_attn",
         "calls": "kvq_append -> kvq_page_scores -> kvq_select_topk -> kvq_sparse_decode_attn"}


def step_parts(step, path: str):
    """The launches of one step of ``path``, in order, as (name, callable) pairs."""
    return {"fused": [("decode_step", step.run_fused)],
            "two": [("score_select", step.score_select), ("sparse_decode_attn", step.attend)],
            "three": [("append_scores", step.append_scores), ("select_topk", step.select),
                      ("sparse_decode_attn", step.attend)],
            "calls": [("append", step.append), ("page_scores", step.scores_), ("select_topk", step.select),
                      ("sparse_decode_attn", step.attend)]}[path]


def dominant_bytes(path: str, nbytes: dict, dom: int) -> int:
    if path == "fused":
        return nbytes["attn"] + nbytes["score"] + nbytes["select"] + nbytes["append"]
    if path == "two":
        return [nbytes["score"] + nbytes["select"] + nbytes["append"], nbytes["attn"]][dom]
    if path == "three":
        return [nbytes["score"] + nbytes["append"], nbytes["select"], nbytes["attn"]][dom]
    return [nbytes["append"], nbytes["score"], nbytes["select"], nbytes["attn"]][dom]


def kernel_files(path: str, quad: bool):
    sc = "quad.cu" if quad else "score.cu"
    return {"fused": ["step.cu"], "two": ["score.cu", "attn.cu"], "three": [sc, "select.cu", "attn.cu"],
            "calls": ["append.cu", sc, "select.cu", "attn.cu"]}[path]


class L2Flush:
    """The L2 flush between timed steps: ``fill_(v)`` writes the whole write buffer (more
    than L2), then reads the read buffer (more than L2), evicting the write's dirty lines;
    ``write_only(v)`` does the write alone."""

    def __init__(self, mib: int, dev):
        import torch
        self.w = torch.empty(mib << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones(max(mib // 2, 160) << 18, dtype=torch.float32, device=dev)

    def fill_(self, v: int):
        self.w.fill_(v)
        self.r.amax()

    def write_only(self, v: int):
        self.w.fill_(v)


def measure(w, cache, step, path: str, K: int, warmup: int, flush, stream, dev, world: int, peak: float,
            quad_rank: int = 0, soak_s: float = 0.0, e2e: bool = True, eager: bool = True):
    """Time one workload's decode step on this rank.

    step time: K replays of a CUDA graph of the step, each after an L2 flush (outside the
    events), timed with CUDA events around each replay, summed and maxed over ranks;
    kernels: a second graph with events between the launches; eager: the same launches
    issued directly (no graph); e2e: the graph with the step's host inputs copied in and
    its outputs copied back inside the events.  ``soak_s`` seconds of further replays
    follow the timed ones, so that the clock sampler running meanwhile has a record longer
    than the timed steps themselves."""
    import torch
    import torch.distributed as dist
    parts = step_parts(step, path)
    run_step = {"fused": step.run_fused, "two": step.run_two, "three": step.run_three, "calls": step.run}[path]
    for _ in range(warmup):
        flush.fill_(1)
        run_step()
    torch.cuda.synchronize(dev)
    assert cache.err_bits() == 0, f"device error bits {cache.err_bits():#x}"
    tier_tbl, _, _ = w.slot_map()
    sel, cnt = step.sel.cpu().numpy(), step.cnt.cpu().numpy()
    nbytes = algorithmic_bytes(w, sel, cnt, tier_tbl, quad_rank)
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        run_step()
    stream.wait_stream(side)
    torch.cuda.synchronize(dev)
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        run_step()
    pev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(parts) + 1)]
    g_prof = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_prof):
        cs = torch.cuda.current_stream()
        pev[0].record(cs)
        for i, (_, fn) in enumerate(parts):
            fn()
            pev[i + 1].record(cs)
    for _ in range(3):
        flush.fill_(1)
        g_step.replay()
        g_prof.replay()
    torch.cuda.synchronize(dev)
    assert cache.err_bits() == 0, f"device error bits {cache.err_bits():#x}"

    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0 = time.time()
    for k in range(K):
        flush.fill_(k & 0xFF)
        e0[k].record(stream)
        g_step.replay()
        e1[k].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    t1 = time.time()
    soak = 0
    while time.time() - t1 < soak_s:   # the same replays, back to back, for the clock record
        for _ in range(200):
            flush.fill_(soak & 0xFF)
            g_step.replay()
            soak += 1
        torch.cuda.synchronize(dev)
    t2 = time.time()
    KP = min(K, 300)
    per = np.zeros((KP, len(parts)))
    for k in range(KP):
        flush.fill_(k & 0xFF)
        g_prof.replay()
        torch.cuda.synchronize(dev)
        per[k] = [pev[i].elapsed_time(pev[i + 1]) for i in range(len(parts))]
    step_ms = np.array([e0[k].elapsed_time(e1[k]) for k in range(K)])
    total_ms = max_over_ranks(float(step_ms.sum()), dev)
    ms_per_step = total_ms / K
    KD = min(K, 300)  # the same replays after the write alone (L2 left full of dirty lines)
    d0 = [torch.cuda.Event(enable_timing=True) for _ in range(KD)]
    d1 = [torch.cuda.Event(enable_timing=True) for _ in range(KD)]
    for k in range(KD):
        flush.write_only(k & 0xFF)
        d0[k].record(stream)
        g_step.replay()
        d1[k].record(stream)
    torch.cuda.synchronize(dev)
    ms_dirty = max_over_ranks(float(np.mean([d0[k].elapsed_time(d1[k]) for k in range(KD)])), dev)

    out = {"ms_per_step": ms_per_step, "tokens_per_s": world * w.B * K / (total_ms / 1e3),
           "nbytes": nbytes, "sel": sel, "cnt": cnt, "tier_tbl": tier_tbl, "names": [n for n, _ in parts],
           "kernel_ms": per.mean(0), "clock_window": (t0, t2), "soak_steps": soak,
           "ms_per_step_write_only_flush": ms_dirty}
    if eager:
        KE = max(1, min(K, 200))
        a = [torch.cuda.Event(enable_timing=True) for _ in range(KE)]
        b_ = [torch.cuda.Event(enable_timing=True) for _ in range(KE)]
        for k in range(KE):
            flush.fill_(k & 0xFF)
            a[k].record(stream)
            run_step()
            b_[k].record(stream)
        torch.cuda.synchronize(dev)
        out["ms_per_step_eager"] = max_over_ranks(float(np.mean([a[k].elapsed_time(b_[k]) for k in range(KE)])), dev)
    if e2e:
        # the step's inputs (q, k_new, v_new: one packed buffer) copied in from pinned host
        # memory and its outputs (out, lse: one packed buffer) copied back, in one graph with
        # the step's calls
        pin_in = torch.empty_like(step.io_in, device="cpu").pin_memory()
        pin_in.copy_(step.io_in)
        pin_out = torch.empty_like(step.io_out, device="cpu").pin_memory()
        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e):
            step.io_in.copy_(pin_in, non_blocking=True)
            run_step()
            pin_out.copy_(step.io_out, non_blocking=True)
        KE = max(1, min(K, 500))
        es = [torch.cuda.Event(enable_timing=True) for _ in range(KE)]
        ee = [torch.cuda.Event(enable_timing=True) for _ in range(KE)]
        for k in range(KE):
            flush.fill_(k & 0xFF)
            es[k].record(stream)
            g_e2e.replay()
            ee[k].record(stream)
        torch.cuda.synchronize(dev)
        del g_e2e
        e2e_ms = max_over_ranks(float(np.mean([es[k].elapsed_time(ee[k]) for k in range(KE)])), dev)
        h2d = pin_in.numel()   # bytes of the packed input buffer
        d2h = pin_out.numel()
        out["e2e"] = {"value": world * w.B / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
                      "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_ms}
    assert cache.err_bits() == 0, f"device error bits {cache.err_bits():#x}"
    del g_prof, g_step
    step_bytes = sum(nbytes[k] for k in ("attn", "score", "select", "append"))
    out["step_hbm"] = {"bytes": step_bytes, "achieved_gbs": step_bytes / (ms_per_step * 1e-3) / 1e9,
                       "peak_gbs": peak, "frac": step_bytes / (ms_per_step * 1e-3) / 1e9 / peak}
    out["kernels_roofline"] = kernel_rooflines(out["names"], out["kernel_ms"], nbytes, peak)
    return out


def config_summary(name: str, w, m: dict, peak: float, dense_ms=None) -> dict:
    """The per-workload object of the JSON line (other workloads than the headline one)."""
    kr = m["kernels_roofline"]
    d = {"workload": f"{name}: {DESCR[name]}", "batch": w.B, "context_max": int(w.lens.max()),
         "selected_pages": int(m["cnt"].sum()), "ms_per_step": m["ms_per_step"], "tokens_per_s": m["tokens_per_s"],
         "ms_per_step_eager": m.get("ms_per_step_eager"),
         "ms_per_step_write_only_flush": m.get("ms_per_step_write_only_flush"), "step_hbm": m["step_hbm"],
         "kernels_ms": {n: float(a) for n, a in zip(m["names"], m["kernel_ms"])},
         "attention_roofline": kr.get("sparse_decode_attn") or kr.get("decode_step"),
         "e2e": m.get("e2e")}
    if dense_ms is not None:
        dense_bytes = dense_attn_bytes(w)
        d["dense_all_pages"] = {"ms": dense_ms, "bytes": dense_bytes,
                                "achieved_gbs": dense_bytes / (dense_ms * 1e-3) / 1e9,
                                "frac": dense_bytes / (dense_ms * 1e-3) / 1e9 / peak,
                                "speedup_of_sparse_step": dense_ms / m["ms_per_step"]}
    return d


def dense_attn_bytes(w) -> int:
    """Attention over every page: all K+V chunks of every (sequence, kv head) + q + out."""
    from sparse_mixed_precision_kvq_b200.kvq import kvq_chunk_bytes
    tier_tbl, _, _ = w.slot_map()
    cb = np.array([2 * kvq_chunk_bytes(t, w.D) for t in range(6)], dtype=np.int64)
    tot = 0
    for b in range(w.B):
        P = w.pages_after(b)
        tot += int(cb[tier_tbl[b, :P]].sum()) * w.Hkv + P * w.Hkv * 4
    return tot + 2 * w.B * w.Hq * w.D * 2


def run_kvq(args, rank: int, world: int, local_rank: int):
    import torch
    from sparse_mixed_precision_kvq_b200 import kvq

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peak, peak_kind = load_peaks()
    flush = L2Flush(args.flush_mib, dev)
    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local_rank)).split(",")[0])
                          if os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")[0].isdigit() else local_rank)
    if rank == 0:
        clocks.start()
        time.sleep(1.0)  # let nvidia-smi start sampling

    w = rank_workload(args.config, rank, args.batch, args.tier)
    quad_rank = args.quad_rank if args.score == "quad" else 0
    basis = None
    if quad_rank:
        basis = np.stack([w.quad_basis(g, quad_rank, "law") for g in range(w.Hkv)])
    cache = kvq.cache_from_workload(w, device=dev, quad_basis=basis, host_tiers=args.host_tiers,
                                    host_v_tiers=args.host_v_tiers)
    step = kvq.DecodeStep(w, cache, device=dev, coverage=args.coverage, quad=bool(quad_rank))
    m = measure(w, cache, step, args.path, args.steps, args.warmup, flush, stream, dev, world, peak,
                quad_rank=quad_rank, soak_s=args.soak_s if rank == 0 else 0.0)
    cw = m["clock_window"]
    dense_ms = None
    if args.dense and not args.no_dense and rank == 0:
        dense_ms = time_dense(w, cache, step, flush, stream, dev)
    names, avg, nbytes = m["names"], m["kernel_ms"], m["nbytes"]
    dom = int(np.argmax(avg))
    dom_bytes = dominant_bytes(args.path, nbytes, dom)
    files = kernel_files(args.path, bool(quad_rank))
    achieved = dom_bytes / (avg[dom] * 1e-3) / 1e9
    plain = (args.coverage is None and args.tier is None and not args.host_tiers and not args.host_v_tiers
             and args.score == "mean" and args.batch is None)
    tr = kernel_traffic(files[dom], args.config if plain else None)
    sel, cnt, tier_tbl = m["sel"], m["cnt"], m["tier_tbl"]
    host = None
    if args.host_tiers or args.host_v_tiers:
        host = host_link(w, sel, cnt, tier_tbl, args.host_tiers, avg[names.index("sparse_decode_attn")]
                         if "sparse_decode_attn" in names else None, dev, vmask=args.host_v_tiers)
    demotion = None
    if args.demote is not None:
        del step, cache
        demotion = time_demotion(w, args.demote, flush, stream, dev, peak, peak_kind)
    else:
        del step, cache
    torch.cuda.empty_cache()

    # the other workloads, same path, default options (each rank its own batch)
    configs = {}
    for name in [c for c in args.configs.split(",") if c and c != args.config] if args.configs != "none" else []:
        wc = rank_workload(name, rank)
        cc = kvq.cache_from_workload(wc, device=dev)
        sc = kvq.DecodeStep(wc, cc, device=dev)
        mc = measure(wc, cc, sc, args.path, args.steps, args.warmup, flush, stream, dev, world, peak)
        configs[name] = config_summary(name, wc, mc, peak)
        del sc, cc
        torch.cuda.empty_cache()
    clocks.stop()
    if rank != 0:
        return None
    line = {
        "metric": METRIC,
        "value": m["tokens_per_s"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": m["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f16",
        "data": "synthetic (seeded; shapes and value laws of the workload; no model weights)",
        "config": {"workload": f"{args.config}: {DESCR[args.config]}", "batch_per_gpu": w.B,
                   "context": int(w.lens.max()), "kv_heads": w.Hkv, "q_heads": w.Hq, "head_dim": w.D,
                   "selected_pages": int(cnt.sum()),
                   "selection": "budget" if args.coverage is None else f"coverage {args.coverage}",
                   "tiers": "the workload's" if args.tier is None else f"every prefilled page at tier {args.tier}",
                   "host_tiers": args.host_tiers, "host_v_tiers": args.host_v_tiers,
                   "page_score": "mean-key" if not quad_rank else
                   f"quad (rank {quad_rank}, basis: eigenvectors of the key law's covariance)",
                   "l2": f"flushed before every timed step: {args.flush_mib} MiB written, then "
                         f"{flush.r.numel() * 4 >> 20} MiB read (no line of the step's data and no dirty "
                         f"line in L2); ms_per_step_write_only_flush: the same steps after the write alone",
                   "parallelism": f"replicas x{world} (independent batches)"},
        "step_hbm": dict(m["step_hbm"], peak_kind=peak_kind),
        "ms_per_step_eager": m.get("ms_per_step_eager"),
        "ms_per_step_write_only_flush": m.get("ms_per_step_write_only_flush"),
        "kernels_ms": {n: float(a) for n, a in zip(names, avg)},
        "kernels_roofline": m["kernels_roofline"],
        "roofline": {"bound": "hbm", "kernel": names[dom], "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)",
                     "algorithmic_bytes_per_launch": dom_bytes,
                     "traffic": None if tr is None else tr["dram_bytes_per_launch"]},
        "e2e": m["e2e"],
        "gpu_launches": (len(names) + (1 if quad_rank and w.append and args.path == "calls" else 0)) * args.steps,
        "path": PATHS[args.path],
        "timing": "step: CUDA-graph replay of the step timed with events around each replay; "
                  "kernels_ms: a second graph with events between the launches (no launch overlap); "
                  "ms_per_step_eager: the same launches issued without a graph",
        "clocks": dict(clocks.summary(cw[0], cw[1]),
                       window=f"the {args.steps} timed steps and {m['soak_steps']} more replays of the same step "
                              f"right after them ({args.soak_s:.1f} s)"),
    }
    if dense_ms is not None:
        dense_bytes = dense_attn_bytes(w)
        line["dense_all_pages"] = {"op": "kvq_sparse_decode_attn over every page of every (sequence, kv head)",
                                   "ms": dense_ms, "bytes": dense_bytes,
                                   "achieved_gbs": dense_bytes / (dense_ms * 1e-3) / 1e9,
                                   "frac": dense_bytes / (dense_ms * 1e-3) / 1e9 / peak,
                                   "sparse_step_speedup": dense_ms / m["ms_per_step"]}
    if configs:
        line["configs"] = configs
    if host is not None:
        line["host_link"] = host
    if demotion is not None:
        line["demotion"] = demotion
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_seconds or 12.0, config=args.config, seed_rank=rank,
                                            batch=args.batch, tier=args.tier)
    return line


def time_dense(w, cache, step, flush, stream, dev, reps=20):
    """Attention over every page of every (sequence, kv head), L2 flushed, events around
    each launch (c1's dense reference point)."""
    import torch
    from sparse_mixed_precision_kvq_b200 import kvq
    P = np.array([w.pages_after(b) for b in range(w.B)])
    kmax = int(P.max())
    sel = np.zeros((w.B, w.Hkv, kmax), dtype=np.int32)
    for b in range(w.B):
        sel[b, :, :P[b]] = np.arange(P[b])
    sel_t = torch.from_numpy(sel).to(dev)
    cnt_t = torch.from_numpy(np.repeat(P[:, None], w.Hkv, 1).astype(np.int32)).to(dev)
    ws = torch.empty(kvq.kvq_workspace_size(cache, kmax) // 4 + 4, dtype=torch.float32, device=dev)
    kvq.kvq_workspace_init(ws)
    out = torch.empty_like(step.out)
    ts = []
    for r in range(reps + 3):
        flush.fill_(r & 0xFF)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        kvq.kvq_sparse_decode_attn(cache, step.q, sel_t, cnt_t, kmax, w.sm_scale, out, None, ws)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        if r >= 3:
            ts.append(a.elapsed_time(b_))
    assert cache.err_bits() == 0, f"device error bits {cache.err_bits():#x}"
    return float(np.mean(ts))


def host_link(w, sel, cnt, tier_tbl, mask: int, attn_ms, dev, reps: int = 5, vmask: int = 0):
    """The attention's bytes read from pinned host memory (K and V chunks of the pools in
    ``mask``, V chunks of the V pools in ``vmask``), their rate over the kernel's
    event-timed duration, against a pinned host -> device copy of 512 MiB timed here."""
    import torch
    from sparse_mixed_precision_kvq_b200.kvq import kvq_chunk_bytes
    cb = np.array([kvq_chunk_bytes(t, w.D) for t in range(6)], dtype=np.int64)
    host = 0
    for b in range(w.B):
        for g in range(w.Hkv):
            for t in tier_tbl[b, sel[b, g, :cnt[b, g]]]:
                t = int(t)
                host += int(2 * cb[t] if (mask >> t) & 1 else (cb[t] if (vmask >> t) & 1 else 0))
    src = torch.empty(512 << 20, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    ts = []
    for r in range(reps + 1):
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        dst.copy_(src, non_blocking=True)
        b_.record()
        torch.cuda.synchronize(dev)
        if r:
            ts.append(a.elapsed_time(b_))
    peak = (512 << 20) / (np.mean(ts) * 1e-3) / 1e9
    out = {"mask": mask, "v_mask": vmask, "attn_host_bytes": host, "h2d_copy_gbs": peak,
           "peak_kind": "pinned host -> device copy of 512 MiB, timed in this run"}
    if attn_ms:
        out.update(achieved_gbs=host / (attn_ms * 1e-3) / 1e9, frac=host / (attn_ms * 1e-3) / 1e9 / peak)
    return out


CASCADE = [0, 5, 1, 2, 3, 4]  # tiers from hot to cold: 16-bit, fp8, int8, int4, int2, 1-bit


def time_demotion(w, tier: int, flush, stream, dev, peak: float, peak_kind: str, reps: int = 20):
    """kvq_requantize_pages over every prefilled page outside the sink and recent windows
    whose tier is hotter than ``tier``, into spare slots of a fresh cache (the block table is
    put back, outside the timed region, before every repetition)."""
    import torch
    from sparse_mixed_precision_kvq_b200 import kvq
    tier_tbl, _, counts = w.slot_map()
    items = []
    nxt = list(counts)
    for b in range(w.B):
        P0 = w.pages_before(b)
        for p in range(w.n_sink, P0 - w.n_recent):
            if CASCADE.index(int(tier_tbl[b, p])) < CASCADE.index(tier):  # hotter than the target
                items.append((b, p, int(np.uint32((tier << 29) | nxt[tier]).view(np.int32))))
                nxt[tier] += 1
    spare = [n - c for n, c in zip(nxt, counts)]
    cache = kvq.cache_from_workload(w, device=dev, spare=spare)
    it = torch.tensor(items, dtype=torch.int32, device=dev)
    bt0 = cache.block_table.clone()
    cb = np.array([2 * kvq.kvq_chunk_bytes(t, w.D) for t in range(6)], dtype=np.int64)
    src = np.array([tier_tbl[b, p] for b, p, _ in items], dtype=np.int64)
    nbytes = int(w.Hkv * (cb[src].sum() + len(items) * cb[tier])) + len(items) * (12 + 8)
    ts = []
    for r in range(reps + 3):
        cache.block_table.copy_(bt0)
        flush.fill_(r & 0xFF)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        kvq.kvq_requantize_pages(cache, it)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        if r >= 3:
            ts.append(a.elapsed_time(b_))
    assert cache.err_bits() == 0, f"device error bits {cache.err_bits():#x}"
    ms = float(np.mean(ts))
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"op": "kvq_requantize_pages (re-encode + block-table switch: two launches)",
            "pages": len(items), "kv_heads": w.Hkv, "to_tier": tier,
            "from_tiers": {int(t): int((src == t).sum()) for t in np.unique(src)},
            "ms": ms, "bytes": nbytes, "pages_per_s": len(items) / (ms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "peak_kind": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)"}}


# ----------------------------------------------------------------------------- CPU oracle
def _oracle_units(config: str, seed_rank: int, units, budget_s: float, batch=None, tier=None):
    """Worker: prepare the listed (b, g) units of the workload (untimed), then run the
    oracle's decode step on them round-robin for ``budget_s`` seconds, numpy/BLAS on one
    thread.  Returns (unit steps run, seconds spent in them)."""
    from threadpoolctl import threadpool_limits
    from oracle.fp import bits16_to_f64
    from oracle.step import prepare, step_pair
    w = rank_workload(config, seed_rank, batch, tier)
    q = bits16_to_f64(w.query_bits(), w.dtype)
    kn, vn = w.new_kv_bits() if w.append else (None, None)
    with threadpool_limits(limits=1):
        prepared = [(b, g, prepare(w, b, g)) for b, g in units]
        saved = [(sh.L, sh.ksum.copy()) for _, _, sh in prepared]
        n, spent = 0, 0.0
        while spent < budget_s and n < 100000:
            for (b, g, sh), (L0, ks0) in zip(prepared, saved):
                t0 = time.perf_counter()
                step_pair(w, sh, b, g, q[b], None if kn is None else kn[b, g], None if vn is None else vn[b, g])
                spent += time.perf_counter() - t0
                n += 1
                sh.L, sh.ksum = L0, ks0.copy()   # undo the append so the next step repeats it
    return n, spent


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w, budget_s: float = 12.0, config: str = "c1", seed_rank: int = 0, all_cores: bool = True,
                 batch=None, tier=None):
    """The oracle's decode step timed on the host cores, on a bounded sample of (b, g) units.

    Cache construction (the oracle's quantise/pack of the prefilled context) is excluded;
    each timed unit is the oracle step of one (sequence, kv head): append, score, select,
    attention of its G query heads.  tokens/s = B / (B * Hkv / unit steps per second).
    One thread: 4 units in one process.  All cores: one spawned worker process per core
    (up to one per unit), each on its own unit(s), its rate summed over the workers."""
    pairs = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    rng = np.random.default_rng(0)
    order = [pairs[i] for i in rng.permutation(len(pairs))]
    n1, t1 = _oracle_units(config, seed_rank, order[:4], budget_s, batch, tier)
    rate1 = n1 / t1
    res = {"value": w.B / (w.B * w.Hkv / rate1), "unit": "tokens/s", "cores": 1, "kind": "oracle",
           "cpu_model": cpu_model(), "nproc": os.cpu_count(),
           "sample": f"{n1} timed oracle steps of single (sequence, kv head) units drawn from 4 units of the "
                     f"same workload; step time = mean unit time x {w.B * w.Hkv} units; cache construction "
                     f"excluded (the appended token is rewritten each time); numpy/BLAS on 1 thread"}
    if all_cores:
        import multiprocessing as mp
        cores = max(1, min(os.cpu_count() or 1, len(pairs), 64))
        groups = [order[i::cores] for i in range(cores)]
        groups = [g[:2] for g in groups if g]
        ctx = mp.get_context("spawn")
        with ctx.Pool(len(groups)) as pool:
            got = pool.starmap(_oracle_units, [(config, seed_rank, g, budget_s, batch, tier) for g in groups])
        rate = sum(n / t for n, t in got if t > 0)
        res["all_cores"] = {"value": w.B / (w.B * w.Hkv / rate), "unit": "tokens/s", "cores": len(groups),
                            "unit_steps": int(sum(n for n, _ in got)),
                            "sample": f"{len(groups)} spawned worker processes, one per core, each running the "
                                      f"oracle step of its own 1-2 (sequence, kv head) units for {budget_s:.0f} s "
                                      f"(numpy/BLAS on 1 thread each); rate = sum of the workers' unit rates"}
    return res


def run_reference(args, rank: int, world: int):
    """The reference arm: the oracle (the plain fp64 restatement of the method) as it
    stands, on the host cores, rank 0 only."""
    from sparse_mixed_precision_kvq_b200 import workloads as W
    if rank != 0:
        return None
    w = W.make(args.config)
    K = args.steps
    budget = args.cpu_seconds if args.cpu_seconds is not None else max(3.0, min(30.0, 90.0 / max(1, K + args.warmup)))
    base = cpu_baseline(w, budget_s=budget, config=args.config)
    best = base.get("all_cores", base)
    line = {
        "metric": METRIC, "value": best["value"], "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": 1e3 * w.B / best["value"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.config}: {DESCR[args.config]}", "batch_per_gpu": w.B,
                   "context": int(w.lens.max()), "kv_heads": w.Hkv, "q_heads": w.Hq, "head_dim": w.D},
        "impl": "reference",
        "cpu_baseline": {"value": best["value"], "unit": "tokens/s", "cores": best["cores"], "kind": "oracle",
                         "sample": best["sample"], "one_thread": base["value"], "cpu_model": base["cpu_model"],
                         "nproc": base["nproc"]},
        "e2e": {"value": best["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="c1", choices=sorted(DESCR))
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--coverage", type=float, default=None,
                    help="coverage (nucleus) selection at this mass fraction instead of the workload's budget "
                         "(four-call path only)")
    ap.add_argument("--path", default="calls", choices=["calls", "three", "two", "fused"],
                    help="the four separate calls; kvq_append_scores + select + attention; kvq_score_select + "
                         "attention; or one kvq_decode_step launch")
    ap.add_argument("--score", default="mean", choices=["mean", "quad"],
                    help="page score: the mean-key score, or the quad (Gaussian-MGF) score (--path calls or three)")
    ap.add_argument("--quad-rank", type=int, default=16, help="r' of the quad score (8, 16, 24 or 32)")
    ap.add_argument("--tier", type=int, default=None, choices=[0, 1, 2, 3, 4, 5],
                    help="store every prefilled page at this tier (0 16-bit, 1 int8, 2 int4, 3 int2, 4 1-bit, 5 fp8)")
    ap.add_argument("--host-tiers", type=int, default=0,
                    help="bit t: pool t lives in pinned host memory that the kernels read in place (DRAM value tier)")
    ap.add_argument("--host-v-tiers", type=int, default=0,
                    help="bit t: the V chunks of tier t live in their own pool in pinned host memory, the K chunks "
                         "on the device (the mem-v variant of the DRAM value tier)")
    ap.add_argument("--dense", action="store_true", default=None,
                    help="also time attention over every page (on by default for c1)")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--configs", default="c2,c3,c4",
                    help="comma-separated other workloads measured after the headline one (same path, default "
                         "options) into the line's `configs` object; 'none' skips them")
    ap.add_argument("--soak-s", type=float, default=1.5,
                    help="seconds of further step replays after the timed ones, while clocks are sampled")
    ap.add_argument("--demote", type=int, default=None, choices=[1, 2, 3, 4, 5],
                    help="also time kvq_requantize_pages moving the workload's pages outside the sink and "
                         "recent windows to this tier (1 int8, 2 int4, 3 int2, 4 1-bit, 5 fp8)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=None,
                    help="seconds of oracle steps per CPU leg (default 12; the reference arm sizes it by K + W)")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch (profiling runs)")
    ap.add_argument("--flush-mib", type=int, default=512, help="L2 flush buffer (must exceed the 126 MB L2)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.coverage is not None and args.path != "calls":
        ap.error("--coverage runs on the four-call path")
    if (args.host_tiers or args.host_v_tiers) and args.path == "fused":
        ap.error("--host-tiers / --host-v-tiers: the fused step reads adjacent device chunks only")
    if args.score == "quad" and args.path not in ("calls", "three"):
        ap.error("--score quad runs on the four-call or the three-call path")
    if args.dense is None:
        args.dense = args.config == "c1"
    special = (args.coverage is not None or args.tier is not None or args.host_tiers or args.host_v_tiers
               or args.score != "mean"
               or args.batch is not None or args.demote is not None)
    if special and args.configs == "c2,c3,c4":
        args.configs = "none"   # the other workloads are measured on plain runs only

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        if world > 1:
            import datetime
            import torch
            import torch.distributed as dist
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
        line = run_kvq(args, rank, world, local_rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if line is not None and rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
