#!/usr/bin/env python
"""Benchmark of the LSA hot path (hierarchical latent-key select + sparse attention).

Default workload: last-chunk prefill at 1M context (4096 new query tokens, 32 query
/ 8 KV heads, d=128, tree 16/16/16/4 with leaf 64, beam 8/32/32/32 -> 2048 keys per
query).  A step = select + sparse attention for the whole chunk; the index over the
cached keys is built once before timing (its time is reported as build_ms).
``--workload decode_10m`` times single-token decode steps at 10,485,760 tokens
(append one key/value row per KV head, select, attend to selection + tail).

Launch: ``python bench.py [--gpus N] [--steps K] [--warmup W]``; for N > 1 under
torchrun, every rank runs its own independent request (weak scaling) and rank 0
prints one JSON line.  ``--impl reference`` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from hierarchical_latent_key_b200 import configs  # noqa: E402

METRIC = "LSA layer queries/sec (select+attn) at 1M/10M ctx; HBM GB/s and tensor % of peak"
L2_FLUSH_BYTES = 512 << 20   # > 126 MB L2


# ---------------------------------------------------------------------------
# host helpers (also exercised by the multi-process CPU tests)
# ---------------------------------------------------------------------------

def rank_seed(base: int, rank: int) -> int:
    """Each rank serves its own request: independent synthetic inputs per rank."""
    return int(base) + 7919 * int(rank)


def aggregate(local_s: float, units_per_rank: int, world: int, reduce_max=None):
    """Whole-job throughput: all ranks' units over the slowest rank's device time."""
    t = reduce_max(local_s) if reduce_max is not None else local_s
    return world * units_per_rank / t, t


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm_gbs=j.get("hbm_gbs", 6650.0), bf16_tflops=j.get("bf16_tflops", 1590.0),
                    bf16_tflops_sustained=j.get("bf16_tflops_sustained", 1400.0), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.file = None

    def __enter__(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        self.file.flush()

    def summary(self):
        rows = []
        try:
            with open(self.file.name) as f:
                for line in f:
                    p = [x.strip() for x in line.split(",")]
                    if len(p) >= 9 and p[1].replace(".", "").isdigit():
                        rows.append(p)
        finally:
            os.unlink(self.file.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]), "reasons": reasons,
                "samples": len(rows)}


def cores_used() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# CUDA arm
# ---------------------------------------------------------------------------

class Prefill:
    """Last-chunk prefill: one step = select + attention for the whole chunk."""

    def __init__(self, cfg, dev, seed):
        from hierarchical_latent_key_b200 import lsa
        self.lsa, self.cfg, self.dev = lsa, cfg, dev
        c = cfg.case(dev, seed)
        self.K, self.V, self.W, self.Q, self.q_pos = c.K, c.V, c.W, c.Q, c.q_pos
        del c
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        self.tree = lsa.build_tree(self.K, self.W, cfg.branching, cfg.leaf, cfg.iters, seed)
        torch.cuda.synchronize(dev)
        self.build_ms = 1e3 * (time.perf_counter() - t0)
        T, Hq, d = self.Q.shape
        self.leaves = torch.empty(cfg.Hkv, T, cfg.beam[-1], dtype=torch.int32, device=dev)
        self.O = torch.empty_like(self.Q)
        self.LSE = torch.empty(T, Hq, dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        need = lsa.lsa_tree_attn_workspace_bytes(self.tree.desc, T, Hq, d, self.Q.dtype, cfg.beam[-1])
        self.ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        need = lsa.lsa_select_batched_workspace_bytes(self.tree.desc, T, cfg.beam)
        self.sel_ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        self.scale = 1.0 / math.sqrt(d)
        self.units = T
        # batched select: latents, top level, then scan, fill, score and rank per level;
        # tree attention: 3 list + 2 tensor-core passes + 2
        self.launches_per_step = 2 + 4 * (len(cfg.beam) - 1) + 7

    def select(self, Q=None):
        self.lsa.lsa_select_batched(self.tree.desc, self.tree.mem, self.Q if Q is None else Q, self.W, self.cfg.beam,
                                    self.q_pos, None, self.leaves, workspace=self.sel_ws, status=self.status)

    def attend(self, Q=None, O=None, LSE=None):
        self.lsa.lsa_tree_attn(self.tree.desc, self.tree.mem, self.Q if Q is None else Q, self.K, self.V,
                               self.leaves, self.q_pos, True, self.scale, self.O if O is None else O,
                               self.LSE if LSE is None else LSE, self.ws, self.status)

    def attn_algorithmic_bytes(self):
        """Bytes the attention must move at least: the K/V rows of every distinct selected
        leaf once, plus queries, outputs, LSE and the leaf lists."""
        d = self.Q.shape[2]
        rows = 0
        for g in range(self.cfg.Hkv):
            v = self.leaves[g]
            rows += int(torch.unique(v[v >= 0]).numel()) * self.cfg.leaf
        esz = self.Q.element_size()
        return (rows * 2 * d * esz + 2 * self.Q.numel() * esz + self.LSE.numel() * 4 + self.leaves.numel() * 4,
                rows)

    def attn_flops(self):
        T, Hq, d = self.Q.shape
        return 4.0 * T * Hq * self.cfg.K_sel * d


class Decode:
    """Single-request decode: step s appends one key and one value row per KV head at
    position n + s, selects for the new token and attends to the selection plus the dense
    tail of appended rows [n, n + s] (causal by position), all in one lsa_decode_step call
    (two kernel launches)."""

    def __init__(self, cfg, dev, seed, steps):
        from hierarchical_latent_key_b200 import lsa
        cfg = cfg.scaled(T=steps)
        self.lsa, self.cfg, self.dev = lsa, cfg, dev
        c = cfg.case(dev, seed)
        self.K, self.V, self.W, self.Q, self.q_pos = c.K, c.V, c.W, c.Q, c.q_pos
        del c
        n = cfg.n
        self.Knew = self.K[:, n:].transpose(0, 1).clone(memory_format=torch.contiguous_format)   # [steps, Hkv, d]: rows the steps append
        self.Vnew = self.V[:, n:].transpose(0, 1).clone(memory_format=torch.contiguous_format)
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        self.tree = lsa.build_tree(self.K, self.W, cfg.branching, cfg.leaf, cfg.iters, seed)
        torch.cuda.synchronize(dev)
        self.build_ms = 1e3 * (time.perf_counter() - t0)
        _, Hq, d = self.Q.shape
        self.dec = lsa.DecodeStep(self.tree, self.W, cfg.beam, self.K, Hq, steps)
        self.O, self.LSE, self.status = self.dec.O, self.dec.LSE, self.dec.status
        self.launches_per_step = 2      # select (with the append), attention (with the split merge)

    def step(self, s, Q=None):
        n = self.cfg.n
        self.dec.step(self.K, self.V, self.Q[s:s + 1] if Q is None else Q, self.Knew[s], self.Vnew[s], n + s, n)

    def capture(self, steps):
        """One CUDA graph per decode step: a step is then one graph launch."""
        self.graphs = []
        for s in range(steps):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self.step(s)
            self.graphs.append(g)
        torch.cuda.synchronize()

    def bytes_per_step(self, s):
        """Algorithmic bytes of one step: gathered K/V rows of the selection and the tail,
        centroid rows scored, projection, query/output, leaf lists and the appended rows."""
        cfg, d = self.cfg, self.Q.shape[2]
        esz = self.Q.element_size()
        attn = cfg.Hkv * (cfg.K_sel + s + 1) * 2 * d * esz + 2 * cfg.Hq * d * esz + cfg.Hkv * cfg.K_sel * 4
        cand = cfg.nodes[0] + sum(cfg.beam[l - 1] * cfg.branching[l] for l in range(1, len(cfg.branching)))
        sel = (cfg.Hkv * cand * (cfg.r * 4 + 4) + cfg.Hkv * d * cfg.r * esz + cfg.Hq * d * esz
               + 2 * cfg.Hkv * d * esz)
        return attn, sel


def time_decode(w, steps, warmup, flush, stream):
    """Per step: one graph replay (append + select + attention), L2 flushed between steps."""
    for s in range(warmup):
        w.graphs[s].replay()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for k in range(steps):
        flush.zero_()
        ev[k][0].record(stream)
        w.graphs[warmup + k].replay()
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    return [ev[k][0].elapsed_time(ev[k][1]) for k in range(steps)]


def time_decode_e2e(w, steps, warmup, flush, stream):
    """Decode steps through the public API from pinned host buffers: H2D of the token's
    query and its new key/value rows into the step's input slots, the step's graph
    (append + select + attention), D2H of O and LSE."""
    first = warmup
    Qh = w.Q[first:first + steps].cpu().pin_memory()
    Kh = w.Knew[first:first + steps].cpu().pin_memory()
    Vh = w.Vnew[first:first + steps].cpu().pin_memory()
    Oh = torch.empty((steps,) + tuple(w.O.shape[1:]), dtype=w.O.dtype).pin_memory()
    Lh = torch.empty((steps,) + tuple(w.LSE.shape[1:]), dtype=torch.float32).pin_memory()
    times = []
    for k in range(steps):
        s = first + k
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        w.Q[s:s + 1].copy_(Qh[k:k + 1], non_blocking=True)
        w.Knew[s].copy_(Kh[k], non_blocking=True)
        w.Vnew[s].copy_(Vh[k], non_blocking=True)
        w.graphs[s].replay()
        Oh[k].copy_(w.O[0], non_blocking=True)
        Lh[k].copy_(w.LSE[0], non_blocking=True)
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize()
    t = [a.elapsed_time(b) for a, b in times]
    h2d = Qh[0].numel() * Qh.element_size() + 2 * Kh[0].numel() * Kh.element_size()
    d2h = Oh[0].numel() * Oh.element_size() + Lh[0].numel() * 4
    return t, h2d, d2h


class Train:
    """Training-shaped layer at 128k: every step rebuilds the index from the step's keys,
    selects for all 131072 causal queries, runs the tree attention forward and the
    backward (dQ, dK, dV) for that selection."""

    def __init__(self, cfg, dev, seed):
        from hierarchical_latent_key_b200 import lsa
        self.lsa, self.cfg, self.dev = lsa, cfg, dev
        c = cfg.case(dev, seed)
        self.K, self.V, self.W, self.Q, self.q_pos, self.dO = c.K, c.V, c.W, c.Q, c.q_pos, c.dO
        del c
        T, Hq, d = self.Q.shape
        self.desc = lsa.lsa_tree_describe(cfg.Hkv, cfg.r, cfg.branching, cfg.leaf)
        self.tree_mem = torch.empty(self.desc.bytes, dtype=torch.uint8, device=dev)
        self.build_ws = torch.empty(lsa.lsa_build_workspace_bytes(self.desc, d), dtype=torch.uint8, device=dev)
        self.leaves = torch.empty(cfg.Hkv, T, cfg.beam[-1], dtype=torch.int32, device=dev)
        self.O = torch.empty_like(self.Q)
        self.LSE = torch.empty(T, Hq, dtype=torch.float32, device=dev)
        self.dQ = torch.empty(T, Hq, d, dtype=torch.float32, device=dev)
        self.dK = torch.empty(self.K.shape, dtype=torch.float32, device=dev)
        self.dV = torch.empty(self.V.shape, dtype=torch.float32, device=dev)
        need = lsa.lsa_tree_attn_workspace_bytes(self.desc, T, Hq, d, self.Q.dtype, cfg.beam[-1])
        self.attn_ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        need = lsa.lsa_tree_attn_bwd_workspace_bytes(self.desc, T, Hq, d, self.Q.dtype, cfg.beam[-1])
        self.bwd_ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        need = lsa.lsa_select_batched_workspace_bytes(self.desc, T, cfg.beam)
        self.sel_ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.scale = 1.0 / math.sqrt(d)
        self.seed = seed

    def phases(self):
        L, c = self.lsa, self.cfg
        return (
            ("build", lambda: L.lsa_build_tree(self.desc, self.tree_mem, self.K, self.W, c.iters, self.seed,
                                              self.build_ws, None, self.status)),
            ("select", lambda: L.lsa_select_batched(self.desc, self.tree_mem, self.Q, self.W, c.beam, self.q_pos,
                                                    None, self.leaves, workspace=self.sel_ws, status=self.status)),
            ("forward", lambda: L.lsa_tree_attn(self.desc, self.tree_mem, self.Q, self.K, self.V, self.leaves,
                                                self.q_pos, True, self.scale, self.O, self.LSE, self.attn_ws,
                                                self.status)),
            ("backward", lambda: L.lsa_tree_attn_bwd(self.desc, self.tree_mem, self.Q, self.K, self.V, self.O,
                                                     self.LSE, self.dO, self.leaves, self.q_pos, True, self.scale,
                                                     self.dQ, self.dK, self.dV, self.bwd_ws, self.status)),
        )


def run_train(args, dev, rank, world, reduce_max, steps=3, warmup=2):
    cfg = configs.get("train_128k")
    if args.small:   # profiling case: the training geometry over 16,384 tokens
        cfg = cfg.scaled(name="train_geometry_16k", n=16384, T=16384, branching=(16, 16), beam=(8, 32), comps=256)
    # (--small: 16 x 16 leaves of 64 keys, beam 8/32 = 2048 keys per query, as the full tree's last level)
    w = Train(cfg, dev, rank_seed(cfg.seed, rank))
    stream = torch.cuda.current_stream(dev)
    ph = w.phases()
    for _ in range(warmup):
        for _, f in ph:
            f()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(ph) + 1)] for _ in range(steps)]
    for k in range(steps):
        ev[k][0].record(stream)
        for i, (_, f) in enumerate(ph):
            f()
            ev[k][i + 1].record(stream)
    torch.cuda.synchronize()
    code = w.lsa.lsa_status_check(w.status)
    if code != 0:
        raise RuntimeError(f"kernel status {code}: {w.lsa.lsa_strerror(code)}")
    total_s = sum(ev[k][0].elapsed_time(ev[k][-1]) for k in range(steps)) / 1e3
    value, t_max = aggregate(total_s, cfg.T * steps, world, reduce_max)
    br = {name: statistics.mean(ev[k][i].elapsed_time(ev[k][i + 1]) for k in range(steps))
          for i, (name, _) in enumerate(ph)}
    flops_fwd = 4.0 * cfg.T * cfg.Hq * cfg.K_sel * cfg.d
    out = {"value": value, "unit": "tokens/s (index build + select + attention forward + backward)",
           "steps": steps, "warmup": warmup, "ms_per_step": 1e3 * t_max / steps,
           "config": {"workload": f"{cfg.name}: causal layer over {cfg.T:,} tokens, {cfg.Hq}/{cfg.Hkv} heads, "
                                  f"d={cfg.d}, r={cfg.r}, tree {'/'.join(map(str, cfg.branching))} leaf {cfg.leaf}, "
                                  f"beam {'/'.join(map(str, cfg.beam))} ({cfg.K_sel} keys/query), index rebuilt "
                                  f"every step", "seq_len": cfg.T},
           "breakdown_ms": br,
           "forward_tflops": flops_fwd / (br["forward"] / 1e3) / 1e12,
           "backward_tflops": 2.5 * flops_fwd / (br["backward"] / 1e3) / 1e12,
           "gpu_launches_per_step": None}
    if rank == 0 and not args.no_cpu_baseline:
        try:
            out["cpu_baseline"] = cpu_baseline_train(w)
        except Exception as e:  # noqa: BLE001
            out["cpu_baseline"] = {"error": f"{type(e).__name__}: {e}"}
    del w
    torch.cuda.empty_cache()
    return out


def run_append(dev, seed):
    """Update of the index on append (lsa_tree_append) at the decode_128k geometry: once a
    top-level subtree's worth of keys (leaf * b_1 * b_2 = 8192) has been appended after the
    131,072 indexed ones, a subtree is built over those keys alone and attached as one more top
    node, instead of rebuilding the whole index.  CUDA events, median of 3, beside the build of
    the 131,072-key index the decode started from; then one decode step's select over the grown
    index."""
    from hierarchical_latent_key_b200 import lsa
    base = configs.get("decode_128k")
    U = base.leaf * int(np.prod(base.branching[1:]))
    cfg = base.scaled(T=U)
    c = cfg.case(dev, seed)
    K, W = c.K, c.W
    stream = torch.cuda.current_stream(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def timed(fn):
        times, out = [], None
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            out = fn()
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        return out, statistics.median(times)

    desc = lsa.lsa_tree_describe(cfg.Hkv, cfg.r, cfg.branching, cfg.leaf)
    bws = torch.empty(lsa.lsa_build_workspace_bytes(desc, cfg.d), dtype=torch.uint8, device=dev)
    aws = torch.empty(lsa.lsa_tree_append_workspace_bytes(desc, cfg.d), dtype=torch.uint8, device=dev)
    tree, build_ms = timed(lambda: lsa.build_tree(K, W, cfg.branching, cfg.leaf, cfg.iters, cfg.seed, workspace=bws,
                                                  status=status, check=False))
    grown, append_ms = timed(lambda: lsa.tree_append(tree, K, W, cfg.iters, cfg.seed, workspace=aws, status=status,
                                                     check=False))
    q_pos = torch.full((1,), cfg.n + U - 1, dtype=torch.int32, device=dev)
    (_, sel_ms) = timed(lambda: lsa.select(grown, c.Q[U - 1:U], W, cfg.beam, q_pos, status=status, check=False))
    code = lsa.lsa_status_check(status)
    if code != 0:
        raise RuntimeError(f"kernel status {code}: {lsa.lsa_strerror(code)}")
    return {"append_ms": append_ms, "build_ms": build_ms, "unit": "ms",
            "keys_appended": U, "top_nodes": [int(tree.desc.nodes[0]), int(grown.desc.nodes[0])],
            "select_after_ms": sel_ms,
            "config": f"decode_128k geometry: tree {'/'.join(map(str, cfg.branching))} leaf {cfg.leaf} over "
                      f"{cfg.n:,} keys x {cfg.Hkv} KV heads; {U:,} appended keys per head get their own subtree "
                      f"({cfg.iters} k-means rounds per level); build_ms is the index of the {cfg.n:,} keys"}


def run_decode(args, dev, rank, world, reduce_max):
    cfg = configs.get("decode_10m")
    if args.small:   # profiling case: the decode step over the 131,072-key index of decode_128k
        cfg = configs.get("decode_128k").scaled(T=cfg.T, beam=(8, 32, 32))
    steps, warmup = cfg.T, args.warmup
    w = Decode(cfg, dev, rank_seed(cfg.seed, rank), warmup + steps)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    w.capture(warmup + steps)
    total = time_decode(w, steps, warmup, flush, stream)
    code = w.lsa.lsa_status_check(w.status)
    if code != 0:
        raise RuntimeError(f"kernel status {code}: {w.lsa.lsa_strerror(code)}")
    total_s = sum(total) / 1e3
    value, t_max = aggregate(total_s, steps, world, reduce_max)
    e2e_t, h2d, d2h = time_decode_e2e(w, steps, warmup, flush, stream)
    e2e_value, _ = aggregate(sum(e2e_t) / 1e3, steps, world, reduce_max)
    peaks = measured_peaks()
    att_b = statistics.mean(w.bytes_per_step(warmup + k)[0] for k in range(steps))
    sel_b = w.bytes_per_step(0)[1]
    step_s = total_s / steps
    out = {
        "value": value, "unit": "queries/s", "steps": steps, "ms_per_step": 1e3 * t_max / steps,
        "config": {"workload": f"{cfg.name}: single-request decode over {cfg.n:,} indexed keys, {cfg.Hq}/{cfg.Hkv} "
                               f"heads, d={cfg.d}, r={cfg.r}, tree {'/'.join(map(str, cfg.branching))} leaf "
                               f"{cfg.leaf}, beam {'/'.join(map(str, cfg.beam))} ({cfg.K_sel} keys) + dense tail "
                               f"of appended keys", "seq_len": cfg.n,
                   "l2": "flushed between timed steps (512 MiB write outside the events)"},
        "breakdown_us": {"step_graph": 1e3 * statistics.mean(total), "step_graph_min": 1e3 * min(total),
                         "build_once_ms": w.build_ms},
        "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "roofline": {"bound": "hbm", "unit": "GB/s", "peak": peaks["hbm_gbs"], "peak_source": peaks["source"],
                     "achieved": (att_b + sel_b) / step_s / 1e9,
                     "frac": (att_b + sel_b) / step_s / 1e9 / peaks["hbm_gbs"],
                     "algorithmic_bytes": att_b + sel_b, "traffic": None,
                     "kernels": "k_select_wide (append, 5-level walk) + k_dec_attn (gather, split merge)"},
        "gpu_launches": w.launches_per_step * steps,
        "cuda_graph": "one graph per decode step (lsa_decode_step: select with the append, attention)",
    }
    if rank == 0 and not args.no_cpu_baseline:
        try:
            out["cpu_baseline"] = cpu_baseline_decode(w)
        except Exception as e:  # noqa: BLE001
            out["cpu_baseline"] = {"error": f"{type(e).__name__}: {e}"}
    w.graphs = None
    del w
    torch.cuda.empty_cache()
    return out


def time_steps(w, steps, warmup, flush, stream):
    """Device time of `steps` steps (select + attention), L2 flushed between steps."""
    for _ in range(warmup):
        flush.zero_()
        w.select()
        w.attend()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for k in range(steps):
        flush.zero_()
        ev[k][0].record(stream)
        w.select()
        ev[k][1].record(stream)
        w.attend()
        ev[k][2].record(stream)
    torch.cuda.synchronize()
    sel = [ev[k][0].elapsed_time(ev[k][1]) for k in range(steps)]
    att = [ev[k][1].elapsed_time(ev[k][2]) for k in range(steps)]
    return sel, att


SINK, WINDOW = 16, 512   # sink tokens and recent window of the sink/window measurement
# DRAM bytes read + written per lsa_tree_attn call of the prefill_1m step, from single-pass ncu
# captures of the full workload (dram__bytes_read.sum + dram__bytes_write.sum, one launch each,
# the first call of the warm-up steps): k_tl_pipe 4,914,926,080 + 1,172,362,496 and k_tl_combine
# 1,111,510,528 + 31,419,904; the five leaf- and chunk-list kernels add about 12 MB and are left out.
# To be taken again whenever one of those kernels changes.
TREE_ATTN_TRAFFIC_BYTES = 4_914_926_080 + 1_172_362_496 + 1_111_510_528 + 31_419_904
POOL = 4                 # keys per block of the pooled index


def time_sink_window(w, steps, warmup, flush, stream, sink=SINK, window=WINDOW):
    """The prefill step with sink and recent-window keys added to every query (lsa_tree_attn_sw)."""
    lsa = w.lsa
    T, Hq, d = w.Q.shape
    need = lsa.lsa_tree_attn_sw_workspace_bytes(w.tree.desc, T, Hq, d, w.Q.dtype, w.cfg.beam[-1], sink, window)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=w.Q.device)

    def attend():
        lsa.lsa_tree_attn_sw(w.tree.desc, w.tree.mem, w.Q, w.K, w.V, w.leaves, w.q_pos, sink, window, w.scale, w.O,
                             w.LSE, ws, w.status)

    for _ in range(warmup):
        flush.zero_()
        w.select()
        attend()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for k in range(steps):
        flush.zero_()
        ev[k][0].record(stream)
        w.select()
        ev[k][1].record(stream)
        attend()
        ev[k][2].record(stream)
    torch.cuda.synchronize()
    code = lsa.lsa_status_check(w.status)
    if code != 0:
        raise RuntimeError(f"kernel status {code}: {lsa.lsa_strerror(code)}")
    sel = statistics.mean(ev[k][0].elapsed_time(ev[k][1]) for k in range(steps))
    att = statistics.mean(ev[k][1].elapsed_time(ev[k][2]) for k in range(steps))
    return {"value": T / ((sel + att) / 1e3), "unit": "queries/s", "n_sink": sink, "window": window,
            "breakdown_ms": {"select": sel, "attention": att},
            "config": f"prefill step as above, every query also attends to positions [0, {sink}) and its last "
                      f"{window} positions (each key once)"}


def time_flat(w, steps, warmup, flush, stream):
    """The prefill step with flat search (every leaf centroid scored, lsa_select_flat) in place of
    the beam walk, then the same tree attention."""
    lsa = w.lsa

    def select():
        lsa.lsa_select_flat(w.tree.desc, w.tree.mem, w.Q, w.W, w.cfg.beam[-1], w.q_pos, None, w.leaves,
                            status=w.status)

    for _ in range(warmup):
        flush.zero_()
        select()
        w.attend()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for k in range(steps):
        flush.zero_()
        ev[k][0].record(stream)
        select()
        ev[k][1].record(stream)
        w.attend()
        ev[k][2].record(stream)
    torch.cuda.synchronize()
    code = lsa.lsa_status_check(w.status)
    if code != 0:
        raise RuntimeError(f"kernel status {code}: {lsa.lsa_strerror(code)}")
    sel = statistics.mean(ev[k][0].elapsed_time(ev[k][1]) for k in range(steps))
    att = statistics.mean(ev[k][1].elapsed_time(ev[k][2]) for k in range(steps))
    T = w.Q.shape[0]
    nl = w.cfg.nodes[-1]
    return {"value": T / ((sel + att) / 1e3), "unit": "queries/s", "breakdown_ms": {"select": sel, "attention": att},
            "config": f"prefill step as above with flat search: {nl} leaf centroids scored per query and group, "
                      f"the best {w.cfg.beam[-1]} kept"}


def time_pooled(w, steps, warmup, flush, stream, pool=POOL):
    """The index over blocks of `pool` consecutive keys (lsa_build_tree_pooled): its build beside
    the plain build (CUDA events, same workspace, median of 3), then the prefill step (select +
    tree attention) on the pooled index."""
    lsa, cfg = w.lsa, w.cfg
    d = w.K.shape[2]
    ws = torch.empty(lsa.lsa_build_workspace_bytes(w.tree.desc, d), dtype=torch.uint8, device=w.K.device)

    def build(p):
        times, tree = [], None
        for _ in range(3):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            tree = lsa.build_tree(w.K, w.W, cfg.branching, cfg.leaf, cfg.iters, cfg.seed, workspace=ws,
                                  status=w.status, check=False, pool=p)
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        return tree, statistics.median(times)

    _, keys_ms = build(1)
    tree, pooled_ms = build(pool)
    plain = w.tree
    w.tree = tree
    try:
        for _ in range(warmup):
            flush.zero_()
            w.select()
            w.attend()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for k in range(steps):
            flush.zero_()
            ev[k][0].record(stream)
            w.select()
            ev[k][1].record(stream)
            w.attend()
            ev[k][2].record(stream)
        torch.cuda.synchronize()
    finally:
        w.tree = plain
    code = lsa.lsa_status_check(w.status)
    if code != 0:
        raise RuntimeError(f"kernel status {code}: {lsa.lsa_strerror(code)}")
    sel = statistics.mean(ev[k][0].elapsed_time(ev[k][1]) for k in range(steps))
    att = statistics.mean(ev[k][1].elapsed_time(ev[k][2]) for k in range(steps))
    T = w.Q.shape[0]
    return {"value": T / ((sel + att) / 1e3), "unit": "queries/s", "pool": pool,
            "build_ms": {"pooled": pooled_ms, "keys": keys_ms},
            "breakdown_ms": {"select": sel, "attention": att},
            "config": f"prefill step as above on an index whose k-means levels cluster blocks of {pool} "
                      f"consecutive keys ({cfg.n // pool:,} blocks per head, {cfg.leaf // pool} per leaf); "
                      f"build times over all {cfg.Hkv} heads with CUDA events"}


def time_projection(w, steps, warmup, flush, stream):
    """The latent projection Z = K . W of the index build (lsa_project_keys, tensor cores) over
    all indexed keys of every KV head, L2 flushed between launches."""
    lsa, cfg = w.lsa, w.cfg
    Hkv, _, d = w.K.shape
    Z = torch.empty(Hkv, cfg.n, cfg.r, dtype=torch.float32, device=w.K.device)
    for _ in range(warmup):
        lsa.lsa_project_keys(w.K, w.W, cfg.n, Z, w.status)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for k in range(steps):
        flush.zero_()
        ev[k][0].record(stream)
        lsa.lsa_project_keys(w.K, w.W, cfg.n, Z, w.status)
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(ev[k][0].elapsed_time(ev[k][1]) for k in range(steps))
    alg = Hkv * cfg.n * (d * w.K.element_size() + cfg.r * 4) + w.W.numel() * w.W.element_size()
    peak = measured_peaks()["hbm_gbs"]
    del Z
    return {"kernel": "k_project_tc", "ms": ms, "keys": Hkv * cfg.n, "algorithmic_bytes": alg,
            "achieved_gbs": alg / (ms / 1e3) / 1e9, "frac": alg / (ms / 1e3) / 1e9 / peak,
            "tflops": 2.0 * Hkv * cfg.n * d * cfg.r / (ms / 1e3) / 1e12}


def time_e2e(w, steps, flush, stream):
    """Same step through the public API with pinned host buffers: H2D of the chunk's
    queries, select + attention, D2H of the outputs, all inside the timed region."""
    Qh = w.Q.cpu().pin_memory()
    Oh = torch.empty(w.O.shape, dtype=w.O.dtype).pin_memory()
    Lh = torch.empty(w.LSE.shape, dtype=torch.float32).pin_memory()
    Qd = torch.empty_like(w.Q)
    times = []
    for k in range(steps + 1):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        Qd.copy_(Qh, non_blocking=True)
        w.select(Qd)
        w.attend(Qd)
        Oh.copy_(w.O, non_blocking=True)
        Lh.copy_(w.LSE, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        if k:  # first pass warms the pinned-copy path
            times.append(a.elapsed_time(b))
    h2d = Qh.numel() * Qh.element_size()
    d2h = Oh.numel() * Oh.element_size() + Lh.numel() * 4
    return times, h2d, d2h


def cpu_baseline_prefill(w, n_queries=4096):
    """The oracle as it stands on this host: select + attention for a sample of the chunk's
    queries on KV head 0 (of 8), on the index the GPU built (exported to float64)."""
    from oracle import oracle as orc
    cfg = w.cfg
    h = 0
    tree = orc.Tree.from_levels(cfg.branching, cfg.leaf,
                                [w.tree.centroids(l)[h].cpu() for l in range(len(cfg.branching))],
                                [w.tree.min_pos(l)[h].cpu() for l in range(len(cfg.branching))],
                                w.tree.leaf_index()[h].cpu())
    Kh = orc._f64(w.K[h].cpu())
    Vh = orc._f64(w.V[h].cpu())
    sel = slice(cfg.T - n_queries, cfg.T)
    Qg = w.Q[sel, h * cfg.G:(h + 1) * cfg.G].cpu()
    Wh = w.W[h].cpu()
    qp = w.q_pos[sel].cpu().numpy()
    t0 = time.perf_counter()
    qlat = orc.query_latent(Qg, Wh)
    idx, _, _ = orc.select(qlat, tree, cfg.beam, q_pos=qp)
    orc.attn_fwd(Qg, Kh, Vh, idx, q_pos=qp, causal=True)
    dt = time.perf_counter() - t0
    qps = n_queries / (dt * cfg.Hkv)
    # single core: 64 of the queries in a one-thread child process (walk on the oracle, attention over
    # each query's visible selected keys, gathered from the GPU's selection)
    rows = np.arange(cfg.T - 64, cfg.T)
    kc, vc = [], []
    for t in rows:
        lv = w.leaves[h][t]
        kk = w.tree.leaf_index()[h].view(-1, cfg.leaf)[lv[lv >= 0].long()].reshape(-1)
        kk = kk[kk <= w.q_pos[t]].long()
        kc.append(w.K[h, kk].double().cpu().numpy())
        vc.append(w.V[h, kk].double().cpu().numpy())
    L = len(cfg.branching)
    one = _single_core("prefill", dict(
        branching=np.asarray(cfg.branching, np.int32), leaf=np.int64(cfg.leaf),
        cents=[w.tree.centroids(l)[h].double().cpu().numpy() for l in range(L)],
        mpos=[w.tree.min_pos(l)[h].cpu().numpy() for l in range(L)], leaf_index=w.tree.leaf_index()[h].cpu().numpy(),
        W=Wh.double().numpy(), beam=np.asarray(cfg.beam), q_pos=w.q_pos[rows].cpu().numpy(),
        Qg=w.Q[rows, h * cfg.G:(h + 1) * cfg.G].double().cpu().numpy(), Kc=kc, Vc=vc))
    return {"value": qps, "unit": "queries/s", "cores": cores_used(), "kind": "oracle",
            "single_core_value": 64 / (one * cfg.Hkv),
            "sample": f"{n_queries} of {cfg.T} chunk queries on KV head 0 of {cfg.Hkv} (select + attention, "
                      f"float64 C oracle, OpenMP), scaled x{cfg.Hkv} heads; index built on the GPU; "
                      f"single_core_value: the last 64 queries with one OpenMP thread (walk on the oracle, attention "
                      f"over each query's visible keys of the GPU's selection)"}


# ---------------------------------------------------------------------------
# oracle timing on the host (the cpu_baseline entries)
# ---------------------------------------------------------------------------

def _oracle_sample(kind, arrays):
    """Run one oracle sample in this process; returns seconds of oracle work."""
    from oracle import oracle as orc
    t0 = time.perf_counter()
    if kind == "prefill":
        tree = orc.Tree.from_levels(arrays["branching"], int(arrays["leaf"]), arrays["cents"], arrays["mpos"],
                                    arrays["leaf_index"])
        qlat = orc.query_latent(arrays["Qg"], arrays["W"])
        orc.select(qlat, tree, arrays["beam"], q_pos=arrays["q_pos"])
        for t in range(arrays["Qg"].shape[0]):
            Kc, Vc = arrays["Kc"][t], arrays["Vc"][t]
            orc.attn_fwd(arrays["Qg"][t:t + 1], Kc, Vc, np.zeros((1, 0), np.int32), tail=(0, Kc.shape[0]))
    elif kind == "decode":
        tree = orc.Tree.from_levels(arrays["branching"], int(arrays["leaf"]), arrays["cents"], arrays["mpos"],
                                    arrays["leaf_index"])
        for s in range(arrays["Qg"].shape[0]):
            qlat = orc.query_latent(arrays["Qg"][s:s + 1], arrays["W"])
            orc.select(qlat, tree, arrays["beam"])
            Kc, Vc = arrays["Kc"][s], arrays["Vc"][s]
            orc.attn_fwd(arrays["Qg"][s:s + 1], Kc, Vc, np.zeros((1, 0), np.int32), tail=(0, Kc.shape[0]))
    elif kind == "train":
        qp = arrays["q_pos"]
        O, LSE = orc.attn_fwd(arrays["Qg"], arrays["K"], arrays["V"], arrays["idx"], q_pos=qp, causal=True)
        orc.attn_bwd(arrays["Qg"], arrays["K"], arrays["V"], arrays["idx"], arrays["dO"], q_pos=qp, causal=True)
    else:
        raise ValueError(kind)
    return time.perf_counter() - t0


def _single_core(kind, arrays):
    """The same oracle sample in a child process limited to one OpenMP thread."""
    import subprocess
    import tempfile
    with tempfile.TemporaryDirectory() as d:
        path = os.path.join(d, "sample.npz")
        packed = {}
        for k, v in arrays.items():
            if isinstance(v, list):
                obj = np.empty(len(v), dtype=object)
                for i, x in enumerate(v):
                    obj[i] = x
                v = obj
            packed[k] = v
        np.savez(path, **packed)
        code = ("import sys, json; sys.path.insert(0, %r); import numpy as np, bench; "
                "z = np.load(%r, allow_pickle=True); a = {k: (list(z[k]) if z[k].dtype == object else z[k]) "
                "for k in z.files}; print(json.dumps(bench._oracle_sample(%r, a)))") % (ROOT, path, kind)
        env = dict(os.environ, OMP_NUM_THREADS="1", CUDA_VISIBLE_DEVICES="")
        r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=900)
        if r.returncode != 0:
            raise RuntimeError(r.stderr[-500:])
        return float(r.stdout.strip().splitlines()[-1])


def cpu_baseline_decode(w, n_steps=8):
    """The oracle per decode step on KV head 0 (of 8): group latent, the beam walk over the
    index the GPU built (exported to float64), attention over the kept leaves' keys and the
    tail (rows gathered on the device first); scaled x8 heads."""
    cfg = w.cfg
    h = 0
    L = len(cfg.branching)
    n = cfg.n
    li = w.tree.leaf_index()[h]
    qg, kcs, vcs = [], [], []
    for s in range(n_steps):
        keys = torch.cat([li.view(-1, cfg.leaf)[w.dec.leaves[h][w.dec.leaves[h] >= 0].long()].reshape(-1),
                          torch.arange(n, n + s + 1, device=li.device, dtype=li.dtype)]).long()
        kcs.append(w.K[h, keys].double().cpu().numpy())
        vcs.append(w.V[h, keys].double().cpu().numpy())
        qg.append(w.Q[s, h * cfg.G:(h + 1) * cfg.G].double().cpu().numpy())
    arrays = dict(branching=np.asarray(cfg.branching, np.int32), leaf=np.int64(cfg.leaf),
                  cents=[w.tree.centroids(l)[h].double().cpu().numpy() for l in range(L)],
                  mpos=[w.tree.min_pos(l)[h].cpu().numpy() for l in range(L)],
                  leaf_index=li.cpu().numpy(), W=w.W[h].double().cpu().numpy(), beam=np.asarray(cfg.beam),
                  Qg=np.stack(qg), Kc=kcs, Vc=vcs)
    dt = _oracle_sample("decode", arrays)
    one = _single_core("decode", arrays)
    return {"value": n_steps / (dt * cfg.Hkv), "unit": "queries/s", "cores": cores_used(), "kind": "oracle",
            "single_core_value": n_steps / (one * cfg.Hkv),
            "sample": f"{n_steps} decode steps on KV head 0 of {cfg.Hkv} (latent, beam walk over the GPU-built "
                      f"index, attention over the kept leaves' keys + tail gathered on the device), float64 C "
                      f"oracle, scaled x{cfg.Hkv} heads; single_core_value: the same with one OpenMP thread"}


def cpu_baseline_train(w, n_queries=48):
    """The oracle's forward + backward for a sample of queries on KV head 0 (of 4), over the
    GPU's selection, extrapolated to the whole layer (all queries, all heads); the oracle's
    own index build for one head is timed too and added once per head."""
    from oracle import oracle as orc
    cfg = w.cfg
    h = 0
    rng = np.random.default_rng(0)
    rows = np.sort(rng.choice(cfg.T, n_queries, replace=False))
    li = w.lsa.Tree(w.desc, w.tree_mem).leaf_index()[h].view(-1, cfg.leaf)
    lv = w.leaves[h][torch.as_tensor(rows, device=w.leaves.device)].long()
    idx = torch.where(lv[..., None] >= 0, li[lv.clamp(min=0)], -1).reshape(len(rows), -1).cpu().numpy()
    arrays = dict(Qg=w.Q[rows][:, h * cfg.G:(h + 1) * cfg.G].double().cpu().numpy(),
                  K=w.K[h].double().cpu().numpy(), V=w.V[h].double().cpu().numpy(), idx=idx,
                  dO=w.dO[rows][:, h * cfg.G:(h + 1) * cfg.G].double().cpu().numpy(),
                  q_pos=w.q_pos.cpu().numpy()[rows])
    dt = _oracle_sample("train", arrays)
    one = _single_core("train", dict(arrays, Qg=arrays["Qg"][:8], idx=idx[:8], dO=arrays["dO"][:8],
                                     q_pos=arrays["q_pos"][:8]))
    Z = orc.project(w.K[h, :cfg.n].cpu(), w.W[h].cpu())
    t0 = time.perf_counter()
    orc.build_tree(Z, cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    build_s = time.perf_counter() - t0
    per_q = dt / n_queries
    total = cfg.Hkv * (build_s + per_q * cfg.T)
    return {"value": cfg.T / total, "unit": "tokens/s", "cores": cores_used(), "kind": "oracle",
            "extrapolated": True, "single_core_value": cfg.T / (cfg.Hkv * (one / 8) * cfg.T),
            "sample": f"{n_queries} of {cfg.T} queries on KV head 0 of {cfg.Hkv}: forward + backward over the GPU's "
                      f"selection ({per_q * 1e3:.1f} ms per query), plus the oracle's index build for one head "
                      f"({build_s:.1f} s); extrapolated to all queries and heads; single_core_value: forward + "
                      f"backward only (8 queries, one OpenMP thread), select and build excluded"}


def bench_config(args):
    cfg = configs.get("prefill_1m")
    if args.small:
        cfg = cfg.scaled(name="prefill_1m_geometry_131k", n=131072, branching=(8, 8, 8, 4), comps=1024)
    return cfg


def run_single(args, rank, world, local_rank):
    """Headline = one of the secondary workloads alone (decode_10m or train_128k)."""
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    pg = world > 1

    def reduce_max(x):
        if not pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())

    if pg:
        torch.distributed.barrier()
    with ClockSampler(local_rank) as clk:
        if args.workload == "decode_10m":
            r = run_decode(args, dev, rank, world, reduce_max)
        else:
            r = run_train(args, dev, rank, world, reduce_max, steps=args.steps, warmup=args.warmup)
        if pg:
            torch.distributed.barrier()
    if rank != 0:
        return None
    unit = r.pop("unit")
    line = {"metric": METRIC, "value": r.pop("value"), "unit": unit, "n_gpus": world,
            "steps": r.pop("steps"), "warmup": r.pop("warmup", args.warmup), "ms_per_step": r.pop("ms_per_step"),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "clocks": clk.summary()}
    line["config"] = dict(r.pop("config"), parallelism=f"dp{world}")
    line.update(r)
    return line


def run_cuda(args, rank, world, local_rank):
    if args.workload in ("decode_10m", "train_128k"):
        return run_single(args, rank, world, local_rank)
    if args.workload != "prefill_1m":
        raise SystemExit(f"workload {args.workload} has no benchmark (parity tests only)")
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = bench_config(args)
    seed = rank_seed(cfg.seed, rank)
    w = Prefill(cfg, dev, seed)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    pg = world > 1
    if pg:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        sel, att = time_steps(w, args.steps, args.warmup, flush, stream)
        if pg:
            torch.distributed.barrier()
        torch.cuda.synchronize()
    code = w.lsa.lsa_status_check(w.status)
    if code != 0:
        raise RuntimeError(f"kernel status {code}: {w.lsa.lsa_strerror(code)}")
    total_s = (sum(sel) + sum(att)) / 1e3

    def reduce_max(x):
        if not pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        return float(t.item())

    value, t_max = aggregate(total_s, w.units * args.steps, world, reduce_max)
    e2e_t, h2d, d2h = time_e2e(w, args.steps, flush, stream)
    e2e_value, _ = aggregate(sum(e2e_t) / 1e3, w.units * args.steps, world, reduce_max)
    alg_bytes, rows = w.attn_algorithmic_bytes()
    cpu = cpu_baseline_prefill(w) if (rank == 0 and not args.no_cpu_baseline) else None
    att_flops = w.attn_flops()
    build_ms = w.build_ms
    att_s = statistics.mean(att) / 1e3
    peaks = measured_peaks()
    achieved = alg_bytes / att_s / 1e9
    launches = w.launches_per_step * args.steps
    try:
        sink_window = time_sink_window(w, args.steps, args.warmup, flush, stream)
    except Exception as e:  # noqa: BLE001
        sink_window = {"error": f"{type(e).__name__}: {e}"}
    try:
        flat = time_flat(w, args.steps, args.warmup, flush, stream)
    except Exception as e:  # noqa: BLE001
        flat = {"error": f"{type(e).__name__}: {e}"}
    try:
        projection = time_projection(w, args.steps, args.warmup, flush, stream)
    except Exception as e:  # noqa: BLE001
        projection = {"error": f"{type(e).__name__}: {e}"}
    try:
        pooled = time_pooled(w, args.steps, args.warmup, flush, stream)
    except Exception as e:  # noqa: BLE001
        pooled = {"error": f"{type(e).__name__}: {e}"}
    decode = train = append = None
    del w
    torch.cuda.empty_cache()
    if not args.small:
        try:
            append = run_append(dev, rank_seed(5, rank))
        except Exception as e:  # noqa: BLE001
            append = {"error": f"{type(e).__name__}: {e}"}
        torch.cuda.empty_cache()
    # secondary workloads: a failure is reported in the line instead of losing the headline
    if not args.no_decode and not args.small:
        try:
            with ClockSampler(local_rank) as clk_dec:
                decode = run_decode(args, dev, rank, world, reduce_max)
            decode["clocks"] = clk_dec.summary()
        except Exception as e:  # noqa: BLE001
            decode = {"error": f"{type(e).__name__}: {e}"}
        torch.cuda.empty_cache()
    if not args.no_train and not args.small:
        try:
            train = run_train(args, dev, rank, world, reduce_max)
        except Exception as e:  # noqa: BLE001
            train = {"error": f"{type(e).__name__}: {e}"}
        torch.cuda.empty_cache()
    line = None
    if rank == 0:
        clocks = clk.summary()
        line = {
            "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * t_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(prefill_config(cfg, world),
                           l2="flushed between timed steps (512 MiB write outside the events)"),
            "breakdown_ms": {"select": statistics.mean(sel), "attention": statistics.mean(att),
                             "build_once": build_ms},
            "e2e": {"value": e2e_value, "unit": "queries/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "roofline": {"kernel": "lsa_tree_attn (leaf lists + k_tl_pipe + k_tl_combine)", "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                         "traffic": TREE_ATTN_TRAFFIC_BYTES if not args.small else None,
                         "peak_source": peaks["source"],
                         "algorithmic_bytes": alg_bytes, "distinct_kv_rows": rows,
                         "tensor_tflops": att_flops / att_s / 1e12},
            "gpu_launches": launches,
            "clocks": clocks,
            "cpu_baseline": cpu,
            "prefill_1m_sink_window": sink_window,
            "prefill_1m_flat": flat,
            "prefill_1m_pooled": pooled,
            "projection_1m": projection,
            "tree_append_128k": append,
            "decode_10m": decode,
            "train_128k": train,
        }
    return line


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle on this host
# ---------------------------------------------------------------------------

def prefill_config(cfg, world):
    """The `config` object of the prefill line (both arms)."""
    return {"workload": f"{cfg.name}: {cfg.T} query tokens over {cfg.n:,} cached keys, "
                        f"{cfg.Hq}/{cfg.Hkv} heads, d={cfg.d}, r={cfg.r}, tree "
                        f"{'/'.join(map(str, cfg.branching))} leaf {cfg.leaf}, beam "
                        f"{'/'.join(map(str, cfg.beam))} ({cfg.K_sel} keys/query), causal",
            "global_batch": cfg.T * world, "seq_len": cfg.n, "parallelism": f"dp{world}"}


def run_reference(args):
    from oracle import oracle as orc
    cfg = bench_config(args)
    one = cfg.scaled(Hkv=1, Hq=cfg.G)
    c = one.case("cpu")
    t0 = time.perf_counter()
    Z = orc.project(c.K[0, :cfg.n], c.W[0])
    tree = orc.build_tree(Z, cfg.branching, cfg.leaf, cfg.iters, cfg.seed)
    build_s = time.perf_counter() - t0
    Kh, Vh = orc._f64(c.K[0]), orc._f64(c.V[0])
    n_q = 256
    times = []
    for k in range(args.warmup + args.steps):
        sel = slice((k * n_q) % cfg.T, (k * n_q) % cfg.T + n_q)
        Qg = c.Q[sel]
        qp = c.q_pos[sel].numpy()
        t0 = time.perf_counter()
        qlat = orc.query_latent(Qg, c.W[0])
        idx, _, _ = orc.select(qlat, tree, cfg.beam, q_pos=qp)
        orc.attn_fwd(Qg, Kh, Vh, idx, q_pos=qp, causal=True)
        if k >= args.warmup:
            times.append(time.perf_counter() - t0)
    per_q = sum(times) / (len(times) * n_q) * cfg.Hkv
    value = 1.0 / per_q
    sample = (f"{n_q} chunk queries per step on one KV head (of {cfg.Hkv}), scaled x{cfg.Hkv}; "
              f"oracle-built index over {cfg.n:,} keys (build {build_s:.0f} s, untimed)")
    return {"metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": prefill_config(cfg, 1),
            "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "cpu_baseline": {"value": value, "unit": "queries/s", "cores": cores_used(), "kind": "oracle",
                             "sample": sample}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["lsa", "reference"], default="lsa")
    ap.add_argument("--workload", default="prefill_1m", choices=sorted(configs.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the 10M-token decode measurement")
    ap.add_argument("--no-train", action="store_true", help="skip the training-shaped 128k layer step")
    ap.add_argument("--small", action="store_true",
                    help="profiling case: the prefill geometry (4096 queries x 2048 keys) over 131,072 cached "
                         "keys, tree 8/8/8/4, so a kernel capture stays small; with --workload decode_10m the "
                         "decode step over a 131,072-key index, with --workload train_128k a 16,384-token layer")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_cuda(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
