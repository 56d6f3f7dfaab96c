#!/usr/bin/env python
"""Decode benchmark of tree-indexed sparse attention on B200.

One step = one decode token for every sequence of the batch through the whole
hot path: append the token to the KV cache and the tree, route the query of
every head top-down through the tree with top-p at every level, and attend
exactly over the selected keys (plus sink and current chunk).  The workload is
the 1M-token decode case: batch 4, 32 query / 8 KV heads, head dim 128, bf16
K/V, N = 1,048,576 keys per sequence, leaf block 64, branching 16, p = 0.95,
planted-cluster synthetic keys and queries.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl own|reference]
                    [--workload decode1m|decode128k|decode8m|prefill256k] [--vsum] [--sweep N1,N2,...]

The step runs as one CUDA graph (append, route with the plan fused, attend); the
phases are timed apart in a second pass.  --workload prefill256k times a chunked
prefill (a 4096-query chunk over a 256K prefix) instead; --vsum decodes with the
dropped subtrees' value summaries and reports their error against dense
attention; --sweep compares the decode step with the dense baseline over context
lengths.

Prints one JSON line on rank 0.  Times are CUDA-event device times on the
launching stream (max over ranks); L2 is flushed (256 MiB write, then a 256 MiB read) before every
timed step, outside the events.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ZHA decode queries/s at 1M ctx + achieved HBM GB/s vs B200 peak"
PREFILL_METRIC = "ZHA chunked prefill queries/s at 256K ctx (4096-query chunk, tensor-core attention)"
FALLBACK_BF16_TFLOPS = 1590.0
UNIT = "queries/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # the B200 spec-sheet HBM3e bandwidth, for a second fraction beside the measured copy
POOL = 64                 # distinct (q, k_new, v_new) sets cycled through by the steps
E2E_WARMUP = 3            # untimed end-to-end steps before the timed ones
PHASE_STEPS = 200         # steps of the per-phase breakdown (after the timed one-graph steps)
ATTEND_SOURCES = ["hierarchical_tree_indexed_b200/csrc/zha_attend.cuh",
                  "hierarchical_tree_indexed_b200/csrc/zha_attend_tc.cuh",
                  "hierarchical_tree_indexed_b200/csrc/zha_umma.cuh",
                  "hierarchical_tree_indexed_b200/csrc/zha_common.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["own", "reference"], default="own")
    ap.add_argument("--workload", default="decode1m")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling cases)")
    ap.add_argument("--seq-len", type=int, default=0, help="override the workload's N (profiling cases)")
    ap.add_argument("--sweep", default="", help="comma-separated context lengths: tree path vs dense baseline")
    ap.add_argument("--run", type=int, default=0,
                    help="keys per planted cluster (0: the calibrated default); with --beta, another in-band calibration")
    ap.add_argument("--beta", type=float, default=0.0, help="query aim strength (0: the calibrated default)")
    ap.add_argument("--vsum", action="store_true",
                    help="decode with value summaries of the dropped subtrees, and report their error against dense")
    return ap.parse_args()


def workload(args):
    import dataclasses

    from hierarchical_tree_indexed_b200 import workloads as W
    w = W.WORKLOADS[args.workload]
    if args.batch:
        w = dataclasses.replace(w, batch=args.batch)
    if args.seq_len:
        w = dataclasses.replace(w, N=args.seq_len, n_clusters=max(1, args.seq_len // 2048))
    return w


def config_dict(w, world: int) -> dict:
    gen = ""
    if getattr(args_global, "run", 0) or getattr(args_global, "beta", 0.0):
        from hierarchical_tree_indexed_b200 import workloads as W
        gen = f", planted clusters of {args_global.run or W.RUN} keys aimed at with beta {args_global.beta or W.BETA}"
    return {"workload": f"{w.name}: batch {w.batch} per GPU, {w.Hq} query / {w.Hkv} KV heads, d {w.d}, "
                        f"bf16 K/V, N={w.N}, leaf block {w.B}, branching {w.b}, p={w.p}{gen}",
            "global_batch": w.batch * world, "seq_len": w.N, "parallelism": f"dp{world}",
            "kv_dtype": w.dtype,
            "l2": L2Flush.NOTE + f"; KV {w.batch * w.Hkv * w.N * w.d * 2 * (2 if w.dtype == 'bf16' else 4) / 2**30:.1f} GiB > L2",
            "step": "append + route (plan fused) + attend as one CUDA graph (phases timed apart, each its own graph)"}


class L2Flush:
    """Flushes L2 between timed steps: writes a 256 MiB buffer (twice L2), then reads another
    256 MiB buffer, so that L2 holds neither the step's inputs nor dirty lines that the timed
    kernels would have to write back to HBM.  Runs outside the timed region."""
    NOTE = "flushed before every timed step (256 MiB write, then 256 MiB read of another buffer: no dirty lines left)"

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones(64 << 20, dtype=torch.float32, device=dev)
        self.out = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        import torch
        self.w.zero_()
        torch.sum(self.r, dim=0, out=self.out)


def measured_peaks(key: str = "hbm_gbs") -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)[key]), "measured"
    except (OSError, KeyError, ValueError):
        return (FALLBACK_HBM_GBS if key == "hbm_gbs" else FALLBACK_BF16_TFLOPS), "fallback"


def source_hash(paths) -> str:
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_hash: str):
    """Per-launch DRAM bytes of the attend kernel from the committed ncu summary, if it
    was taken on this exact kernel source (scaled by rows when captured on a smaller case)."""
    p = os.path.join(ROOT, "profiles", "attend_traffic.txt")
    try:
        kv = dict(line.split(":", 1) for line in open(p) if ":" in line and not line.startswith("#"))
    except OSError:
        return None
    if kv.get("kernel_source_sha256_16", "").strip() != kernel_hash:
        return None
    try:
        return float(kv["bytes_per_row"]), float(kv.get("fixed_bytes", "0"))
    except (KeyError, ValueError):
        return None


class Clocks:
    """nvidia-smi sampler (every 200 ms) around the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-lms", "200", "-i", str(gpu_index)], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self) -> dict:
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.f.name)
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ CPU oracle arm

def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def time_oracle(calls, seconds: float, threads: int, steps: int | None = None):
    """Runs the oracle calls (closures, cycled) on `threads` host threads for about `seconds` of
    wall time (or exactly `steps` calls); the oracle is C behind ctypes, which releases the
    GIL, so the threads run in parallel.  Returns (seconds per call, calls made)."""
    import concurrent.futures as cf
    import threading

    lock = threading.Lock()
    state = {"i": 0, "done": 0}
    t_end = time.perf_counter() + seconds

    def worker():
        while True:
            with lock:
                if (steps is None and time.perf_counter() >= t_end) or (steps is not None and state["i"] >= steps):
                    return
                k = state["i"]
                state["i"] += 1
            calls[k % len(calls)]()
            with lock:
                state["done"] += 1

    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        for f in [ex.submit(worker) for _ in range(threads)]:
            f.result()
    spent = time.perf_counter() - t0
    return spent / max(state["done"], 1), state["done"]


def oracle_sample(w, seconds: float, warmup: int = 1, steps: int | None = None, threads: int = 1):
    """Times the oracle's route + attend of single query heads on one (sequence, KV head) slice of
    the workload drawn on the host (tree built once, not timed).  Decode: the query of the token
    appended at N.  Chunked prefill: queries of the chunk at t = N + i over a tree on the first N
    keys.  Returns (seconds per head-query, head-queries timed, setup seconds)."""
    import torch

    from hierarchical_tree_indexed_b200 import workloads as W
    from oracle import oracle as O

    t0 = time.perf_counter()
    extra = w.steps if w.prefill else 1
    K = torch.zeros((w.N + extra, w.d), dtype=torch.bfloat16)
    V = torch.zeros_like(K)
    cl = W.fill_planted_slice(w.name, 0, 0, w.N, w.d, w.n_clusters, K, V)
    kn, vn = W.background_tokens(w.name, 0, 0, extra, w.d, "cpu", "chunk" if w.prefill else "append")
    K[w.N:], V[w.N:] = kn.to(torch.bfloat16), vn.to(torch.bfloat16)
    qref = W.reference_queries(w.name, w.Hkv, 1, w.d)[0]
    tree = O.build_tree(K, w.N if w.prefill else w.N + 1, w.B, w.b, qref)
    nq = 64
    qs = W.cluster_queries(w.name, 0, 0, w.G, nq, cl, stream="chunk_queries" if w.prefill else "queries")
    qs = qs.to(torch.bfloat16).float().reshape(-1, w.d)
    pos = [w.N + ((k // w.G) * 61) % extra if w.prefill else w.N for k in range(len(qs))]
    setup = time.perf_counter() - t0
    for _ in range(warmup):
        O.decode_query(qs[0], tree, K, V, pos[0], w.p)
    calls = [lambda k=k: O.decode_query(qs[k], tree, K, V, pos[k], w.p) for k in range(len(qs))]
    per, done = time_oracle(calls, seconds, threads, steps)
    return per, done, setup


MARGIN = 1e-4   # index sets must be bit-exact where the oracle's cut margin exceeds this


def oracle_leg(run, w, seconds: float, slices, n_queries: int = 8):
    """The CPU-oracle leg, after the timed region, on the GPU run's own data: for each sampled
    (sequence, KV head) slice the host copies its keys and values, the oracle builds its tree
    (untimed), and then
      * parity: the GPU routes n_queries pool queries at the current N and its index sets are
        compared with the oracle's (bit-exact required where the cut margin exceeds 1e-4; the
        mismatch rate below it is reported);
      * timing: the oracle's route + attend of single query heads over the slices' pool
        queries, on one host core and on every core this process may use."""
    import numpy as np
    import torch

    from oracle import oracle as O
    zha, dev = run.zha, run.dev
    t0 = time.perf_counter()
    torch.cuda.synchronize()
    N = run.N.cpu()
    host, trees = {}, {}
    for (s, h) in slices:
        n = int(N[s])
        host[(s, h)] = (run.K[s, h, :n].cpu(), run.V[s, h, :n].cpu())
        trees[(s, h)] = O.build_tree(host[(s, h)][0], n, w.B, w.b, run.qref[h].cpu())
    setup = time.perf_counter() - t0
    rep = {"queries": 0, "exact_required": 0, "mismatches_required": 0, "low_margin": 0,
           "mismatches_low_margin": 0}
    calls = []
    for j in range(n_queries):
        q = run.Qp[j].reshape(w.batch, 1, w.Hq, w.d).contiguous()
        zha.route(run.cfg, run.tree, q, run.N, run.sel, run.cnt, run.ws)
        torch.cuda.synchronize()
        sel, cnt, qh = run.sel.cpu(), run.cnt.cpu(), q.cpu().float()
        for (s, h) in slices:
            n = int(N[s])
            for hq in range(h * w.G, (h + 1) * w.G):
                rt = O.route(qh[s, 0, hq], trees[(s, h)], w.p)
                g = sel[s, 0, hq, :int(cnt[s, 0, hq])].numpy().astype(np.int64)
                same = len(g) == len(rt.sel) and bool(np.array_equal(g, rt.sel))
                rep["queries"] += 1
                if rt.min_margin > MARGIN:
                    rep["exact_required"] += 1
                    rep["mismatches_required"] += 0 if same else 1
                else:
                    rep["low_margin"] += 1
                    rep["mismatches_low_margin"] += 0 if same else 1
                K_h, V_h = host[(s, h)]
                calls.append(lambda q_=qh[s, 0, hq], t_=trees[(s, h)], K_=K_h, V_=V_h, n_=n:
                             O.decode_query(q_, t_, K_, V_, n_ - 1, w.p))
    run.check_status("the parity sample")
    rep["slices"] = [list(x) for x in slices]
    rep["note"] = (f"{n_queries} pool queries routed on the GPU at the current N, each query head of the sampled "
                   f"slices checked against the fp64 oracle on the same keys; index sets must be bit-exact where the "
                   f"oracle's cut margin exceeds {MARGIN:g}")
    calls[0]()   # warm-up
    per1, done1 = time_oracle(calls, seconds / 2, 1)
    cores = host_cores()
    perN, doneN = time_oracle(calls, seconds / 2, cores)
    cpu = {"value": 1.0 / (perN * w.Hq), "unit": UNIT, "cores": cores, "kind": "oracle",
           "single_core_value": 1.0 / (per1 * w.Hq),
           "sample": f"fp64 C oracle route + attend of single query heads on {len(slices)} (sequence, KV head) slices "
                     f"of {w.name} (the GPU run's keys at N={int(N[slices[0][0]])}, trees built in {setup:.1f}s "
                     f"untimed): {done1} calls on 1 core, {doneN} calls on {cores} threads, scaled to decode "
                     f"queries of all {w.Hq} heads"}
    return cpu, rep


def reference_arm(args, rank):
    if rank.rank != 0:
        return 0
    w = workload(args)
    cores = host_cores()
    # each step is a bounded sample: one call per host thread
    per_head, done, setup = oracle_sample(w, 0.0, warmup=args.warmup, steps=args.steps * cores, threads=cores)
    value = 1.0 / (per_head * w.Hq)
    sample = (f"{done} single-head route+attend calls of the fp64 C oracle on {cores} host threads, on one "
              f"(sequence, KV head) slice of {w.name} (N={w.N}, tree built once in {setup:.1f}s untimed), scaled to "
              f"{'chunk' if w.prefill else 'decode'} queries of all {w.Hq} heads")
    line = {"metric": PREFILL_METRIC if w.prefill else METRIC, "value": value, "unit": UNIT, "impl": "reference",
            "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_head * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": dict(config_dict(w, args.gpus), step="one query head's route + attend in the fp64 oracle"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

class DecodeRun:
    """Device buffers of one decode workload and its three captured phases."""

    def __init__(self, w, dev, N_cap, rank, vsum=False):
        import torch

        from hierarchical_tree_indexed_b200 import workloads as W
        from hierarchical_tree_indexed_b200 import zha
        self.w, self.dev, self.zha = w, dev, zha
        # weak scaling: every rank owns a batch of w.batch sequences of its own
        gen = {}
        if getattr(args_global, "run", 0):
            gen["run"] = args_global.run
        if getattr(args_global, "beta", 0.0):
            gen["beta"] = args_global.beta
        data = W.planted(w, device=dev, N_cap=N_cap, n_queries=POOL, seq_base=rank.rank * w.batch, **gen)
        self.K, self.V, self.Qp, self.knp, self.vnp = data["K"], data["V"], data["Q"], data["k_new"], data["v_new"]
        self.cfg = zha.Config(d=w.d, Hq=w.Hq, Hkv=w.Hkv, B=w.B, b=w.b, batch=w.batch, N_cap=N_cap,
                              dtype=w.dtype, p=w.p, vsum=1 if vsum else 0)
        self.qref = data["qref"]
        cfg = self.cfg
        self.N = torch.full((w.batch,), w.N, dtype=torch.int32, device=dev)
        self.tree = zha.alloc_tree(cfg, dev)
        self.ws = zha.alloc_workspace(cfg, device=dev)
        self.sel = torch.zeros((w.batch, 1, w.Hq, max(N_cap // w.B, 1)), dtype=torch.int32, device=dev)
        self.cnt = torch.zeros((w.batch, 1, w.Hq), dtype=torch.int32, device=dev)
        self.O = torch.zeros((w.batch, 1, w.Hq, w.d), dtype=torch.float32, device=dev)
        self.q_in = torch.empty((w.batch, 1, w.Hq, w.d), dtype=self.K.dtype, device=dev)
        self.k_in = torch.empty((w.batch, w.Hkv, w.d), dtype=self.K.dtype, device=dev)
        self.v_in = torch.empty_like(self.k_in)
        self.rows_v, self.cand_v, self.scan_v = zha.workspace_stats_view(cfg, self.ws)
        zha.get_status(clear=True)
        self.qref_dev = zha.build(cfg, self.K, data["qref"], self.N, self.tree, V=self.V)
        del data
        torch.cuda.synchronize()
        self.load(0)
        self.append(); self.route(); self.attend()
        torch.cuda.synchronize()
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        self.graphs = []
        for fn in (self.append, self.route, self.attend):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                fn()
            self.graphs.append(g)
        # route and attend back to back, one graph: the two kernels the route + attend figure covers
        self.g_ra = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_ra, stream=s):
            self.route(); self.attend()
        # the whole step as one graph: what a decode loop launches
        self.g_step = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_step, stream=s):
            self.append(); self.route(); self.attend()
        self.dense()
        torch.cuda.synchronize()
        self.g_dense = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.g_dense, stream=s):
            self.dense()
        torch.cuda.synchronize()
        self.step = 1

    def load(self, i):
        j = i % POOL
        w = self.w
        self.q_in.copy_(self.Qp[j].reshape(w.batch, 1, w.Hq, w.d))
        self.k_in.copy_(self.knp[j])
        self.v_in.copy_(self.vnp[j])

    def append(self):
        self.zha.append(self.cfg, self.K, self.V, self.k_in, self.v_in, self.N, self.tree)

    def route(self):
        self.zha.route(self.cfg, self.tree, self.q_in, self.N, self.sel, self.cnt, self.ws)

    def attend(self):
        self.zha.attend(self.cfg, self.K, self.V, self.tree, self.q_in, self.N, None, None, self.O, self.ws)

    def dense(self):
        self.zha.dense(self.cfg, self.K, self.V, self.q_in, self.N, self.O, self.ws)

    def check_status(self, what):
        bits = self.zha.get_status(clear=True)
        if bits:
            raise RuntimeError(f"device status after {what}: {self.zha.status_names(bits)}")

    def timed_steps(self, steps, flush, clocks=None):
        """Device times of `steps` decode steps, each the one-graph step (append, route, attend)
        after an L2 flush; then the phases (each its own graph) over min(steps, PHASE_STEPS) more
        steps, for the breakdown; then as many steps of route + attend as one graph (the append
        replayed untimed before each)."""
        import torch
        stream = torch.cuda.current_stream()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        rows_acc = torch.zeros((), dtype=torch.float64, device=self.dev)
        cand_acc = torch.zeros((), dtype=torch.float64, device=self.dev)
        scan_acc = torch.zeros((), dtype=torch.float64, device=self.dev)
        for k in range(steps):
            self.load(self.step)
            self.step += 1
            flush()
            ev[k][0].record(stream)
            self.g_step.replay()
            ev[k][1].record(stream)
            rows_acc += self.rows_v.sum()
            cand_acc += self.cand_v.sum()
            scan_acc += self.scan_v.sum()
        torch.cuda.synchronize()
        self.check_status("the timed steps")
        t_step = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
        n_ph = min(steps, PHASE_STEPS)
        pev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_ph)]
        for k in range(n_ph):
            self.load(self.step)
            self.step += 1
            flush()
            e = pev[k]
            e[0].record(stream)
            for i, g in enumerate(self.graphs):
                g.replay()
                e[i + 1].record(stream)
        # route + attend as one graph, after the step's append (untimed) and an L2 flush
        rev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_ph)]
        for k in range(n_ph):
            self.load(self.step)
            self.step += 1
            flush()
            self.graphs[0].replay()
            rev[k][0].record(stream)
            self.g_ra.replay()
            rev[k][1].record(stream)
        torch.cuda.synchronize()
        self.check_status("the phase steps")
        t = [sum(e[i].elapsed_time(e[i + 1]) for e in pev) / 1e3 * steps / n_ph for i in range(3)]
        t_ra = sum(e[0].elapsed_time(e[1]) for e in rev) / 1e3 * steps / n_ph
        return dict(t_app=t[0], t_route=t[1], t_att=t[2], t_ra=t_ra, t_step=t_step, t_phases=sum(t),
                    rows=rows_acc.item() / steps, cand=cand_acc.item() / steps, scanned=scan_acc.item() / steps)

    def dense_time(self, reps, flush):
        import torch
        stream = torch.cuda.current_stream()
        evs = []
        for _ in range(reps + 2):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream); self.g_dense.replay(); b.record(stream)
            evs.append((a, b))
        torch.cuda.synchronize()
        self.check_status("the dense baseline")
        return sum(a.elapsed_time(b) for a, b in evs[2:]) / reps / 1e3

    def bytes_per_step(self, rows, scanned):
        """Algorithmic bytes of one step: the attention's K and V rows gathered (the union over a
        KV head's query heads) plus q read and O written; the route's tree nodes read (the
        distinct nodes per KV head, 4d + 4 bytes each) plus q; the append's token and its share
        of a leaf block's summary."""
        w = self.w
        es = 2 if w.dtype == "bf16" else 4
        attend = rows * w.d * es * 2 + w.batch * w.Hq * w.d * (es + 4)
        route = scanned * (4 * w.d + 4) + w.batch * w.Hq * w.d * es
        append = w.batch * w.Hkv * (2 * w.d * es + (w.B * w.d * es + (w.d + 1) * 4 * 4) / w.B)
        return attend, route, append


def sweep(args, rank):
    """Tree path vs the in-library dense baseline across context lengths (batch from --batch, 1 by
    default): per N, decode steps (append + route + attend) and dense steps, L2 flushed before each."""
    import dataclasses

    import torch

    from hierarchical_tree_indexed_b200 import dist as D
    from hierarchical_tree_indexed_b200 import workloads as W
    dev = torch.device("cuda", rank.local)
    torch.cuda.set_device(dev)
    base = W.WORKLOADS["decode1m"]
    flush = L2Flush(dev)
    points = []
    for n in [int(x) for x in args.sweep.split(",")]:
        w = dataclasses.replace(base, N=n, n_clusters=max(1, n // 2048), batch=args.batch or 1)
        run = DecodeRun(w, dev, n + args.warmup + args.steps + 2 * min(args.steps, PHASE_STEPS) + 8, rank)
        for _ in range(args.warmup):
            run.load(run.step); run.step += 1
            for g in run.graphs:
                g.replay()
        r = run.timed_steps(args.steps, flush)
        td = run.dense_time(5, flush)
        ms = r["t_step"] / args.steps * 1e3
        points.append({"N": n, "tree_ms": ms, "dense_ms": td * 1e3, "speedup": td * 1e3 / ms,
                       "read_fraction": r["rows"] / (w.batch * w.Hkv * n),
                       "route_ms": r["t_route"] / args.steps * 1e3, "attend_ms": r["t_att"] / args.steps * 1e3})
        del run
        torch.cuda.empty_cache()
    cross = None
    for a_, b_ in zip(points, points[1:]):
        if a_["speedup"] < 1.0 <= b_["speedup"]:
            # log-linear interpolation of the crossover in N
            import math
            fa, fb = math.log(a_["speedup"]), math.log(b_["speedup"])
            x = math.log(a_["N"]) + (0 - fa) * (math.log(b_["N"]) - math.log(a_["N"])) / (fb - fa)
            cross = round(math.exp(x))
    if points and points[0]["speedup"] >= 1.0:
        cross = f"<= {points[0]['N']}"
    if rank.leader:
        print(json.dumps({"metric": "decode step time, tree path vs in-library dense baseline", "unit": "ms",
                          "batch": args.batch or 1, "steps": args.steps, "points": points,
                          "crossover_N": cross}), flush=True)
    D.finish(rank)
    return 0


def prefill_main(args, rank, w):
    """One step = one chunk of w.steps queries per sequence over a tree on the first N keys:
    zha_route + zha_attend with n_q = w.steps (each one CUDA graph), L2 flushed before each."""
    import torch

    from hierarchical_tree_indexed_b200 import dist as D
    from hierarchical_tree_indexed_b200 import workloads as W
    from hierarchical_tree_indexed_b200 import zha

    dev = torch.device("cuda", rank.local)
    torch.cuda.set_device(dev)
    D.init(rank, "nccl")
    n_q, Np = w.steps, w.N
    N_cap = Np + n_q
    data = W.planted(w, device=dev, N_cap=N_cap, n_queries=n_q, seq_base=rank.rank * w.batch)
    K, V = data["K"], data["V"]
    K[:, :, Np:] = data["k_new"].permute(1, 2, 0, 3)
    V[:, :, Np:] = data["v_new"].permute(1, 2, 0, 3)
    Q = data["Q"].permute(1, 0, 2, 3).contiguous()
    qref = data["qref"]
    del data
    cfg = zha.Config(d=w.d, Hq=w.Hq, Hkv=w.Hkv, B=w.B, b=w.b, batch=w.batch, N_cap=N_cap, dtype=w.dtype, p=w.p)
    N = torch.full((w.batch,), N_cap, dtype=torch.int32, device=dev)
    tree = zha.alloc_tree(cfg, dev)
    ws = zha.alloc_workspace(cfg, n_q, device=dev)
    sel_cap = Np // w.B
    sel = torch.zeros((w.batch, n_q, w.Hq, sel_cap), dtype=torch.int32, device=dev)
    cnt = torch.zeros((w.batch, n_q, w.Hq), dtype=torch.int32, device=dev)
    O = torch.zeros((w.batch, n_q, w.Hq, w.d), dtype=torch.float32, device=dev)
    Od = torch.zeros_like(O)
    steps_v, cand_v, _ = zha.workspace_stats_view(cfg, ws, n_q)
    zha.get_status(clear=True)
    zha.build(cfg, K, qref, torch.full((w.batch,), Np, dtype=torch.int32, device=dev), tree)

    def do_route():
        zha.route(cfg, tree, Q, N, sel, cnt, ws, n_q=n_q)

    def do_attend():
        zha.attend(cfg, K, V, tree, Q, N, sel, cnt, O, ws, n_q=n_q)

    def do_dense():
        zha.dense(cfg, K, V, Q, N, Od, ws, n_q=n_q)

    for fn in (do_route, do_attend, do_dense):
        fn()
    torch.cuda.synchronize()
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    graphs = []
    for fn in (do_route, do_attend, do_dense):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            fn()
        graphs.append(g)
    torch.cuda.synchronize()
    g_route, g_att, g_dense = graphs
    flush = L2Flush(dev)
    for _ in range(args.warmup):
        g_route.replay(); g_att.replay()
    torch.cuda.synchronize()
    bits = zha.get_status(clear=True)
    if bits:
        raise RuntimeError(f"device status after warm-up: {zha.status_names(bits)}")
    stream = torch.cuda.current_stream()
    K_steps = args.steps
    D.barrier(rank, dev)
    torch.cuda.synchronize()
    clocks = Clocks(rank.local) if rank.leader else None
    time.sleep(0.25)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K_steps)]
    for k in range(K_steps):
        flush()
        e = ev[k]
        e[0].record(stream); g_route.replay(); e[1].record(stream); g_att.replay(); e[2].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None
    bits = zha.get_status(clear=True)
    if bits:
        raise RuntimeError(f"device status after the timed steps: {zha.status_names(bits)}")
    t_route = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_att = sum(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    t_step = t_route + t_att
    D.barrier(rank, dev)
    t_max = D.max_over_ranks(t_step, rank, dev)
    queries = w.batch * n_q * K_steps * rank.world
    value = queries / t_max
    # work of the method: every (query, head) row attends over |I(q)| keys (QK and PV,
    # 2 flops per multiply-add each); the tensor cores load `steps` 64-key blocks for 128 rows
    blocks = cnt.to(torch.int64).sum().item()
    tail = sum((Np - (Np // w.B) * w.B) + i + 1 for i in range(n_q)) * w.batch * w.Hq
    # rows whose block 0 was not selected still read key 0 (the sink)
    sink = ((cnt == 0) | (sel[..., 0] != 0)).sum().item() if Np >= w.B else 0
    keys = blocks * w.B + tail + sink
    useful_flops = keys * w.d * 4
    issued_flops = steps_v.to(torch.int64).sum().item() * 128 * 64 * w.d * 4
    peak, peak_src = measured_peaks("bf16_tflops_sustained")
    att_tflops = useful_flops / (t_att / K_steps) / 1e12
    issued_tflops = issued_flops / (t_att / K_steps) / 1e12
    # dense causal prefill, same kernel without the selection
    dense_ev = []
    for _ in range(5):
        flush()
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream); g_dense.replay(); b_.record(stream)
        dense_ev.append((a_, b_))
    torch.cuda.synchronize()
    t_dense = sum(a_.elapsed_time(b_) for a_, b_ in dense_ev[1:]) / 4 / 1e3
    dense_flops = sum(Np + i + 1 for i in range(n_q)) * w.batch * w.Hq * w.d * 4
    # the pages' U_p(W), with S_p(q) read as the routed set: the union of the blocks the last W
    # chunk queries selected, as a fraction of the prefix's blocks (mean over (sequence, query head))
    n1 = Np // w.B
    coverage = {}
    for W_ in (1, 16, 256, n_q):
        fr = []
        for s_ in range(w.batch):
            for hq in range(w.Hq):
                c = cnt[s_, n_q - W_:, hq].to(torch.int64)
                ids = sel[s_, n_q - W_:, hq]
                mask = torch.arange(ids.shape[1], device=dev)[None, :] < c[:, None]
                u = torch.zeros(n1, dtype=torch.bool, device=dev)
                u[ids[mask].long()] = True
                fr.append(u.sum().item() / n1)
        coverage[str(W_)] = sum(fr) / len(fr)
    # causal chunk insertion: the chunk in block-aligned sub-chunks; before each, zha_extend indexes
    # the chunk's blocks completed so far, so query t routes over exactly the blocks before its own
    causal = None
    if w.batch == 1 and Np % w.B == 0:
        subs = [(i0, min(i0 + w.B, n_q)) for i0 in range(0, n_q, w.B)]
        ws_sub = zha.alloc_workspace(cfg, w.B, device=dev)
        Oc = torch.zeros_like(O)
        N_tree = [torch.full((1,), Np + i0, dtype=torch.int32, device=dev) for i0, _ in subs]
        N_end = [torch.full((1,), Np + i1, dtype=torch.int32, device=dev) for _, i1 in subs]

        def causal_chunk():
            zha.build(cfg, K, qref, N_tree[0], tree)
            for k, (i0, i1) in enumerate(subs):
                if k:
                    zha.extend(cfg, K, N_tree[k], tree)
                zha.route(cfg, tree, Q[:, i0:i1], N_end[k], sel[:, i0:i1], cnt[:, i0:i1], ws_sub, n_q=i1 - i0)
                zha.attend(cfg, K, V, tree, Q[:, i0:i1], N_end[k], sel[:, i0:i1], cnt[:, i0:i1], Oc[:, i0:i1],
                           ws_sub, n_q=i1 - i0)
        causal_chunk()
        torch.cuda.synchronize()
        gc_ = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gc_, stream=s):
            causal_chunk()
        torch.cuda.synchronize()
        cev = []
        for _ in range(4):
            flush()
            a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a_.record(stream); gc_.replay(); b_.record(stream)
            cev.append((a_, b_))
        torch.cuda.synchronize()
        bits = zha.get_status(clear=True)
        if bits:
            raise RuntimeError(f"device status after the causal chunk: {zha.status_names(bits)}")
        t_c = sum(a_.elapsed_time(b_) for a_, b_ in cev[1:]) / 3 / 1e3
        causal = {"ms_per_chunk": t_c * 1e3, "queries_per_s": n_q / t_c, "sub_chunks": len(subs),
                  "note": "tree rebuilt on the prefix then extended block by block (zha_extend), each sub-chunk "
                          "routed and attended over the tree of the keys before it; timed including the rebuild"}
        del gc_
        zha.build(cfg, K, qref, torch.full((w.batch,), Np, dtype=torch.int32, device=dev), tree)
    # end to end: host Q and chunk K/V in, O out, through the public calls
    e2e = None
    if not args.no_e2e:
        e2e_steps = max(1, min(K_steps, 10))
        qh = Q.cpu().pin_memory()
        kh = K[:, :, Np:].cpu().pin_memory()
        vh = V[:, :, Np:].cpu().pin_memory()
        oh = torch.empty_like(O, device="cpu").pin_memory()
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for k in range(E2E_WARMUP + e2e_steps):
            if k == E2E_WARMUP:   # untimed warm-up steps first
                torch.cuda.synchronize()
                a_.record(stream)
            Q.copy_(qh, non_blocking=True)
            K[:, :, Np:].copy_(kh, non_blocking=True)
            V[:, :, Np:].copy_(vh, non_blocking=True)
            do_route()
            do_attend()
            oh.copy_(O, non_blocking=True)
        b_.record(stream)
        torch.cuda.synchronize()
        t_e2e = D.max_over_ranks(a_.elapsed_time(b_) / 1e3, rank, dev)
        e2e = {"value": w.batch * n_q * e2e_steps * rank.world / t_e2e, "unit": UNIT,
               "h2d_bytes_per_step": qh.numel() * 2 + kh.numel() * 2 + vh.numel() * 2,
               "d2h_bytes_per_step": oh.numel() * 4, "steps": e2e_steps,
               "note": "zha_route + zha_attend per chunk (not graphed) after 3 untimed chunks, pinned host Q, chunk K/V and O"}
    cpu = None
    if rank.leader and rank.world == 1 and not args.no_cpu_baseline:
        per1, done1, setup = oracle_sample(w, args.cpu_seconds / 2)
        cores = host_cores()
        perN, doneN, _ = oracle_sample(w, args.cpu_seconds / 2, threads=cores)
        cpu = {"value": 1.0 / (perN * w.Hq), "unit": UNIT, "cores": cores, "kind": "oracle",
               "single_core_value": 1.0 / (per1 * w.Hq),
               "sample": f"single-head route+attend calls of the fp64 C oracle for chunk queries of one (sequence, KV "
                         f"head) slice of {w.name} drawn on the host (tree built once, {setup:.1f}s untimed): {done1} "
                         f"calls on 1 core, {doneN} on {cores} threads, scaled to chunk queries of all {w.Hq} heads"}
    if rank.leader:
        line = {
            "metric": PREFILL_METRIC, "value": value, "unit": UNIT, "n_gpus": rank.world, "steps": K_steps,
            "warmup": args.warmup, "ms_per_step": t_max / K_steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{w.name}: batch {w.batch} per GPU, {w.Hq} query / {w.Hkv} KV heads, d {w.d}, "
                                   f"bf16, prefix N={Np} in the tree, chunk of {n_q} causal queries, leaf block "
                                   f"{w.B}, branching {w.b}, p={w.p}",
                       "global_batch": w.batch * rank.world, "seq_len": N_cap, "parallelism": f"dp{rank.world}",
                       "l2": L2Flush.NOTE,
                       "step": "zha_route + zha_attend of one chunk, each one CUDA graph"},
            "roofline": {"bound": "tensor", "kernel": "attend phase (plan + attend_prefill_kernel + merge)",
                         "achieved": att_tflops, "peak": peak, "unit": "TFLOP/s", "frac": att_tflops / peak,
                         "traffic": None, "peak_source": f"{peak_src} bf16 dense (sustained)",
                         "algorithmic_flops_per_launch": useful_flops, "issued_mma_flops_per_launch": issued_flops,
                         "issued_tflops": issued_tflops},
            "phases_ms": {"route": t_route / K_steps * 1e3, "attend": t_att / K_steps * 1e3},
            "keys_per_row": keys / (w.batch * n_q * w.Hq),
            "coverage_U_W": coverage,
            "causal_chunk": causal,
            "dense_baseline": {"ms_per_step": t_dense * 1e3, "tflops": dense_flops / t_dense / 1e12,
                               "queries_per_s": w.batch * n_q / t_dense,
                               "speedup_of_tree": t_dense / (t_max / K_steps)},
            "gpu_launches": 8 * K_steps,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    del graphs, g_route, g_att, g_dense
    D.finish(rank)
    return 0


def value_summary_report(run, args, queries=8, ps=(None, 0.8, 0.5)):
    """Relative L2 error against dense attention of the decode outputs with and without the
    dropped subtrees' value summaries, on the same queries and the same cache, for a few p
    (None = the workload's).  The tree without summaries is built apart (its layout differs)."""
    import dataclasses

    import torch

    zha, w = run.zha, run.w
    cfg_v = run.cfg
    cfg_0 = dataclasses.replace(cfg_v, vsum=0)
    tree_0 = zha.alloc_tree(cfg_0, run.dev)
    q_keep = zha.build(cfg_0, run.K, run.qref, run.N, tree_0)
    ws_0 = zha.alloc_workspace(cfg_0, device=run.dev)
    out = {}
    for p in ps:
        pv = w.p if p is None else p
        cv, c0 = dataclasses.replace(cfg_v, p=pv), dataclasses.replace(cfg_0, p=pv)
        ev, e0 = [], []
        for j in range(queries):
            q = run.Qp[j].reshape(w.batch, 1, w.Hq, w.d).contiguous()
            ov, o0, od = (torch.zeros_like(run.O) for _ in range(3))
            zha.route(cv, run.tree, q, run.N, run.sel, run.cnt, run.ws)
            zha.attend(cv, run.K, run.V, run.tree, q, run.N, None, None, ov, run.ws)
            zha.route(c0, tree_0, q, run.N, run.sel, run.cnt, ws_0)
            zha.attend(c0, run.K, run.V, tree_0, q, run.N, None, None, o0, ws_0)
            zha.dense(c0, run.K, run.V, q, run.N, od, ws_0)
            nd = od.norm(dim=-1)
            ev.append(((ov - od).norm(dim=-1) / nd).mean().item())
            e0.append(((o0 - od).norm(dim=-1) / nd).mean().item())
        out[str(pv)] = {"with": sum(ev) / len(ev), "without": sum(e0) / len(e0)}
    torch.cuda.synchronize()
    run.check_status("the value-summary report")
    del q_keep
    return {"error_vs_dense": out, "queries": queries * w.batch * w.Hq,
            "note": "mean over (query, head) of |o - o_dense| / |o_dense|, decode queries of the workload"}


args_global = None   # the parsed command line (generator overrides read by the workload helpers)


def main():
    global args_global
    args = parse()
    args_global = args
    from hierarchical_tree_indexed_b200 import dist as D
    rank = D.from_env()
    if args.impl == "reference":
        return reference_arm(args, rank)
    if args.sweep:
        return sweep(args, rank)
    if workload(args).prefill:
        return prefill_main(args, rank, workload(args))

    import torch

    from hierarchical_tree_indexed_b200 import zha

    dev = torch.device("cuda", rank.local)
    torch.cuda.set_device(dev)
    D.init(rank, "nccl")
    w = workload(args)
    K_steps, W_steps = args.steps, args.warmup
    e2e_steps = 0 if args.no_e2e else min(K_steps, 500)
    N_cap = w.N + W_steps + K_steps + 2 * min(K_steps, PHASE_STEPS) + E2E_WARMUP + e2e_steps + 8
    run = DecodeRun(w, dev, N_cap, rank, vsum=args.vsum)
    flush = L2Flush(dev)
    for _ in range(W_steps):
        run.load(run.step)
        run.step += 1
        for g in run.graphs:
            g.replay()
    torch.cuda.synchronize()
    run.check_status("warm-up")

    D.barrier(rank, dev)
    torch.cuda.synchronize()
    clocks = Clocks(rank.local) if rank.leader else None
    time.sleep(0.25)
    r = run.timed_steps(K_steps, flush)
    clk = clocks.stop() if clocks else None
    D.barrier(rank, dev)
    t_max = D.max_over_ranks(r["t_step"], rank, dev)
    queries = w.batch * K_steps * rank.world
    value = queries / t_max

    attend_bytes, route_bytes, append_bytes = run.bytes_per_step(r["rows"], r["scanned"])
    step_bytes = attend_bytes + route_bytes + append_bytes
    peak, peak_src = measured_peaks()
    att_gbs = attend_bytes / (r["t_att"] / K_steps) / 1e9
    step_gbs = step_bytes / (r["t_step"] / K_steps) / 1e9
    ra_gbs = (attend_bytes + route_bytes) / (r["t_ra"] / K_steps) / 1e9
    read_fraction = r["rows"] / (w.batch * w.Hkv * w.N)
    khash = source_hash(ATTEND_SOURCES)
    tr = profiled_traffic(khash)
    traffic = (tr[0] * r["rows"] + tr[1]) if tr else None

    t_dense = run.dense_time(8, flush)
    es = 2 if w.dtype == "bf16" else 4
    dense_gbs = (w.batch * w.Hkv * int(run.N[0].item()) * w.d * es * 2) / t_dense / 1e9

    vsum_report = value_summary_report(run, args) if args.vsum else None

    # ---- end to end through the public C-ABI call with host buffers
    e2e = None
    if e2e_steps:
        stream = torch.cuda.current_stream()
        # one step's inputs (q, k_new, v_new) sit side by side in one pinned host row and one device
        # buffer, so each step is one host-to-device copy; the calls take views of that buffer
        nq, nk = w.batch * w.Hq * w.d, w.batch * w.Hkv * w.d
        sh = torch.empty((POOL, nq + 2 * nk), dtype=run.K.dtype).pin_memory()
        sh[:, :nq].copy_(run.Qp.reshape(POOL, nq).cpu())
        sh[:, nq:nq + nk].copy_(run.knp.reshape(POOL, nk).cpu())
        sh[:, nq + nk:].copy_(run.vnp.reshape(POOL, nk).cpu())
        sd = torch.empty((nq + 2 * nk,), dtype=run.K.dtype, device=dev)
        q_e = sd[:nq].view(w.batch, 1, w.Hq, w.d)
        k_e = sd[nq:nq + nk].view(w.batch, w.Hkv, w.d)
        v_e = sd[nq + nk:].view(w.batch, w.Hkv, w.d)
        oh = torch.empty((E2E_WARMUP + e2e_steps, w.batch, 1, w.Hq, w.d), dtype=torch.float32).pin_memory()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for k in range(E2E_WARMUP + e2e_steps):
            if k == E2E_WARMUP:   # untimed warm-up steps first
                torch.cuda.synchronize()
                D.barrier(rank, dev)
                a.record(stream)
            sd.copy_(sh[k % POOL], non_blocking=True)
            zha.decode(run.cfg, run.K, run.V, run.tree, q_e, k_e, v_e, run.N, run.O, run.ws)
            oh[k].copy_(run.O, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        t_e2e = D.max_over_ranks(a.elapsed_time(b) / 1e3, rank, dev)
        e2e = {"value": w.batch * e2e_steps * rank.world / t_e2e, "unit": UNIT,
               "h2d_bytes_per_step": sd.numel() * es,
               "d2h_bytes_per_step": run.O.numel() * 4, "steps": e2e_steps,
               "note": "zha_decode per step (not graphed) after 3 untimed steps; the step's q, k_new, v_new in one pinned "
                       "host row copied in once, O copied out; L2 not flushed"}
        run.check_status("the e2e steps")

    cpu, parity = None, None
    if rank.leader and rank.world == 1 and not args.no_cpu_baseline:
        cpu, parity = oracle_leg(run, w, args.cpu_seconds, [(0, 0), (w.batch - 1, w.Hkv - 1)])

    if rank.leader:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": rank.world, "steps": K_steps,
            "warmup": W_steps, "ms_per_step": t_max / K_steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {**config_dict(w, rank.world), **({"value_summaries": True} if args.vsum else {})},
            "hbm_gbs": step_gbs, "hbm_frac_of_peak": step_gbs / peak, "hbm_frac_of_nominal": step_gbs / NOMINAL_HBM_GBS,
            "roofline": {"bound": "hbm", "kernel": run.zha.attend_kernel(run.cfg), "achieved": att_gbs, "peak": peak,
                         "unit": "GB/s", "frac": att_gbs / peak, "traffic": traffic,
                         "peak_source": f"{peak_src} copy bandwidth", "algorithmic_bytes_per_launch": attend_bytes,
                         "frac_of_nominal": att_gbs / NOMINAL_HBM_GBS, "frac_of_dense_kernel": att_gbs / dense_gbs,
                         "kernel_source_sha256_16": khash},
            "route_attend": {"gbs": ra_gbs, "frac_of_peak": ra_gbs / peak, "frac_of_nominal": ra_gbs / NOMINAL_HBM_GBS,
                             "frac_of_dense_kernel": ra_gbs / dense_gbs, "bytes": attend_bytes + route_bytes,
                             "ms": r["t_ra"] / K_steps * 1e3,
                             "ms_phases_apart": (r["t_route"] + r["t_att"]) / K_steps * 1e3,
                             "note": "route (plan fused) and attend as one CUDA graph after the step's append and an "
                                     "L2 flush, over the algorithmic bytes: distinct tree nodes read, K and V rows "
                                     "gathered, q and O (ms_phases_apart: the two phases each in its own graph)"},
            "phases_ms": {"append": r["t_app"] / K_steps * 1e3, "route": r["t_route"] / K_steps * 1e3,
                          "attend": r["t_att"] / K_steps * 1e3},
            "bytes_per_step": {"attend": attend_bytes, "route": route_bytes, "append": append_bytes},
            "route_nodes": {"distinct_per_step": r["scanned"], "per_head_sum_per_step": r["cand"]},
            "read_fraction": read_fraction,
            "value_summaries": vsum_report,
            "dense_baseline": {"ms_per_step": t_dense * 1e3, "hbm_gbs": dense_gbs,
                               "queries_per_s": w.batch / t_dense, "speedup_of_tree": t_dense / (t_max / K_steps)},
            "gpu_launches": 3 * K_steps,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "parity": parity,
        }
        print(json.dumps(line), flush=True)
    del run
    D.finish(rank)
    return 0


if __name__ == "__main__":
    sys.exit(main())
