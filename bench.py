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

Prints one JSON line on rank 0.  Times are CUDA-event device times on the
launching stream (max over ranks); L2 is flushed (256 MiB write) before every
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
UNIT = "queries/s"
FALLBACK_HBM_GBS = 6650.0
POOL = 64                 # distinct (q, k_new, v_new) sets cycled through by the steps
ATTEND_SOURCES = ["hierarchical_tree_indexed_b200/csrc/zha_attend.cuh",
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
    return {"workload": f"{w.name}: batch {w.batch} per GPU, {w.Hq} query / {w.Hkv} KV heads, d {w.d}, "
                        f"bf16 K/V, N={w.N}, leaf block {w.B}, branching {w.b}, p={w.p}",
            "global_batch": w.batch * world, "seq_len": w.N, "parallelism": f"dp{world}",
            "kv_dtype": w.dtype, "l2": "flushed (256 MiB write) before every timed step; KV 16 GiB > L2",
            "step": "append + route + attend, each phase one CUDA graph"}


def measured_peaks() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


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

def oracle_sample(w, seconds: float, warmup: int = 1, steps: int | None = None):
    """Times the oracle's route + attend of single query heads on one (sequence, KV head)
    slice of the workload (tree built once, not timed).  Returns (seconds per head-query,
    head-queries timed, setup seconds)."""
    import torch

    from hierarchical_tree_indexed_b200 import workloads as W
    from oracle import oracle as O

    t0 = time.perf_counter()
    K = torch.zeros((w.N + 1, w.d), dtype=torch.bfloat16)
    V = torch.zeros_like(K)
    cl = W.fill_planted_slice(w.name, 0, 0, w.N, w.d, w.n_clusters, K, V)
    kn, vn = W.background_tokens(w.name, 0, 0, 1, w.d, "cpu")
    K[w.N], V[w.N] = kn[0].to(torch.bfloat16), vn[0].to(torch.bfloat16)
    qref = W.reference_queries(w.name, w.Hkv, 1, w.d)[0]
    tree = O.build_tree(K, w.N + 1, w.B, w.b, qref)
    qs = W.cluster_queries(w.name, 0, 0, w.G, 64, cl).to(torch.bfloat16).float().reshape(-1, w.d)
    setup = time.perf_counter() - t0
    done, spent, i = 0, 0.0, 0
    for _ in range(warmup):
        O.decode_query(qs[0], tree, K, V, w.N, w.p)
    while (steps is None and spent < seconds) or (steps is not None and done < steps):
        q = qs[i % len(qs)]
        i += 1
        t = time.perf_counter()
        O.decode_query(q, tree, K, V, w.N, w.p)
        spent += time.perf_counter() - t
        done += 1
    return spent / done, done, setup


def reference_arm(args, rank):
    if rank.rank != 0:
        return 0
    w = workload(args)
    per_head, done, setup = oracle_sample(w, 0.0, warmup=args.warmup, steps=args.steps)
    value = 1.0 / (per_head * w.Hq)
    sample = (f"{done} single-head route+attend calls of the fp64 C oracle on one (sequence, KV head) "
              f"slice of {w.name} (N={w.N}, tree built once in {setup:.1f}s untimed), scaled to decode "
              f"queries of all {w.Hq} heads")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_head * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": dict(config_dict(w, args.gpus), step="one query head's route + attend in the fp64 oracle"),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm

def main():
    args = parse()
    from hierarchical_tree_indexed_b200 import dist as D
    rank = D.from_env()
    if args.impl == "reference":
        return reference_arm(args, rank)

    import torch

    from hierarchical_tree_indexed_b200 import workloads as W
    from hierarchical_tree_indexed_b200 import zha

    dev = torch.device("cuda", rank.local)
    torch.cuda.set_device(dev)
    D.init(rank, "nccl")
    w = workload(args)
    K_steps, W_steps = args.steps, args.warmup
    e2e_steps = 0 if args.no_e2e else min(K_steps, 500)
    N_cap = w.N + W_steps + K_steps + e2e_steps + 8
    # weak scaling: every rank owns a batch of w.batch sequences of its own
    data = W.planted(w, device=dev, N_cap=N_cap, n_queries=POOL, seq_base=rank.rank * w.batch)
    K, V, Qp, knp, vnp = data["K"], data["V"], data["Q"], data["k_new"], data["v_new"]
    cfg = zha.Config(d=w.d, Hq=w.Hq, Hkv=w.Hkv, B=w.B, b=w.b, batch=w.batch, N_cap=N_cap, dtype=w.dtype, p=w.p)
    N = torch.full((w.batch,), w.N, dtype=torch.int32, device=dev)
    tree = zha.alloc_tree(cfg, dev)
    ws = zha.alloc_workspace(cfg, device=dev)
    sel = torch.zeros((w.batch, 1, w.Hq, max(N_cap // w.B, 1)), dtype=torch.int32, device=dev)
    cnt = torch.zeros((w.batch, 1, w.Hq), dtype=torch.int32, device=dev)
    O = torch.zeros((w.batch, 1, w.Hq, w.d), dtype=torch.float32, device=dev)
    q_in = torch.empty((w.batch, 1, w.Hq, w.d), dtype=K.dtype, device=dev)
    k_in = torch.empty((w.batch, w.Hkv, w.d), dtype=K.dtype, device=dev)
    v_in = torch.empty_like(k_in)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rows_v, cand_v = zha.workspace_stats_view(cfg, ws)
    zha.get_status(clear=True)

    qref_dev = zha.build(cfg, K, data["qref"], N, tree)
    torch.cuda.synchronize()

    def load_inputs(i):
        j = i % POOL
        q_in.copy_(Qp[j].reshape(w.batch, 1, w.Hq, w.d))
        k_in.copy_(knp[j])
        v_in.copy_(vnp[j])

    def do_append():
        zha.append(cfg, K, V, k_in, v_in, N, tree)

    def do_route():
        zha.route(cfg, tree, q_in, N, sel, cnt, ws)

    def do_attend():
        zha.attend(cfg, K, V, tree, q_in, N, None, None, O, ws)

    # one untimed pass outside capture (kernel attributes), then capture each phase in a graph
    load_inputs(0)
    do_append(); do_route(); do_attend()
    torch.cuda.synchronize()
    graphs = []
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    for fn in (do_append, do_route, do_attend):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            fn()
        graphs.append(g)
    torch.cuda.synchronize()
    g_app, g_route, g_att = graphs

    stream = torch.cuda.current_stream()
    for i in range(W_steps):
        load_inputs(i + 1)
        g_app.replay(); g_route.replay(); g_att.replay()
    torch.cuda.synchronize()
    bits = zha.get_status(clear=True)
    if bits:
        raise RuntimeError(f"device status after warm-up: {zha.status_names(bits)}")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K_steps)]
    rows_acc = torch.zeros((), dtype=torch.float64, device=dev)
    cand_acc = torch.zeros((), dtype=torch.float64, device=dev)
    D.barrier(rank, dev)
    torch.cuda.synchronize()
    clocks = Clocks(rank.local) if rank.leader else None
    time.sleep(0.25)
    for k in range(K_steps):
        load_inputs(W_steps + 1 + k)
        flush.zero_()
        e = ev[k]
        e[0].record(stream)
        g_app.replay()
        e[1].record(stream)
        g_route.replay()
        e[2].record(stream)
        g_att.replay()
        e[3].record(stream)
        rows_acc += rows_v.sum()
        cand_acc += cand_v.sum()
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None
    D.barrier(rank, dev)
    bits = zha.get_status(clear=True)
    if bits:
        raise RuntimeError(f"device status after the timed steps: {zha.status_names(bits)}")

    t_app = sum(e[0].elapsed_time(e[1]) for e in ev) / 1e3
    t_route = sum(e[1].elapsed_time(e[2]) for e in ev) / 1e3
    t_att = sum(e[2].elapsed_time(e[3]) for e in ev) / 1e3
    t_step = sum(e[0].elapsed_time(e[3]) for e in ev) / 1e3
    t_max = D.max_over_ranks(t_step, rank, dev)
    queries = w.batch * K_steps * rank.world
    value = queries / t_max

    # ---- algorithmic bytes (bf16 K/V, fp32 summaries)
    es = 2 if w.dtype == "bf16" else 4
    rows_mean = rows_acc.item() / K_steps                    # keys gathered per step, all groups
    cand_mean = cand_acc.item() / K_steps                    # tree nodes scored per step, all heads
    attend_bytes = rows_mean * w.d * es * 2 + w.batch * w.Hq * w.d * (es + 4)
    route_bytes = cand_mean * (4 * w.d + 4) + w.batch * w.Hq * w.d * es
    append_bytes = w.batch * w.Hkv * (2 * w.d * es + (w.B * w.d * es + (w.d + 1) * 4 * 4) / w.B)
    step_bytes = attend_bytes + route_bytes + append_bytes
    peak, peak_src = measured_peaks()
    att_gbs = attend_bytes / (t_att / K_steps) / 1e9
    step_gbs = step_bytes / (t_step / K_steps) / 1e9
    read_fraction = rows_mean / (w.batch * w.Hkv * w.N)
    khash = source_hash(ATTEND_SOURCES)
    tr = profiled_traffic(khash)
    traffic = (tr[0] * rows_mean + tr[1]) if tr else None

    # ---- dense baseline at the same N (in-library, same loader)
    def do_dense():
        zha.dense(cfg, K, V, q_in, N, O, ws)
    do_dense()
    torch.cuda.synchronize()
    gd = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gd, stream=s):
        do_dense()
    dense_ev = []
    for k in range(10):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream); gd.replay(); b.record(stream)
        dense_ev.append((a, b))
    torch.cuda.synchronize()
    t_dense = sum(a.elapsed_time(b) for a, b in dense_ev[2:]) / len(dense_ev[2:]) / 1e3
    dense_rows = w.batch * w.Hkv * int(N[0].item())
    dense_gbs = (dense_rows * w.d * es * 2) / t_dense / 1e9

    # ---- end to end through the public C-ABI call with host buffers
    e2e = None
    if e2e_steps:
        qh = torch.empty((POOL, w.batch, 1, w.Hq, w.d), dtype=K.dtype).pin_memory()
        qh.copy_(Qp.reshape(POOL, w.batch, 1, w.Hq, w.d).cpu())
        kh = knp.cpu().pin_memory()
        vh = vnp.cpu().pin_memory()
        oh = torch.empty((e2e_steps, w.batch, 1, w.Hq, w.d), dtype=torch.float32).pin_memory()
        torch.cuda.synchronize()
        D.barrier(rank, dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for k in range(e2e_steps):
            j = k % POOL
            q_in.copy_(qh[j], non_blocking=True)
            k_in.copy_(kh[j], non_blocking=True)
            v_in.copy_(vh[j], non_blocking=True)
            zha.decode(cfg, K, V, tree, q_in, k_in, v_in, N, O, ws)
            oh[k].copy_(O, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        t_e2e = D.max_over_ranks(a.elapsed_time(b) / 1e3, rank, dev)
        e2e = {"value": w.batch * e2e_steps * rank.world / t_e2e, "unit": UNIT,
               "h2d_bytes_per_step": (q_in.numel() + k_in.numel() + v_in.numel()) * es,
               "d2h_bytes_per_step": O.numel() * 4, "steps": e2e_steps,
               "note": "zha_decode per step (not graphed), pinned host inputs/outputs, L2 not flushed"}
        bits = zha.get_status(clear=True)
        if bits:
            raise RuntimeError(f"device status after the e2e steps: {zha.status_names(bits)}")

    cpu = None
    if rank.leader and rank.world == 1 and not args.no_cpu_baseline:
        per_head, done, setup = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": 1.0 / (per_head * w.Hq), "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{done} single-head route+attend calls of the fp64 C oracle on one (sequence, KV head) "
                         f"slice of {w.name} (tree built once, {setup:.1f}s untimed), scaled to decode queries "
                         f"of all {w.Hq} heads"}

    if rank.leader:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": rank.world, "steps": K_steps,
            "warmup": W_steps, "ms_per_step": t_max / K_steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_dict(w, rank.world),
            "hbm_gbs": step_gbs, "hbm_frac_of_peak": step_gbs / peak,
            "roofline": {"bound": "hbm", "kernel": "attend_kernel", "achieved": att_gbs, "peak": peak,
                         "unit": "GB/s", "frac": att_gbs / peak, "traffic": traffic,
                         "peak_source": f"{peak_src} copy bandwidth", "algorithmic_bytes_per_launch": attend_bytes,
                         "kernel_source_sha256_16": khash},
            "phases_ms": {"append": t_app / K_steps * 1e3, "route": t_route / K_steps * 1e3,
                          "attend": t_att / K_steps * 1e3},
            "bytes_per_step": {"attend": attend_bytes, "route": route_bytes, "append": append_bytes},
            "read_fraction": read_fraction,
            "dense_baseline": {"ms_per_step": t_dense * 1e3, "hbm_gbs": dense_gbs,
                               "queries_per_s": w.batch / t_dense, "speedup_of_tree": t_dense / (t_max / K_steps)},
            "gpu_launches": 4 * K_steps,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    del qref_dev
    D.finish(rank)
    return 0


if __name__ == "__main__":
    sys.exit(main())
