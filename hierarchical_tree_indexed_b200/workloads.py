"""Seeded synthetic workloads for the tree-indexed sparse attention path.

This module only draws random inputs: keys, values, queries and reference
queries.  It holds none of the method's arithmetic (no summaries, scores,
routing or attention), so both the CUDA path and the CPU oracle can take their
inputs from it.

Every (workload, sequence, KV head, stream) draws from its own seed, derived
with numpy's ``SeedSequence(0, spawn_key=...)``, so any slice can be
regenerated on its own.  Large arrays are drawn with ``torch`` on the device
they are created on; small discrete choices (cluster positions, Zipf picks,
permutations) are drawn with numpy on the host.  A given device type always
yields the same values for the same seed; CPU and CUDA streams differ, so a
comparison always feeds both sides the very same tensors.

Workload shapes follow the pages' setting: decode over a long KV cache with
grouped-query attention, keys with a few strongly attended regions ("needle"
retrieval, the narrow-lookup case of "Subquadratic Attention with a
Hierarchical Tree-Structured Indexer", §Variable Sparsity Across Tasks).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

# Reference queries are drawn for this many levels, whatever the depth, so
# that the values for level l never depend on N.
MAX_LEVELS = 16

_WORKLOAD_IDS = {"tiny": 0, "decode128k": 1, "decode1m": 2, "prefill256k": 3, "decode8m": 4,
                 "test": 5}
_STREAMS = {"keys": 0, "values": 1, "clusters": 2, "queries": 3, "append": 4, "qref": 5,
            "chunk": 6, "chunk_queries": 7}

# Planted-cluster constants.  SHIFT is the workload's "keys shifted toward a
# random unit direction x3".  RUN (w, keys per cluster) and BETA (query aim
# strength) were calibrated with the oracle on the 1M workload so that the
# fraction of the cache read lands in the 1-6 % band.
SHIFT = 3.0
RUN = 8192
BETA = 48.0
ZIPF_S = 1.1


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    Hq: int
    Hkv: int
    d: int
    N: int              # keys in the cache when decode starts (prefill: prefix length)
    B: int              # leaf block
    b: int              # branching factor
    p: float            # top-p threshold at every level
    dtype: str          # "bf16" or "f32"
    n_clusters: int = 0
    steps: int = 1      # decode steps (tokens appended), or the prefill chunk length
    R: int = 1
    prefill: bool = False
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 64, 4096, 16, 4, 0.9, "f32", steps=8),
    "decode128k": Workload("decode128k", 1, 32, 8, 128, 131072, 64, 16, 0.95, "bf16",
                           n_clusters=64, steps=1024),
    "decode1m": Workload("decode1m", 4, 32, 8, 128, 1048576, 64, 16, 0.95, "bf16",
                         n_clusters=512, steps=64),
    "prefill256k": Workload("prefill256k", 1, 32, 8, 128, 262144, 64, 16, 0.95, "bf16",
                            n_clusters=128, steps=4096, prefill=True),
    "decode8m": Workload("decode8m", 1, 32, 8, 128, 8388608, 64, 16, 0.95, "bf16",
                         n_clusters=4096, steps=256),
}


def seed_for(workload: str, seq: int, kv_head: int, stream: str) -> int:
    """64-bit seed of one (workload, sequence, KV head, stream) slice."""
    ss = np.random.SeedSequence(0, spawn_key=(_WORKLOAD_IDS[workload], seq, kv_head,
                                              _STREAMS[stream]))
    return int(ss.generate_state(1, np.uint64)[0] & np.uint64(0x7FFFFFFFFFFFFFFF))


def _torch_gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(seed)
    return g


def zipf_weights(n: int, s: float = ZIPF_S) -> np.ndarray:
    """Probabilities of ranks 1..n under a Zipf(s) law truncated to n ranks."""
    w = np.arange(1, n + 1, dtype=np.float64) ** (-s)
    return w / w.sum()


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def reference_queries(workload: str, Hkv: int, R: int, d: int, device="cpu") -> torch.Tensor:
    """q-hat[h][level][r][d], i.i.d. N(0, 1)/sqrt(d), fp32, for MAX_LEVELS levels."""
    out = torch.empty((Hkv, MAX_LEVELS, R, d), dtype=torch.float32, device=device)
    for h in range(Hkv):
        g = _torch_gen(seed_for(workload, 0, h, "qref"), device)
        out[h] = torch.randn((MAX_LEVELS, R, d), generator=g, device=device) / math.sqrt(d)
    return out


# ----------------------------------------------------------------------------- tiny

def tiny(device="cpu") -> dict:
    """The small fp32 case: 1 KV head, 1 query head, d=64, N=4096.

    Keys and values i.i.d. N(0,1).  Eight queries q = 4*k_j + noise (std 0.5),
    j drawn from a Zipf(1.1) law over the positions, rank -> position through a
    seeded permutation.
    """
    w = WORKLOADS["tiny"]
    N, d = w.N, w.d
    gk = _torch_gen(seed_for("tiny", 0, 0, "keys"), device)
    gv = _torch_gen(seed_for("tiny", 0, 0, "values"), device)
    gq = _torch_gen(seed_for("tiny", 0, 0, "queries"), device)
    K = torch.randn((1, 1, N, d), generator=gk, device=device)
    V = torch.randn((1, 1, N, d), generator=gv, device=device)
    rng = np.random.default_rng(seed_for("tiny", 0, 0, "clusters"))
    perm = rng.permutation(N)
    ranks = rng.choice(N, size=w.steps, p=zipf_weights(N))
    pos = perm[ranks]
    noise = 0.5 * torch.randn((w.steps, d), generator=gq, device=device)
    Q = 4.0 * K[0, 0, torch.as_tensor(pos, device=device)] + noise
    return dict(workload=w, K=K, V=V, Q=Q.reshape(w.steps, 1, 1, d).contiguous(),
                positions=pos, qref=reference_queries("tiny", 1, 1, d, device), N=N)


# ------------------------------------------------------------------ planted clusters

@dataclass
class SliceClusters:
    directions: torch.Tensor   # [M, d] fp32 unit vectors
    starts: np.ndarray         # [M] first key of each run
    perm: np.ndarray           # rank -> cluster id


def slice_clusters(workload: str, seq: int, kv: int, N: int, d: int, M: int, run: int,
                   device) -> SliceClusters:
    rng = np.random.default_rng(seed_for(workload, seq, kv, "clusters"))
    starts = rng.integers(1, max(2, N - run + 1), size=M)
    perm = rng.permutation(M)
    g = _torch_gen(seed_for(workload, seq, kv, "clusters"), device)
    u = torch.randn((M, d), generator=g, device=device)
    u = u / torch.linalg.vector_norm(u, dim=1, keepdim=True)
    return SliceClusters(u, starts, perm)


def fill_planted_slice(workload: str, seq: int, kv: int, N: int, d: int, M: int,
                       K_out: torch.Tensor, V_out: torch.Tensor, run: int = RUN,
                       shift: float = SHIFT) -> SliceClusters:
    """Writes keys/values [0, N) of one (sequence, KV head) slice into K_out/V_out.

    K_out, V_out: [>= N, d] views (fp32 or bf16) on any device.  Keys are
    N(0, I) with M runs of `run` contiguous keys shifted by shift*u_c.
    """
    device = K_out.device
    cl = slice_clusters(workload, seq, kv, N, d, M, run, device)
    gk = _torch_gen(seed_for(workload, seq, kv, "keys"), device)
    gv = _torch_gen(seed_for(workload, seq, kv, "values"), device)
    k = torch.randn((N, d), generator=gk, device=device)
    for c in range(M):
        s = int(cl.starts[c])
        e = min(N, s + run)
        k[s:e] += shift * cl.directions[c]
    K_out[:N].copy_(k)
    del k
    V_out[:N].copy_(torch.randn((N, d), generator=gv, device=device))
    return cl


def cluster_queries(workload: str, seq: int, kv: int, G: int, n: int, cl: SliceClusters,
                    beta: float = BETA, stream: str = "queries") -> torch.Tensor:
    """n x G queries [n, G, d] fp32: beta * sum of 1-4 chosen directions + N(0, I)."""
    device = cl.directions.device
    M, d = cl.directions.shape
    rng = np.random.default_rng(seed_for(workload, seq, kv, stream))
    zw = zipf_weights(M)
    sel = torch.zeros((n * G, M), dtype=torch.float32)
    for i in range(n * G):
        cnt = int(rng.integers(1, 5))
        chosen: list[int] = []
        while len(chosen) < min(cnt, M):
            c = int(cl.perm[rng.choice(M, p=zw)])
            if c not in chosen:
                chosen.append(c)
        sel[i, chosen] = 1.0
    g = _torch_gen(seed_for(workload, seq, kv, stream), device)
    noise = torch.randn((n * G, d), generator=g, device=device)
    q = beta * (sel.to(device) @ cl.directions) + noise
    return q.reshape(n, G, d)


def background_tokens(workload: str, seq: int, kv: int, n: int, d: int, device,
                      stream: str = "append") -> tuple[torch.Tensor, torch.Tensor]:
    """n appended (k, v) pairs [n, d] fp32 from the background law N(0, I)."""
    g = _torch_gen(seed_for(workload, seq, kv, stream), device)
    k = torch.randn((n, d), generator=g, device=device)
    v = torch.randn((n, d), generator=g, device=device)
    return k, v


def planted(w: Workload, device="cpu", N_cap: int | None = None, seqs=None, kv_heads=None,
            n_queries: int | None = None, run: int = RUN, beta: float = BETA, seq_base: int = 0) -> dict:
    """Generates a planted-cluster workload.

    Returns K, V [batch][Hkv][N_cap][d] (w.dtype), the decode queries
    Q [n_queries][batch][Hq][d] (w.dtype), the appended tokens
    k_new/v_new [n_queries][batch][Hkv][d], and the reference queries.
    `seqs`/`kv_heads` restrict which slices are filled (others stay zero);
    sequence s is drawn from the seeds of sequence seq_base + s.
    """
    N_cap = N_cap or (w.N + (0 if w.prefill else w.steps))
    n_queries = w.steps if n_queries is None else n_queries
    dt = torch_dtype(w.dtype)
    K = torch.zeros((w.batch, w.Hkv, N_cap, w.d), dtype=dt, device=device)
    V = torch.zeros_like(K)
    Q = torch.zeros((n_queries, w.batch, w.Hq, w.d), dtype=dt, device=device)
    k_new = torch.zeros((n_queries, w.batch, w.Hkv, w.d), dtype=dt, device=device)
    v_new = torch.zeros_like(k_new)
    seqs = range(w.batch) if seqs is None else seqs
    kv_heads = range(w.Hkv) if kv_heads is None else kv_heads
    clusters = {}
    for s in seqs:
        for h in kv_heads:
            sg = seq_base + s
            cl = fill_planted_slice(w.name, sg, h, w.N, w.d, w.n_clusters, K[s, h], V[s, h], run)
            clusters[(s, h)] = cl
            if n_queries:
                stream = "chunk_queries" if w.prefill else "queries"
                q = cluster_queries(w.name, sg, h, w.G, n_queries, cl, beta, stream)
                Q[:, s, h * w.G:(h + 1) * w.G] = q.to(dt)
                kn, vn = background_tokens(w.name, sg, h, n_queries, w.d, device,
                                           "chunk" if w.prefill else "append")
                k_new[:, s, h] = kn.to(dt)
                v_new[:, s, h] = vn.to(dt)
    return dict(workload=w, K=K, V=V, Q=Q, k_new=k_new, v_new=v_new, N=w.N, N_cap=N_cap,
                qref=reference_queries(w.name, w.Hkv, w.R, w.d, device), clusters=clusters)
