"""Seeded synthetic inputs for the SSA forward workloads.

This module holds random-number generation only: none of the layer's
arithmetic.  Both the CUDA path and the CPU oracle are fed from it.

Recipe (one generator per workload, seed = 1000 + workload id):
  * draws are standard normal float32, taken one batch element at a time in
    the order Q, K noise, V, block centroids (clustered workloads only),
    needle noise;
  * clustered keys: k_j = centroid(block of j) + 0.3 * noise_j, centroids and
    noise N(0, 1), a centroid per (batch, block, kv-head), or per run of
    `cluster_span` consecutive blocks when that is above 1 (keys whose nearby
    blocks are alike);
  * planted needles: a query row i (query head h) and an earlier key j of the
    kv-head serving h get k_j = 4 * q_i / ||q_i|| * sqrt(d) + N(0, 0.1) noise
    (variance 0.1).  Placement comes from a NumPy generator with the same
    seed: i uniform in [W + B, n), j uniform in [0, i - W) so the needle is
    outside the query's window and in a fully visible block; (j, kv-head)
    pairs are distinct.  Decode workloads plant at the single new query;
  * finally Q, K, V are cast to the workload dtype (bf16 by round to nearest
    even).

Random streams are device specific: the same seed gives different numbers on
``cpu`` and ``cuda``.  Small parity cases are drawn on the CPU and copied to
the GPU; full-size cases are drawn on the GPU and sampled back to the host.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, asdict

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int
    batch: int
    n: int
    h_q: int
    h_kv: int
    d: int
    dtype: str          # "f32" | "bf16"
    block: int
    sigma: str          # "diag" | "full"
    topk: int
    window: int
    needles: int        # total needles (per head or per sequence: see needle_mode)
    needle_mode: str    # "total" | "per_head" | "per_seq"
    clustered: bool = False
    decode: bool = False
    beta: float = 2.0
    subblocks: int = 1  # summaries per block (sub-block max-pool routing when > 1)
    cluster_span: int = 1   # consecutive blocks sharing a centroid (clustered keys)
    outlier: bool = False   # route with the outlier-channel row per block

    @property
    def n_q(self) -> int:
        return 1 if self.decode else self.n

    @property
    def q_offset(self) -> int:
        return self.n - 1 if self.decode else 0

    def scaled(self, **kw) -> "Workload":
        """Same structure with some sizes overridden (small parity variants)."""
        d = asdict(self)
        d.update(kw)
        return Workload(**d)


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_fp32_4k", 0, 1, 4096, 1, 1, 64, "f32", 64, "full", 8, 64, 32, "total"),
        Workload("mha_bf16_32k", 1, 1, 32768, 8, 8, 128, "bf16", 64, "diag", 32, 128, 256, "per_head"),
        Workload("decode_bf16_64x256k", 2, 64, 262144, 32, 8, 128, "bf16", 64, "diag", 32, 256, 16,
                 "per_seq", decode=True),
        Workload("gqa_bf16_128k", 3, 1, 131072, 32, 8, 128, "bf16", 64, "diag", 32, 256, 1024, "total",
                 clustered=True),
        Workload("gqa_bf16_1m", 4, 1, 1048576, 8, 1, 128, "bf16", 128, "diag", 16, 256, 4096, "total",
                 clustered=True),
    ]
}


def _needle_plan(w: Workload, rng: np.random.Generator):
    """List of (batch, query row, query head, key row) needle placements."""
    G = w.h_q // w.h_kv
    plans = []
    used = set()

    def place(bi, head, i):
        for _ in range(64):
            hi = i - w.window
            if hi <= 0:
                return
            j = int(rng.integers(0, hi))
            key = (bi, j, head // G)
            if key not in used:
                used.add(key)
                plans.append((bi, i if not w.decode else 0, head, j))
                return

    lo = w.window + w.block
    if w.decode:
        for bi in range(w.batch):
            for _ in range(w.needles):
                place(bi, int(rng.integers(0, w.h_q)), w.n - 1)
        return plans
    if w.n <= lo:
        return plans
    if w.needle_mode == "per_head":
        for bi in range(w.batch):
            for head in range(w.h_q):
                for _ in range(w.needles):
                    place(bi, head, int(rng.integers(lo, w.n)))
    else:
        for _ in range(w.needles):
            place(int(rng.integers(0, w.batch)), int(rng.integers(0, w.h_q)), int(rng.integers(lo, w.n)))
    return plans


def make_inputs(w: Workload, device="cpu", seed: int | None = None):
    """Q [b, n_q, h_q, d], K/V [b, n, h_kv, d] in the workload dtype, plus the
    needle plan.  Memory is bounded by drawing one batch element at a time:
    for each batch element, in order, Q, K noise, V, centroids (clustered
    workloads) and the needle noise are drawn from the one generator."""
    seed = 1000 + w.wid if seed is None else seed
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(seed)
    rng = np.random.default_rng(seed)
    out_dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    G = w.h_q // w.h_kv
    plan = _needle_plan(w, rng)

    def draw(shape):
        return torch.randn(*shape, generator=gen, device=dev, dtype=torch.float32)

    Q = torch.empty(w.batch, w.n_q, w.h_q, w.d, device=dev, dtype=out_dt)
    K = torch.empty(w.batch, w.n, w.h_kv, w.d, device=dev, dtype=out_dt)
    V = torch.empty(w.batch, w.n, w.h_kv, w.d, device=dev, dtype=out_dt)
    for bi in range(w.batch):
        Qb = draw((w.n_q, w.h_q, w.d)).to(out_dt)
        Q[bi] = Qb
        Kb = draw((w.n, w.h_kv, w.d))
        V[bi] = draw((w.n, w.h_kv, w.d)).to(out_dt)
        if w.clustered:
            span = w.block * w.cluster_span
            cent = draw(((w.n + span - 1) // span, w.h_kv, w.d))
            Kb = cent.repeat_interleave(span, dim=0)[:w.n] + 0.3 * Kb
            del cent
        mine = [p for p in plan if p[0] == bi]
        if mine:
            pi = torch.tensor([p[1] for p in mine], device=dev)
            ph = torch.tensor([p[2] for p in mine], device=dev)
            pj = torch.tensor([p[3] for p in mine], device=dev)
            qv = Qb[pi, ph].to(torch.float32)       # the query as the layer sees it
            noise = draw((len(mine), w.d)) * math.sqrt(0.1)
            Kb[pj, ph // G] = 4.0 * qv / qv.norm(dim=1, keepdim=True) * math.sqrt(w.d) + noise
        K[bi] = Kb.to(out_dt)
        del Kb, Qb
    return Q, K, V, plan


def problem_dict(w: Workload) -> dict:
    """Layer parameters of a workload (argument names of the C struct)."""
    return dict(batch=w.batch, n_q=w.n_q, n_kv=w.n, h_q=w.h_q, h_kv=w.h_kv, d=w.d,
                block=w.block, topk=w.topk, window=w.window, q_offset=w.q_offset,
                beta=w.beta, scale=1.0 / math.sqrt(w.d), dtype=w.dtype, sigma=w.sigma,
                subblocks=w.subblocks, outlier=w.outlier)
