"""The bench's bookkeeping of algorithmic work, on the CPU: the attended key
count per (row, kv-head) equals the size of the oracle's key set, and the
block-major slot and block counts equal a direct count of the used entries
(the ones the kernels take: in range, larger than every earlier entry)."""
import os
import sys

import numpy as np
import torch

from content_routed_block_ssa_b200.workload import WORKLOADS, make_inputs, problem_dict
from oracle import ssa_oracle as O

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _case():
    w = WORKLOADS["gqa_bf16_128k"].scaled(n=1536, needles=12, window=200)
    Q, K, V, _ = make_inputs(w, "cpu")
    p = O.Problem(**problem_dict(w))
    stored = O.stored_summaries(*O.block_summaries(K.float().numpy(), p), p)
    idx, _ = O.route_topk(Q.float().numpy(), stored, p)
    return w, p, idx


def test_attended_keys_is_the_key_set_size():
    w, p, idx = _case()
    got = bench.attended_keys(torch.from_numpy(idx), w).numpy()
    for i in range(0, w.n_q, 7):
        for g in range(w.h_kv):
            assert got[0, i, g] == len(O.key_set(p.q_offset + i, idx[0, i, g], p)), (i, g)


def test_block_major_counts_by_direct_count():
    w, p, idx = _case()
    bad = idx.copy()
    bad[0, 100, 0, 3] = bad[0, 100, 0, 2]       # a repeat and an out-of-range entry are not used
    bad[0, 200, 1, 5] = p.nb + 3
    for arr in (idx, bad):
        n_e, n_b = bench.block_major_counts(torch.from_numpy(arr), w)
        used, blocks = 0, set()
        for i in range(w.n_q):
            nvis = O.visible_blocks(p.q_offset + i, p)
            for g in range(w.h_kv):
                last = -1
                for v in arr[0, i, g]:
                    if 0 <= v < nvis and v > last:
                        used += 1
                        blocks.add((g, int(v)))
                    if 0 <= v < nvis:
                        last = max(last, int(v))
        assert (n_e, n_b) == (used, len(blocks))


def test_kernel_report_fractions_and_dominant_stage():
    """On a synthetic result the report's achieved rates are the algorithmic
    work over the stage time, its fractions those rates over the peaks, and
    the dominant stage the longest bounded one (decode state excluded)."""
    w, p, idx = _case()
    work = bench.algorithmic_work(w, torch.from_numpy(idx))
    ms = {"summary": 0.5, "route": 2.0, "attn_plan": 0.1, "attn_blocks": 4.0, "attn_window": 0.3,
          "attn_merge": 1.0}
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    rep = bench.kernel_report(w, {"ms_kernels": ms, "work": work}, peaks, {})
    for name in ("summary", "attn_plan", "attn_merge"):
        e = rep[name]
        assert abs(e["achieved"] - e["algorithmic_bytes"] / (ms[name] * 1e-3) / 1e9) < 1e-6 * e["achieved"]
        assert abs(e["frac"] - e["achieved"] / 6000.0) < 1e-12
    r = rep["route"]
    assert r["bound"] == "tensor" and abs(r["achieved"] - work["route_flops"] / 2e-3 / 1e12) < 1e-9 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / 1400.0) < 1e-12
    name, d = bench.dominant(rep)
    assert name == "attn_blocks" and d["ms"] == 4.0
    assert bench.dominant(rep, exclude=("attn_blocks",))[0] == "route"
