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


def _direct_slots(arr, w, p):
    """The slot rule written out row by row: used entries; the hot blocks of
    each kv-head (count over every 8th row >= the smallest
    T >= 2 that leaves at most 128 of them) are paired two at a time in
    block order."""
    from collections import Counter
    used_rows = {}
    cnt = Counter()
    for i in range(w.n_q):
        nvis = O.visible_blocks(p.q_offset + i, p)
        for g in range(w.h_kv):
            last, used = -1, []
            for v in arr[0, i, g]:
                if 0 <= v < nvis and v > last:
                    used.append(int(v))
                if 0 <= v < nvis:
                    last = max(last, int(v))
            used_rows[(i, g)] = used
            if i % 8 == 0:
                cnt.update((g, c) for c in used)
    n_e = sum(len(u) for u in used_rows.values())
    hot = {}
    for g in range(w.h_kv):
        counts = [cnt[(g, c)] for c in range(w.n // w.block)]
        T = 2
        while sum(x >= T for x in counts) > 128:
            T += 1
        hot[g] = [c for c, x in enumerate(counts) if x >= T]
    n_s, keys = 0, set()
    for (i, g), used in used_rows.items():
        hs = [c for c in used if c in hot[g]]
        npair = len(hs) // 2
        pairs = [(hs[2 * m], hs[2 * m + 1]) for m in range(npair)]
        paired = set(hs[:2 * npair])
        singles = [c for c in used if c not in paired]
        n_s += npair + len(singles)
        keys.update((g, "p", a, b) for a, b in pairs)
        keys.update((g, "s", c) for c in singles)
    return n_e, n_s, len(keys)


def test_block_major_counts_by_direct_count():
    w, p, idx = _case()
    bad = idx.copy()
    rng = np.random.default_rng(5)
    bad[rng.random(bad.shape) < 0.05] = 10 ** 6
    bad[rng.random(bad.shape) < 0.05] = 0
    for arr in (idx, bad):
        got = bench.block_major_counts(torch.from_numpy(arr), w)
        assert got == _direct_slots(arr, w, p)
        assert got[1] < got[0]          # some entries pair up
    # 128-key blocks pair the same way
    w2 = w.scaled(block=128)
    p2 = O.Problem(**problem_dict(w2))
    arr2 = np.where(idx >= 0, idx // 2, idx)
    got2 = bench.block_major_counts(torch.from_numpy(arr2), w2)
    assert got2 == _direct_slots(arr2, w2, p2) and got2[1] < got2[0]
    # a block chosen only by rows the hot-set count skips is not hot: sampled
    # and full counts give different slot totals here
    arr3 = idx.copy()
    arr3[:, :, :, :] = -1
    arr3[0, 700:720, 0, 0] = 3          # rows 700..719 (704, 712 sampled): blocks 3 and 5
    arr3[0, 700:720, 0, 1] = 5
    arr3[0, 701, 0, 2] = 7              # blocks 7 and 9: rows 701 and 703, never sampled
    arr3[0, 703, 0, 2] = 7
    arr3[0, 701, 0, 3] = 9
    arr3[0, 703, 0, 3] = 9
    got3 = bench.block_major_counts(torch.from_numpy(arr3), w)
    assert got3 == _direct_slots(arr3, w, p)
    # 3 and 5 are hot (two sampled rows each), 7 and 9 are not: 20 pairs + 4 singles
    assert got3 == (44, 24, 3)


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
    # the tiles are rated on the method's flops; the design's bytes ride along
    for name, key in (("attn_blocks", "blocks_flops"), ("attn_window", "window_flops")):
        e = rep[name]
        assert e["bound"] == "tensor" and e["algorithmic_flops"] == work[key]
        assert abs(e["achieved"] - work[key] / (ms[name] * 1e-3) / 1e12) < 1e-9 * e["achieved"]
        assert abs(e["frac"] - e["achieved"] / 1400.0) < 1e-12
        dt = e["design_traffic"]
        assert abs(dt["achieved"] - dt["algorithmic_bytes"] / (ms[name] * 1e-3) / 1e9) < 1e-6 * dt["achieved"]
    # per selected slot the block tiles do 4 G B d flops (S = Q K^T, O = P V)
    G = w.h_q // w.h_kv
    assert work["blocks_flops"] == 4.0 * work["n_entries"] * G * w.block * w.d
    name, d = bench.dominant(rep)
    assert name == "attn_blocks" and d["ms"] == 4.0
    assert bench.dominant(rep, exclude=("attn_blocks",))[0] == "route"


def test_layer_report_against_both_roofs():
    """The layer line: method flops (route scores + attention over the
    attended keys) and compulsory bytes over the step time, recomputed here
    from the definitions."""
    w, p, idx = _case()
    work = bench.algorithmic_work(w, torch.from_numpy(idx))
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    lay = bench.layer_report(w, work, 2.0, peaks)
    S = bench.attended_keys(torch.from_numpy(idx), w).sum().item()
    G = w.h_q // w.h_kv
    nvis = sum(min(w.n // w.block, (i + 1) // w.block) for i in range(w.n_q))
    flops = 4.0 * S * G * w.d + 2.0 * 2 * w.d * nvis * w.h_kv
    assert abs(lay["method_flops"] - flops) < 1e-9 * flops
    assert abs(lay["frac_tensor"] - flops / 2e-3 / 1e12 / 1400.0) < 1e-12
    nb = w.n // w.block
    nbytes = (2 * w.n_q * w.h_q * w.d * 2 + 2 * w.n * w.h_kv * w.d * 2 + w.n_q * w.h_q * 4
              + 2 * w.h_kv * nb * 2 * w.d * 2 + 2 * w.n_q * w.h_kv * w.topk * 4)
    assert lay["compulsory_bytes"] == nbytes
    assert abs(lay["frac_hbm"] - nbytes / 2e-3 / 1e9 / 6000.0) < 1e-12


def test_clock_sampler_follows_the_device_uuid(monkeypatch):
    """With CUDA_VISIBLE_DEVICES remapping, CUDA device 0 may be nvidia-smi's
    GPU 5: the sampler is pointed at the index whose UUID matches; with no
    match (or no properties) it keeps the CUDA ordinal."""
    class Props:
        uuid = "0f1e2d3c-4b5a-6978-8796-a5b4c3d2e1f0"
    listing = ("0, GPU-11111111-2222-3333-4444-555555555555\n"
               "5, GPU-0F1E2D3C-4B5A-6978-8796-A5B4C3D2E1F0\n")
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda d: Props())
    assert bench.smi_index(0, listing) == 5
    assert bench.smi_index(0, "0, GPU-11111111-2222-3333-4444-555555555555\n") == 0
    assert bench.smi_index(2, "") == 2

    def fail(d):
        raise RuntimeError("no device")
    monkeypatch.setattr(torch.cuda, "get_device_properties", fail)
    assert bench.smi_index(1, listing) == 1
