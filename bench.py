"""Benchmark of the SSA forward on B200: query-heads/s at 128K (and 1M) tokens.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-secondary] [--no-cpu-baseline] [--no-e2e]
                    [--subblocks S] [--outlier] [--router flat|hier [--fanout M] [--probe P] [--escalate] [--levels L]]
                    [--cluster-span S]

One step is one pass of the whole layer over the workload's synthetic input:
block summaries -> routing features + tensor-core route with fused top-k ->
exact attention (block-major: plan, block tiles, window tiles, merge), each a
call of the libssa C ABI on the current stream (ssa_forward issues the same
calls).  Inputs are resident in HBM when the timed region starts; L2 is
flushed between steps.  Step time is the sum of CUDA-event intervals around
the step's kernels, the reported time the max over ranks.  With N > 1 every
rank runs its own replica of the workload (independent problems, no
collective on the data path): weak scaling.  The decode workload's block
summaries (and, with --router hier, its node store) are precomputed state of
the cache: built once before the timed steps and reported beside them.  The
line gives the mean and the median step time, and the dominant kernel's
roofline fraction against the measured peaks and the nominal ones.  SM
clocks and throttle reasons are sampled by nvidia-smi every 100 ms during
the timed steps, on the GPU whose UUID is the CUDA device's (nvidia-smi's
index can differ from the CUDA ordinal under CUDA_VISIBLE_DEVICES).

`e2e` repeats the step through ssa_forward_hostio with page-locked host
inputs and outputs, every step's host<->device copies inside the timed
region; consecutive steps go round-robin to up to three streams (each with its
own device buffer), so one step's copies overlap the others' compute.

`--impl reference` times the CPU oracle (float64 NumPy) on a bounded sample of
the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from content_routed_block_ssa_b200.workload import WORKLOADS, make_inputs, problem_dict  # noqa: E402

METRIC = "SSA fwd query-heads/s at 128K and 1M; % HBM BW (gather) / % TC peak (route)"
UNIT = "query-heads/s"
PRIMARY = "gqa_bf16_128k"
SECONDARY = "gqa_bf16_1m"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# FP32 FMA peak for ALU-bound kernels: 148 SMs x 128 FP32 lanes x 2 flop x 1.965 GHz.
FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# nominal datasheet peaks, for context beside the measured ones
NOMINAL = {"GB/s": 7700.0, "TFLOP/s": 2250.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "of measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "of fallback"


def load_traffic():
    """Per-launch DRAM bytes of the dominant kernels from the committed ncu summary."""
    out = {}
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return out
    for line in open(path):
        parts = line.split()
        if len(parts) == 3 and not line.startswith("#"):
            out[(parts[0], parts[1])] = float(parts[2])
    return out


# ------------------------------------------------------------------ distributed

def dist_setup(n_gpus, backend=None):
    """One process per GPU (torchrun sets RANK / LOCAL_RANK / WORLD_SIZE).
    The layer has no exchange step: ranks run independent replicas and only
    meet for the barriers and the max-over-ranks of the timings (NCCL on the
    GPUs; gloo when there is no GPU, which the CPU tests use)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, ws):
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank, ws, ms_max):
    """Units all ranks processed per second over the slowest rank's time
    (weak scaling: every rank runs the full workload)."""
    return ws * units_per_rank / (ms_max / 1e3)


# ------------------------------------------------------------------ clocks

def smi_index(device, listing=None):
    """The nvidia-smi index of CUDA device `device` (which may differ from
    the CUDA ordinal when CUDA_VISIBLE_DEVICES remaps devices): matched by
    UUID against `nvidia-smi --query-gpu=index,uuid` (or `listing`, its
    output, for tests); the CUDA ordinal when nothing matches."""
    try:
        uuid = str(torch.cuda.get_device_properties(device).uuid).lower()
        uuid = uuid[4:] if uuid.startswith("gpu-") else uuid
        if listing is None:
            listing = subprocess.run(["nvidia-smi", "--query-gpu=index,uuid", "--format=csv,noheader"],
                                     capture_output=True, text=True, timeout=20).stdout
        for line in listing.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) == 2 and uuid and f[1].lower().removeprefix("gpu-") == uuid:
                return int(f[0])
    except Exception:
        pass
    return int(device)


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "smi_index": self.gpu}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "smi_index": self.gpu}


# ------------------------------------------------------------------ algorithmic work

def attended_keys(idx, w):
    """|S_i| per (batch, row, kv-head): selected blocks' keys plus window keys
    outside them (bookkeeping for the roofline, not part of the layer)."""
    B, W = w.block, w.window
    pos = torch.arange(w.n_q, device=idx.device, dtype=torch.int64).view(1, -1, 1, 1) + w.q_offset
    lo = torch.clamp(pos - W + 1, min=0)
    valid = idx >= 0
    c = idx.to(torch.int64)
    ov_lo = torch.maximum(c * B, lo)
    ov_hi = torch.minimum(c * B + B - 1, pos)
    overlap = torch.where(valid, torch.clamp(ov_hi - ov_lo + 1, min=0), torch.zeros_like(c)).sum(-1)
    n_sel = valid.sum(-1).to(torch.int64)
    wcount = (pos - lo + 1).squeeze(-1)
    return n_sel * B + wcount - overlap


HOT_BLOCKS = 128   # hot set size of the paired slots
HOT_SAMPLE = 8     # the hot set is counted over every 8th query row


def block_major_counts(idx, w):
    """Selected slots of the block-major attention, by the kernels' rules
    (bookkeeping for the roofline, not part of the layer).  A row's used
    entries are its in-range block_idx entries larger than every earlier
    in-range entry.  The entries of each (batch, kv-head)'s hot blocks (its
    at most HOT_BLOCKS most selected blocks, counted over every
    HOT_SAMPLE-th query row: count >= T for the smallest T >= 2 that keeps
    the set that small) pair up in block order, two per slot; other entries
    are a slot each.  Returns (used entries, slots, distinct tile keys: pairs
    and single blocks)."""
    nb = w.n // w.block
    B = w.block
    pos = torch.arange(w.n_q, device=idx.device, dtype=torch.int64).view(1, -1, 1, 1) + w.q_offset
    nvis = torch.clamp((pos + 1) // B, max=nb)
    v = idx.to(torch.int64)
    inr = (v >= 0) & (v < nvis)
    run = torch.cummax(torch.where(inr, v, torch.full_like(v, -1)), dim=-1).values
    prev = torch.cat([torch.full_like(run[..., :1], -1), run[..., :-1]], dim=-1)
    valid = inr & (v > prev)
    sel = torch.where(valid, v, torch.zeros_like(v))
    n_entries = int(valid.sum().item())
    bgi = (torch.arange(w.batch, device=idx.device).view(-1, 1, 1, 1) * w.h_kv
           + torch.arange(w.h_kv, device=idx.device).view(1, 1, -1, 1)).expand_as(v)
    gkey = bgi * nb + sel
    bgs = w.batch * w.h_kv
    rows = torch.arange(w.n_q, device=idx.device).view(1, -1, 1, 1)
    sampled = valid & (rows % HOT_SAMPLE == 0)
    cnt = torch.bincount(gkey[sampled], minlength=bgs * nb).view(bgs, nb)
    srt = cnt.sort(dim=1, descending=True).values
    c129 = srt[:, HOT_BLOCKS] if nb > HOT_BLOCKS else torch.zeros(bgs, dtype=cnt.dtype, device=cnt.device)
    T = torch.clamp(c129 + 1, min=2)
    hot_blk = cnt >= T[:, None]
    hid_tab = torch.where(hot_blk, torch.cumsum(hot_blk.to(torch.int64), dim=1) - 1, torch.full_like(cnt, -1))
    hid = torch.where(valid, hid_tab.view(-1)[gkey], torch.full_like(v, -1))
    hot = hid >= 0
    nhot = hot.sum(-1, keepdim=True)
    npair = nhot // 2
    n_slots = n_entries - int(npair.sum().item())
    # pair keys: the hot entries in order, taken two at a time
    order = torch.sort((~hot).to(torch.int8), dim=-1, stable=True).indices
    hs = hid.gather(-1, order)
    m = torch.arange(v.shape[-1] // 2, device=v.device)
    first, second = hs[..., 0::2][..., :m.numel()], hs[..., 1::2][..., :m.numel()]
    is_pair = m < npair
    pkey = (bgi[..., :m.numel()] * (nb + HOT_BLOCKS * HOT_BLOCKS) + nb + first * HOT_BLOCKS + second)[is_pair]
    rank = torch.cumsum(hot.to(torch.int64), dim=-1) - 1
    single = valid & ~(hot & (rank < 2 * npair))
    skey = (bgi * (nb + HOT_BLOCKS * HOT_BLOCKS) + sel)[single]
    n_keys = int(torch.unique(torch.cat([pkey, skey])).numel())
    return n_entries, n_slots, n_keys


def algorithmic_work(w, idx):
    es = 4 if w.dtype == "f32" else 2
    nb = w.n // w.block
    G = w.h_q // w.h_kv
    pos = np.arange(w.n_q) + w.q_offset
    nvis = np.minimum(nb, (pos + 1) // w.block).sum()
    # one summary row and one routing dot product per sub-block (float32:
    # mu and Sigma rows, d + d^2 for a full Sigma)
    R = w.subblocks + (1 if w.outlier else 0)      # summary rows per block
    summary_bytes = w.batch * w.n * w.h_kv * w.d * es + w.batch * w.h_kv * nb * R * 2 * w.d * 2
    route_flops = 2.0 * (2 * w.d) * float(nvis) * R * w.h_kv * w.batch
    if w.dtype == "f32":
        per = w.d + (w.d * w.d if w.sigma == "full" else w.d)
        route_flops = 2.0 * per * float(nvis) * R * w.h_q * w.batch
        summary_bytes = w.batch * w.n * w.h_kv * w.d * es + w.batch * w.h_kv * nb * per * 4
    route_table_bytes = float(nvis) * R * w.h_kv * w.batch * 2 * w.d * 2
    S = attended_keys(idx, w)
    gathered = float(S.sum().item()) * w.d * 2 * es
    qo = 2.0 * w.batch * w.n_q * w.h_q * w.d * es
    attn_flops = 4.0 * float(S.sum().item()) * G * w.d
    # one pass over the routing table (the node summaries read every block row once)
    route_table_bytes_once = float(w.batch * w.h_kv * nb) * R * 2 * w.d * 2
    out = dict(summary_bytes=summary_bytes, route_flops=route_flops, route_table_bytes=route_table_bytes,
               route_table_bytes_once=route_table_bytes_once,
               attn_bytes=gathered + qo,
               gathered_bytes=gathered, attn_flops=attn_flops, mean_keys=float(S.float().mean().item()))
    if w.dtype == "bf16":
        # block-major stages.  Per selected slot (a used selected block of a
        # row) the tile kernel reads the G query rows and writes G partial rows
        # + (log-sum-exp, scale), and reads each distinct key block's K, V
        # once.  Per window chunk of a row the window kernel reads the G query
        # rows and writes G partial rows; it reads the window's K, V once.
        # The merge reads all slot partials and writes O and lse per row.
        # (method flops count the keys the row attends, 4 G B d per used
        # entry; the design's bytes follow its slots: one per pair of hot
        # entries or per other entry, each a tile of twice the block's keys)
        ne, nsl, nkeys = block_major_counts(idx, w)
        items = w.batch * w.n_q * w.h_kv
        nwc = (w.window + 255) // 256
        nwin = items * nwc
        wkeys = float(np.minimum(w.window, pos + 1).sum()) * w.batch * w.h_kv
        tile_keys = 2 * w.block
        out["blocks_bytes"] = nsl * G * (w.d * 2 * 2 + 8) + nkeys * 2 * tile_keys * w.d * 2
        out["blocks_flops"] = 4.0 * ne * G * w.block * w.d
        out["window_bytes"] = nwin * G * (w.d * 2 * 2 + 8) + w.batch * w.n * w.h_kv * 2 * w.d * 2
        out["window_flops"] = 4.0 * wkeys * G * w.d
        out["merge_bytes"] = items * (G * w.d * 2 + G * 4 + w.topk * 4) + (nsl + nwin) * G * (w.d * 2 + 8)
        out["plan_bytes"] = items * w.topk * 4 * 3 + nsl * 4 + items * 12
        out["n_entries"] = ne
        out["n_slots"] = nsl
        out["n_blocks"] = nkeys
    return out


# ------------------------------------------------------------------ our arm

def needle_recall(plan, idx, w):
    """Fraction of planted needles whose key block the row selected."""
    if not plan:
        return None
    G = w.h_q // w.h_kv
    b = torch.tensor([p[0] for p in plan], device=idx.device)
    i = torch.tensor([p[1] for p in plan], device=idx.device)
    g = torch.tensor([p[2] // G for p in plan], device=idx.device)
    blk = torch.tensor([p[3] // w.block for p in plan], device=idx.device, dtype=idx.dtype)
    return float((idx[b, i, g] == blk[:, None]).any(dim=1).float().mean())


def run_ours(w, steps, warmup, ws, rank, with_e2e=True, hier=None):
    """hier: None (the flat router) or (fanout, probe, escalate, levels) for
    the hierarchical router, whose node summaries are then rebuilt every step."""
    from content_routed_block_ssa_b200 import ssa
    dev = torch.device("cuda", torch.cuda.current_device())
    Q, K, V, plan = make_inputs(w, dev)
    p = ssa.make_params(**problem_dict(w))
    mu_s, sig_s, tab_s = ssa.summary_shapes(p)
    if w.dtype == "f32":   # float32 problems route on float32 mu / Sigma, no table
        mu = torch.empty(mu_s, dtype=torch.float32, device=dev)
        sig = torch.empty(sig_s, dtype=torch.float32, device=dev)
        tab = None
    else:
        mu = sig = None
        tab = torch.empty(tab_s, dtype=torch.bfloat16, device=dev)
    idx = torch.empty(ssa.idx_shape(p), dtype=torch.int32, device=dev)
    rws = ssa.byte_buffer(ssa.ssa_route_workspace_size(p), dev)
    aw_bytes = ssa.ssa_attn_workspace_size(p)
    aws = ssa.byte_buffer(aw_bytes, dev) if aw_bytes else None
    O = torch.empty_like(Q)
    lse = torch.empty(Q.shape[:3], dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    # stages of one step, each bracketed by events on the launching stream;
    # block-major attention runs as its staged calls
    cert = None
    if hier is not None:
        hp = ssa.make_hier_params(*hier)
        nodes = ssa.byte_buffer(ssa.ssa_hier_nodes_size(p, hp), dev)
        hws = ssa.byte_buffer(ssa.ssa_route_hier_workspace_size(p, hp), dev)
        cert = torch.zeros(idx.shape[:3], dtype=torch.uint8, device=dev)
        route_stages = [("hier_nodes", lambda: ssa.ssa_hier_nodes(p, hp, tab, nodes)),
                        ("route", lambda: ssa.ssa_route_hier(p, hp, Q, tab, nodes, idx, cert, hws))]
    else:
        route_stages = [("route", lambda: ssa.ssa_route_topk(p, Q, mu, sig, tab, idx, None, rws))]
    if aws is not None:
        stages = [("summary", lambda: ssa.ssa_block_summary(p, K, None, None, tab))] + route_stages + [
                  ("attn_plan", lambda: ssa.ssa_attn_plan(p, idx, aws)),
                  ("attn_blocks", lambda: ssa.ssa_attn_blocks(p, Q, K, V, aws)),
                  ("attn_window", lambda: ssa.ssa_attn_window(p, Q, K, V, aws)),
                  ("attn_merge", lambda: ssa.ssa_attn_merge(p, idx, O, lse, None, aws))]
    else:
        stages = [("summary", lambda: ssa.ssa_block_summary(p, K, mu, sig, tab))] + route_stages + [
                  ("attn_gather", lambda: ssa.ssa_sparse_attn(p, Q, K, V, idx, O, lse))]
    # decode: the cache's block summaries (and node store) are precomputed
    # state, as the decode workload states; they are built once before the
    # timed steps and timed on their own, outside the step
    state = [st for st in stages if w.decode and st[0] in ("summary", "hier_nodes")]
    stages = [st for st in stages if st not in state]
    ms_state = {}
    for name, fn in state:
        for _ in range(2):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.zero_()
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ms_state[name] = e0.elapsed_time(e1)
    ns = len(stages)

    def step(ev=None):
        for k, (_, fn) in enumerate(stages):
            if ev:
                ev[k].record(stream)
            fn()
        if ev:
            ev[ns].record(stream)

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(ns + 1)] for _ in range(steps)]
    barrier(ws)
    torch.cuda.synchronize()
    l0 = ssa.ssa_launch_count()
    with ClockSampler(smi_index(torch.cuda.current_device())) as clk:
        for k in range(steps):
            flush.zero_()
            step(evs[k])
        torch.cuda.synchronize()
    launches = ssa.ssa_launch_count() - l0
    barrier(ws)
    assert ssa.ssa_device_error() == 0
    per = np.array([[e[k].elapsed_time(e[k + 1]) for k in range(ns)] for e in evs])
    ms_kernels = {name: float(x) for (name, _), x in zip(stages, per.mean(axis=0))}
    ms_kernels.update(ms_state)
    ms_step_local = float(per.sum(axis=1).mean())
    ms_step = max_over_ranks(ms_step_local, ws)
    ms_step_median = max_over_ranks(float(np.median(per.sum(axis=1))), ws)
    work = algorithmic_work(w, idx)
    selection = {"needle_recall": needle_recall(plan, idx, w)}
    if cert is not None:
        selection["certified"] = float(cert.float().mean())
        selection["router"] = {"fanout": hier[0], "probe": hier[1], "escalate": bool(hier[2]), "levels": hier[3]}

    e2e = None
    if with_e2e:
        # Through the public host-buffer call, every step copying its inputs in
        # from pinned host memory and its output back.  Consecutive steps go
        # round-robin to NS streams, each with its own device buffer and host
        # output, as a caller pipelining steps would: a step's copies overlap
        # the other streams' compute (the copy engines run both directions at
        # once).  As many streams as fit in a third of the device memory, up to 3.
        hQ, hK, hV = Q.cpu().pin_memory(), K.cpu().pin_memory(), V.cpu().pin_memory()
        del O, lse, aws, stages
        torch.cuda.empty_cache()
        hbytes = ssa.ssa_hostio_buffer_size(p)
        NS = max(1, min(3, int(torch.cuda.mem_get_info(dev)[0] // max(hbytes, 1)) - 1))
        outs = [(torch.empty(Q.shape, dtype=Q.dtype).pin_memory(),
                 torch.empty(Q.shape[:3], dtype=torch.float32).pin_memory()) for _ in range(NS)]
        bufs = [ssa.byte_buffer(hbytes, dev) for _ in range(NS)]
        streams = [stream] + [torch.cuda.Stream(dev) for _ in range(NS - 1)]

        def e2e_step(k):
            hO, hl = outs[k % NS]
            ssa.ssa_forward_hostio(p, hQ, hK, hV, hO, hl, bufs[k % NS], stream=streams[k % NS])

        for k in range(max(NS, warmup)):
            e2e_step(k)
        torch.cuda.synchronize()
        barrier(ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(streams[0])
        for st in streams[1:]:
            st.wait_event(e0)
        # ten steps per stream: the pipeline's fill and drain (one step's
        # kernels and output copy after the last input copy) are amortised
        n_e2e = 10 * NS
        for k in range(n_e2e):
            e2e_step(k)
        for st in streams[1:]:
            done = torch.cuda.Event()
            done.record(st)
            streams[0].wait_event(done)
        e1.record(streams[0])
        torch.cuda.synchronize()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1) / n_e2e, ws)
        hO, hl = outs[0]
        h2d = hQ.numel() * hQ.element_size() + 2 * hK.numel() * hK.element_size()
        d2h = hO.numel() * hO.element_size() + hl.numel() * hl.element_size()
        e2e = {"value": whole_job_rate(w.batch * w.n_q * w.h_q, ws, ms_e2e), "unit": UNIT,
               "ms_per_step": ms_e2e, "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": n_e2e, "streams": NS}
        del bufs
    return dict(ms_step=ms_step, ms_step_median=ms_step_median, ms_kernels=ms_kernels, work=work,
                launches=int(launches),
                clocks=clk.summary(), e2e=e2e, selection=selection, untimed_state=sorted(ms_state))


KERNEL_NAMES = {"summary": "summary_bf16_warp_kernel", "route": "route_tiled_kernel", "attn_plan": "inv_*_kernel (6)",
                "hier_nodes": "hier_nodes_kernel",
                "attn_blocks": "attn_block_kernel", "attn_window": "attn_window_kernel",
                "attn_merge": "attn_merge_kernel",
                "attn_gather": "attn_bf16_kernel"}


def kernel_report(w, res, peaks, traffic):
    """Per stage: time, algorithmic work and the fraction of the measured
    peak of the unit that bounds it (the larger of the HBM and tensor
    fractions where both apply)."""
    ms = res["ms_kernels"]
    wk = res["work"]
    hbm = peaks["hbm_gbs"]
    tc = peaks["bf16_tflops_sustained"]
    rep = {}

    def hbm_entry(name, nbytes, extra=None):
        t = ms[name] * 1e-3
        gbs = nbytes / t / 1e9
        e = {"ms": ms[name], "bound": "hbm", "achieved": gbs, "unit": "GB/s", "frac": gbs / hbm, "peak": hbm,
             "algorithmic_bytes": nbytes, "kernel": KERNEL_NAMES[name],
             "traffic": traffic.get((KERNEL_NAMES[name].split()[0], w.name))}
        e.update(extra or {})
        rep[name] = e

    hbm_entry("summary", wk["summary_bytes"])
    if "hier_nodes" in ms:
        # node summaries: one pass over the routing table; the hierarchical
        # route (node router + per-row probe of L2-served table rows + any
        # escalation) is reported by time, outside the roofline
        hbm_entry("hier_nodes", wk["route_table_bytes_once"])
        rep["route"] = {"ms": ms["route"], "kernel": "route_tiled_kernel / route_rowwise_bf16_kernel (nodes or "
                                                     "super-nodes) + hier_probe2_kernel (two levels) + "
                                                     "hier_probe_kernel (+ escalation)"}
    elif w.dtype == "f32":
        rep["summary"]["kernel"] = "summary_diag_kernel" if w.sigma == "diag" else "summary_full_kernel"
        # float32 rows score their blocks with FMA on the CUDA cores (row-wise router)
        r_tf = wk["route_flops"] / (ms["route"] * 1e-3) / 1e12
        rep["route"] = {"ms": ms["route"], "bound": "alu", "achieved": r_tf, "unit": "TFLOP/s",
                        "frac": r_tf / FP32_TFLOPS, "peak": FP32_TFLOPS, "algorithmic_flops": wk["route_flops"],
                        "kernel": "route_qtile_f32_kernel", "traffic": None}
    elif w.n_q < 128:
        # decode: each row streams its (batch, kv-head) table once (row-wise router)
        e = wk["route_table_bytes"] / (ms["route"] * 1e-3) / 1e9
        rep["route"] = {"ms": ms["route"], "bound": "hbm", "achieved": e, "unit": "GB/s", "frac": e / hbm,
                        "peak": hbm, "algorithmic_bytes": wk["route_table_bytes"],
                        "kernel": "route_rowwise_bf16_kernel",
                        "traffic": traffic.get(("route_rowwise_bf16_kernel", w.name))}
    else:
        r_tf = wk["route_flops"] / (ms["route"] * 1e-3) / 1e12
        rep["route"] = {"ms": ms["route"], "bound": "tensor", "achieved": r_tf, "unit": "TFLOP/s",
                        "frac": r_tf / tc, "peak": tc, "algorithmic_flops": wk["route_flops"],
                        "kernel": KERNEL_NAMES["route"], "traffic": traffic.get(("route_tiled_kernel", w.name))}
    if "attn_gather" in ms:
        hbm_entry("attn_gather", wk["attn_bytes"], {"mean_keys_per_row": wk["mean_keys"]})
        if w.dtype == "f32":
            rep["attn_gather"]["kernel"] = "attn_f32_kernel"
    else:
        hbm_entry("attn_plan", wk["plan_bytes"])
        # The block and window tiles are rated on the method's work: the
        # attention's flops (QK^T and PV, 4 G B d per selected slot; 4 G d
        # per window key), against the tensor-core peak.  Their HBM figure
        # counts the block-major design's own traffic (query rows re-read
        # per slot, partial outputs written for the merge), so it is kept
        # beside the headline as `design_traffic`, not as the bound.
        for name, fl_key in (("attn_blocks", "blocks_flops"), ("attn_window", "window_flops")):
            hbm_entry(name, wk[name.replace("attn_", "") + "_bytes"])
            e = rep[name]
            design = {"achieved": e["achieved"], "unit": "GB/s", "frac": e["frac"], "peak": hbm,
                      "algorithmic_bytes": e["algorithmic_bytes"], "traffic": e["traffic"]}
            t_f = wk[fl_key] / (ms[name] * 1e-3) / 1e12
            e.update(bound="tensor", achieved=t_f, unit="TFLOP/s", frac=t_f / tc, peak=tc,
                     algorithmic_flops=wk[fl_key], design_traffic=design)
            del e["algorithmic_bytes"]
        rep["attn_blocks"].update(n_entries=wk["n_entries"], n_slots=wk["n_slots"], n_tile_keys=wk["n_blocks"])
        hbm_entry("attn_merge", wk["merge_bytes"])
    # the pages' attention figure: algorithmic gathered K+V (+ q, o) bytes over
    # the whole attention time, whichever way it is evaluated
    t_att = sum(v for k, v in ms.items() if k.startswith("attn_")) * 1e-3
    rep["attention_gather_equivalent"] = {"ms": t_att * 1e3, "achieved": wk["attn_bytes"] / t_att / 1e9,
                                          "unit": "GB/s", "algorithmic_bytes": wk["attn_bytes"],
                                          "mean_keys_per_row": wk["mean_keys"]}
    return rep


def layer_report(w, wk, ms_step, peaks):
    """The whole layer against both roofs: the method's flops (routing scores
    and exact attention over the attended keys) per step over the step time,
    against the sustained tensor-core peak; and its compulsory HBM bytes (Q,
    K, V read once, O and lse written once, the routing table and block_idx
    each written and read once) over the step time, against the copy
    bandwidth."""
    es = 4 if w.dtype == "f32" else 2
    nb = w.n // w.block
    flops = wk["route_flops"] + wk["attn_flops"]
    io = (w.batch * w.n_q * w.h_q * w.d * es * 2 + w.batch * w.n * w.h_kv * w.d * es * 2
          + w.batch * w.n_q * w.h_q * 4)
    table = w.batch * w.h_kv * nb * (w.subblocks + (1 if w.outlier else 0)) * 2 * w.d * (2 if w.dtype == "bf16" else 4)
    idx = w.batch * w.n_q * w.h_kv * w.topk * 4
    nbytes = io + 2 * table + 2 * idx
    t = ms_step * 1e-3
    tf = flops / t / 1e12
    gbs = nbytes / t / 1e9
    return {"ms": ms_step, "method_flops": flops, "achieved_tflops": tf,
            "frac_tensor": tf / peaks["bf16_tflops_sustained"], "tensor_peak": peaks["bf16_tflops_sustained"],
            "compulsory_bytes": nbytes, "achieved_gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
            "hbm_peak": peaks["hbm_gbs"], "mean_keys_per_row": wk["mean_keys"]}


def dominant(rep, exclude=()):
    name = max((k for k in rep if "bound" in rep[k] and k not in exclude), key=lambda k: rep[k]["ms"])
    return name, rep[name]


# ------------------------------------------------------------------ oracle (CPU)

def run_oracle_sample(w, rows_per_step, steps, warmup, seed=7):
    """Times the oracle on the host: full block summaries once (amortised per
    step by the sampled fraction), then route + attention of `rows_per_step`
    query rows (all heads) per step.  Returns (query-heads/s, seconds, info)."""
    from oracle import ssa_oracle as O
    Q, K, V, _ = make_inputs(w, "cuda" if torch.cuda.is_available() else "cpu")
    Kn = K.float().cpu().numpy()
    Vn = V.float().cpu().numpy()
    rng = np.random.default_rng(seed)
    op = O.Problem(**problem_dict(w))
    t0 = time.perf_counter()
    mu, sig = O.block_summaries(Kn, op)
    stored = O.stored_summaries(mu, sig, op)
    t_sum = time.perf_counter() - t0
    times = []
    G = w.h_q // w.h_kv
    for k in range(warmup + steps):
        rows_i = np.sort(rng.choice(w.n_q, size=rows_per_step, replace=False))
        Qs = Q[:, torch.from_numpy(rows_i).to(Q.device)].float().cpu().numpy()   # [b, rows, h_q, d]
        t1 = time.perf_counter()
        for bi in range(w.batch):
            for r, i in enumerate(rows_i):
                pos = w.q_offset + int(i)
                pr = O.Problem(**{**problem_dict(w), "n_q": rows_per_step, "q_offset": pos - r})
                for g in range(w.h_kv):
                    s = O.route_scores_row(Qs, stored, pr, bi, r, g)
                    sel, _ = O.select_topk(s, w.topk)
                    S = O.key_set(pos, sel, op)
                    O.softmax_attend(Qs[bi, r, g * G:(g + 1) * G], Kn[bi, S, g], Vn[bi, S, g], op.scale)
        dt = time.perf_counter() - t1
        if k >= warmup:
            times.append(dt + t_sum * rows_per_step / w.n_q)
    sec = float(np.mean(times))
    qh = w.batch * rows_per_step * w.h_q
    info = {"summary_s": t_sum, "rows_per_step": rows_per_step}
    return qh / sec, sec, info


def cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=PRIMARY, choices=list(WORKLOADS))
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--n", type=int, default=None,
                    help="shorter sequence of the same workload (profiling captures); not a bench line")
    ap.add_argument("--subblocks", type=int, default=1,
                    help="route on S sub-block summaries per block, max-pooled (S in 1, 2, 4; block / S >= 32)")
    ap.add_argument("--outlier", action="store_true",
                    help="route with the outlier-channel row per block (largest-norm key, max-pooled)")
    ap.add_argument("--router", default="flat", choices=["flat", "hier"],
                    help="hier: the hierarchical router (nodes of --fanout blocks, --probe nodes per row); "
                         "a measurement of that router, not the bench line")
    ap.add_argument("--fanout", type=int, default=16)
    ap.add_argument("--probe", type=int, default=2)
    ap.add_argument("--escalate", action="store_true", help="re-route uncertified rows over all blocks")
    ap.add_argument("--levels", type=int, default=1, choices=[1, 2], help="tree levels of the hierarchical router")
    ap.add_argument("--cluster-span", type=int, default=1,
                    help="clustered keys: S consecutive blocks share a centroid (nearby blocks alike); "
                         "a measurement of the routers on that structure, not the bench line")
    a = ap.parse_args()
    w = WORKLOADS[a.workload]
    if a.n is not None:
        w = w.scaled(n=a.n, needles=max(1, w.needles * a.n // w.n))
    if a.subblocks != 1:
        w = w.scaled(subblocks=a.subblocks)
    if a.outlier:
        w = w.scaled(outlier=True)
    if a.cluster_span != 1:
        if not w.clustered or a.cluster_span < 1:
            raise SystemExit("--cluster-span needs a clustered workload and S >= 1")
        w = w.scaled(cluster_span=a.cluster_span)
    ws, rank, local = dist_setup(a.gpus)
    peaks, peak_src = load_peaks()

    config = {"workload": w.name, "batch": w.batch, "n": w.n, "n_q": w.n_q, "h_q": w.h_q, "h_kv": w.h_kv,
              "d": w.d, "block": w.block, "topk": w.topk, "window": w.window, "sigma": w.sigma,
              "subblocks": w.subblocks, "outlier": w.outlier,
              "beta": w.beta, "keys": "block-clustered + planted needles" if w.clustered else "iid + planted needles",
              "cluster_span": w.cluster_span,
              "l2": "flushed between steps (256 MiB write); inputs larger than L2",
              "parallelism": f"replicas x{ws} (independent problems)"}

    if a.impl == "reference":
        if rank != 0:
            return
        rows = 16
        val, sec, info = run_oracle_sample(w, rows, a.steps, a.warmup)
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": a.gpus,
                "steps": a.steps, "warmup": a.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores(), "kind": "oracle",
                                 "sample": f"{rows} query rows x {w.h_q} heads per step, block summaries of all "
                                           f"{w.n} keys amortised by {rows}/{w.n_q}"},
                "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    # the committed DRAM counters were taken with whole-block summaries
    traffic = load_traffic() if w.subblocks == 1 and not w.outlier else {}
    hier = (a.fanout, a.probe, a.escalate, a.levels) if a.router == "hier" else None
    if w.decode:
        config["state"] = "block summaries precomputed (built once, untimed; kernels.summary times one build)"
    if hier is not None:
        config["router"] = {"kind": "hierarchical", "fanout": a.fanout, "probe": a.probe, "escalate": a.escalate,
                            "levels": a.levels}
    res = run_ours(w, a.steps, a.warmup, ws, rank, with_e2e=not a.no_e2e and hier is None, hier=hier)
    kern = kernel_report(w, res, peaks, traffic)
    value = whole_job_rate(w.batch * w.n_q * w.h_q, ws, res["ms_step"])
    dname, dk = dominant(kern, exclude=res["untimed_state"])
    roof = {"bound": dk["bound"], "achieved": dk["achieved"], "peak": dk["peak"], "unit": dk["unit"],
            "frac": dk["frac"], "traffic": dk["traffic"], "kernel": dk["kernel"], "stage": dname,
            "peak_source": peak_src,
            # the same against the nominal datasheet peaks (HBM3e 7.7 TB/s, dense bf16 2.25 PFLOP/s)
            "peak_nominal": NOMINAL[dk["unit"]] if dk["bound"] in ("hbm", "tensor") else None,
            "frac_nominal": dk["achieved"] / NOMINAL[dk["unit"]] if dk["bound"] in ("hbm", "tensor") else None,
            "algorithmic_per_launch": dk.get("algorithmic_flops") if dk["bound"] in ("tensor", "alu")
            else dk["algorithmic_bytes"]}
    if "design_traffic" in dk:
        roof["design_traffic"] = dk["design_traffic"]
    roof["layer"] = layer_report(w, res["work"], res["ms_step"], peaks)
    secondary = None
    if not a.no_secondary and w.name == PRIMARY and a.n is None:
        torch.cuda.empty_cache()
        w2 = WORKLOADS[SECONDARY]
        if w.subblocks != 1 and w2.block // w.subblocks >= 32:
            w2 = w2.scaled(subblocks=w.subblocks)
        if w.outlier:
            w2 = w2.scaled(outlier=True)
        r2 = run_ours(w2, max(3, a.steps // 2), a.warmup, ws, rank, with_e2e=False)
        k2 = kernel_report(w2, r2, peaks, traffic)
        secondary = {"workload": w2.name, "subblocks": w2.subblocks, "outlier": w2.outlier,
                     "selection": r2["selection"],
                     "value": whole_job_rate(w2.batch * w2.n_q * w2.h_q, ws, r2["ms_step"]),
                     "unit": UNIT, "ms_per_step": r2["ms_step"], "kernels": k2, "gpu_launches": r2["launches"],
                     "clocks": r2["clocks"]}
    cpu = None
    if rank == 0 and ws == 1 and not a.no_cpu_baseline:
        rows = 256   # ~10-15 s of host work with the full block summaries
        val, sec, info = run_oracle_sample(w, rows, 2, 1)
        cpu = {"value": val, "unit": UNIT, "cores": cores(), "kind": "oracle",
               "sample": f"{rows} query rows x {w.h_q} heads per step, block summaries of all {w.n} keys "
                         f"amortised by {rows}/{w.n_q}; 2 steps after 1 warm-up"}
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": a.steps, "warmup": a.warmup,
                "ms_per_step": res["ms_step"], "ms_per_step_median": res["ms_step_median"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": w.dtype, "data": "synthetic", "config": config, "roofline": roof, "cpu_baseline": cpu,
                "e2e": res["e2e"], "gpu_launches": res["launches"], "clocks": res["clocks"], "kernels": kern,
                "selection": res["selection"], "secondary": secondary}
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
