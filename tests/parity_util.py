"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same input bytes, and compare.

Comparison rules (from the layer's statement of correctness):
  * block indices: bit-exact on every row whose oracle gap between the k-th
    and (k+1)-th score is at least NEAR_TIE_BAND relative (a float32
    accumulation-order band); rows inside the literal 1e-3 near-tie band are
    counted and reported;
  * outputs: max-abs <= 1e-4 (float32 problems); max-abs <= 2e-2 and
    relative L2 <= 1e-2 (bf16 problems).
"""
from __future__ import annotations

import numpy as np
import torch

from content_routed_block_ssa_b200 import ssa
from oracle import ssa_oracle as O

NEAR_TIE_BAND = 1e-5
LITERAL_NEAR_TIE = 1e-3
TOL = {"f32": dict(max_abs=1e-4, rel_l2=1e-4), "bf16": dict(max_abs=2e-2, rel_l2=1e-2)}


def oracle_problem(pd: dict) -> O.Problem:
    return O.Problem(**pd)


def params(pd: dict, route_impl=ssa.SSA_ROUTE_AUTO):
    return ssa.make_params(**pd, route_impl=route_impl)


def gpu_summary(p, K):
    mu_s, sig_s, tab_s = ssa.summary_shapes(p)
    dev = K.device
    mu = torch.empty(mu_s, dtype=torch.float32, device=dev)
    sig = torch.empty(sig_s, dtype=torch.float32, device=dev)
    tab = torch.empty(tab_s, dtype=torch.bfloat16, device=dev) if p.dtype == ssa.SSA_BF16 else None
    ssa.ssa_block_summary(p, K, mu, sig, tab)
    return mu, sig, tab


def gpu_route(p, Q, mu, sig, tab):
    idx = torch.full(ssa.idx_shape(p), -7, dtype=torch.int32, device=Q.device)
    sc = torch.empty(ssa.idx_shape(p), dtype=torch.float32, device=Q.device)
    ws = ssa.byte_buffer(ssa.ssa_route_workspace_size(p), Q.device)
    ssa.ssa_route_topk(p, Q, mu, sig, tab, idx, sc, ws)
    return idx, sc


def gpu_attn(p, Q, K, V, idx, workspace=True):
    """Sparse attention through the C ABI.  With ``workspace`` the call gets
    the attention workspace, so problems that qualify run block-major;
    without it every problem takes the per-row gather path."""
    O_ = torch.empty_like(Q)
    lse = torch.empty(Q.shape[:3], dtype=torch.float32, device=Q.device)
    bad = torch.zeros(1, dtype=torch.int32, device=Q.device)
    nbytes = ssa.ssa_attn_workspace_size(p) if workspace else 0
    ws = ssa.byte_buffer(nbytes, Q.device) if nbytes else None
    ssa.ssa_sparse_attn(p, Q, K, V, idx, O_, lse, bad, ws)
    return O_, lse, bad


def check_no_device_error():
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0


def compare_idx(gpu_idx: np.ndarray, ref_idx: np.ndarray, gaps: np.ndarray, rows=None):
    """Returns (n_rows_checked, n_strict_mismatch, n_flagged_literal, n_in_band)."""
    if rows is not None:
        sel = [(b, i) for b, i in rows]
        g = np.stack([gpu_idx[b, i] for b, i in sel])
        r = np.stack([ref_idx[b, i] for b, i in sel])
        gp = np.stack([gaps[b, i] for b, i in sel])
    else:
        g, r, gp = gpu_idx, ref_idx, gaps
    g = g.reshape(-1, g.shape[-1])
    r = r.reshape(-1, r.shape[-1])
    gp = gp.reshape(-1)
    strict = gp >= NEAR_TIE_BAND
    mism = np.any(g != r, axis=1)
    return (len(gp), int(np.sum(mism & strict)), int(np.sum(gp < LITERAL_NEAR_TIE)),
            int(np.sum(mism & ~strict)))


def compare_out(got: np.ndarray, ref: np.ndarray, dtype: str):
    d = got.astype(np.float64) - ref
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-30))
    tol = TOL[dtype]
    return max_abs, rel, (max_abs <= tol["max_abs"] and rel <= tol["rel_l2"])


def as_np(t):
    return t.detach().float().cpu().numpy() if t.dtype in (torch.bfloat16, torch.float16) else t.detach().cpu().numpy()
