"""Parity at the full workload sizes, in the launch configuration the bench
times: block summaries, the router and the attention (block-major where the
problem qualifies) run through the C ABI on the whole problem; the oracle
recomputes every block summary and, one row at a time, the selection and the
attention of a seeded sample of rows:

  * every row holding a planted needle,
  * 1024 rows at uniform positions,
  * the first 2B rows and the last 64 rows,
  * decode: 8 of the 64 sequences (their single query row).

Criteria as for the small cases: summaries bit-exact (the bf16 routing table)
or within one float32 ulp; block indices bit-exact outside the near-tie band;
outputs within the float32 / bf16 tolerances.
"""
import numpy as np
import pytest
import torch

from content_routed_block_ssa_b200 import ssa
from content_routed_block_ssa_b200.workload import WORKLOADS, make_inputs, problem_dict
from oracle import ssa_oracle as O
from parity_util import TOL, check_no_device_error, compare_idx, compare_out, gpu_summary, params

pytestmark = pytest.mark.gpu


def sample_rows(w, plan, rng):
    if w.decode:
        return sorted(int(b) for b in rng.choice(w.batch, size=min(8, w.batch), replace=False))
    needles = sorted({int(p[1]) for p in plan})
    uniform = [int(x) for x in rng.choice(w.n_q, size=min(1024, w.n_q), replace=False)]
    edge = list(range(min(w.n_q, 2 * w.block))) + list(range(max(0, w.n_q - 64), w.n_q))
    return sorted(set(needles) | set(uniform) | set(edge))


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_full_size_sampled_parity(name):
    w = WORKLOADS[name]
    dev = torch.device("cuda")
    torch.cuda.empty_cache()
    Q, K, V, plan = make_inputs(w, dev)
    p = params(problem_dict(w))
    mu, sig, tab = gpu_summary(p, K)
    idx = torch.empty(ssa.idx_shape(p), dtype=torch.int32, device=dev)
    rws = ssa.byte_buffer(ssa.ssa_route_workspace_size(p), dev)
    route_mu, route_sig = (mu, sig) if w.dtype == "f32" else (None, None)
    ssa.ssa_route_topk(p, Q, route_mu, route_sig, tab, idx, None, rws)
    aw = ssa.ssa_attn_workspace_size(p)
    aws = ssa.byte_buffer(aw, dev) if aw else None
    Og = torch.empty_like(Q)
    lse = torch.empty(Q.shape[:3], dtype=torch.float32, device=dev)
    bad = torch.zeros(1, dtype=torch.int32, device=dev)
    ssa.ssa_sparse_attn(p, Q, K, V, idx, Og, lse, bad, aws)
    check_no_device_error()
    assert int(bad.item()) == 0

    rng = np.random.default_rng(2024 + w.wid)
    rows = sample_rows(w, plan, rng)
    if w.decode:   # a sub-problem of the sampled sequences
        sel = torch.tensor(rows, device=dev)
        Qs, Ks, Vs = Q[sel], K[sel], V[sel]
        gi = idx[sel].cpu().numpy()
        go, gl = Og[sel].float().cpu().numpy(), lse[sel].cpu().numpy()
        gtab = tab[sel].float().cpu().numpy() if tab is not None else None
        pd = dict(problem_dict(w), batch=len(rows))
        orows = [(bi, 0) for bi in range(len(rows))]
    else:
        Qs, Ks, Vs = Q, K, V
        gi = idx.cpu().numpy()
        go, gl = Og.float().cpu().numpy(), lse.cpu().numpy()
        gtab = tab.float().cpu().numpy() if tab is not None else None
        pd = problem_dict(w)
        orows = [(0, i) for i in rows]
    gmu = mu.cpu().numpy() if w.dtype == "f32" else None
    del mu, sig, tab, idx, Og, lse, rws, aws
    op = O.Problem(**pd)
    Qn = Qs.float().cpu().numpy()
    Kn = Ks.float().cpu().numpy()
    Vn = Vs.float().cpu().numpy()
    del Q, K, V, Qs, Ks, Vs
    torch.cuda.empty_cache()

    parts = []   # one sequence at a time keeps the float64 temporaries small
    for bi in range(op.batch):
        m64, s64 = O.block_summaries(Kn[bi:bi + 1], op)
        parts.append(O.stored_summaries(m64, s64, op))
        del m64, s64
    stored = tuple(None if parts[0][k] is None else np.concatenate([q[k] for q in parts]) for k in range(3))
    del parts
    if gtab is not None:
        assert np.array_equal(gtab.astype(np.float64), stored[2])
    else:
        assert np.array_equal(gmu.astype(np.float64), stored[0])

    bidx, gaps = O.route_topk(Qn, stored, op, rows=orows)
    n, strict, literal, in_band = compare_idx(gi, bidx, gaps, rows=orows)
    # reported, not asserted: rows inside the literal 1e-3 near-tie band, GPU
    # mismatches inside the 1e-5 band, and (bf16) rows whose selection without
    # the bf16 rounding of features and summaries would differ
    unq = None
    if w.dtype == "bf16":
        ub, _ = O.route_topk_unquantised(Qn, stored, op, rows=orows)
        unq = sum(int(not np.array_equal(ub[b, i, g], bidx[b, i, g])) for b, i in orows for g in range(op.h_kv))
    print(f"\nSELECTION {name} rows={n} literal_near_tie={literal} ({literal / max(n, 1):.2%}) "
          f"band_mismatch={in_band} unquantised_differs={unq}", flush=True)
    assert strict == 0, f"{strict} of {n} sampled rows differ outside the near-tie band"

    # attention on the GPU's own selection, row by row
    Oo, Lo = O.attention(Qn, Kn, Vn, gi.astype(np.int64), op, rows=orows)
    got = np.stack([go[b, i] for b, i in orows])
    ref = np.stack([Oo[b, i] for b, i in orows])
    max_abs, rel, ok = compare_out(got, ref, w.dtype)
    assert ok, (max_abs, rel)
    gls = np.stack([gl[b, i] for b, i in orows])
    rls = np.stack([Lo[b, i] for b, i in orows])
    assert np.abs(gls - rls).max() <= (1e-4 if w.dtype == "f32" else 2e-2)
