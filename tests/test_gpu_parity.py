"""GPU parity: every stage of the CUDA path, called through the C ABI, against
the CPU oracle on the same seeded inputs.

Stages are isolated by feeding the CUDA kernel the oracle's output of the
previous stage (oracle summaries -> CUDA router; oracle block indices ->
CUDA attention), then the whole layer is compared end to end.  Sizes span
several row tiles, a ragged last tile and several blocks per window.
"""
import ctypes as C

import numpy as np
import pytest
import torch

from content_routed_block_ssa_b200 import ssa
from content_routed_block_ssa_b200.workload import Workload, make_inputs, problem_dict
from oracle import ssa_oracle as O

from parity_util import (as_np, check_no_device_error, compare_idx, compare_out, gpu_attn, gpu_route,
                         gpu_summary, params, NEAR_TIE_BAND)

pytestmark = pytest.mark.gpu

CASES = {
    "bf16_gqa4_d128_b64": Workload("c", 101, 2, 1152, 8, 2, 128, "bf16", 64, "diag", 8, 256, 6, "total",
                                   clustered=True),
    "bf16_mha_d128_b64_k32": Workload("c", 102, 1, 2112, 2, 2, 128, "bf16", 64, "diag", 32, 128, 8, "per_head"),
    "bf16_gqa8_d128_b128_k16": Workload("c", 103, 1, 3072, 8, 1, 128, "bf16", 128, "diag", 16, 256, 12, "total",
                                        clustered=True),
    "bf16_gqa4_d128_b64_k32_b2": Workload("c", 109, 2, 2560, 8, 2, 128, "bf16", 64, "diag", 32, 256, 8, "total",
                                          clustered=True),
    "bf16_gqa2_d128_b64_w100": Workload("c", 113, 1, 2304, 4, 2, 128, "bf16", 64, "diag", 16, 100, 6, "per_head"),
    # block-major variants: cp.async Q rows with 128-key blocks (G = 4, 2; a
    # window of 300 keys, not block aligned) and TMA Q boxes with 64-key
    # blocks (G = 8)
    "bf16_gqa4_d128_b128_k16": Workload("c", 114, 1, 2560, 8, 2, 128, "bf16", 128, "diag", 16, 256, 6, "total"),
    "bf16_gqa2_d128_b128_w300_b2": Workload("c", 116, 2, 1536, 4, 2, 128, "bf16", 128, "diag", 8, 300, 4,
                                            "per_head"),
    "bf16_gqa8_d128_b64_k16": Workload("c", 115, 1, 2048, 16, 2, 128, "bf16", 64, "diag", 16, 192, 6, "total",
                                       clustered=True),
    "bf16_gqa2_d64_b64": Workload("c", 104, 1, 1024, 4, 2, 64, "bf16", 64, "diag", 4, 64, 6, "total"),
    "bf16_mha_d64_b128_w200": Workload("c", 105, 1, 1280, 1, 1, 64, "bf16", 128, "diag", 8, 200, 4, "total"),
    "f32_full_d64": Workload("c", 106, 1, 1024, 1, 1, 64, "f32", 64, "full", 8, 64, 8, "total"),
    "f32_diag_d128_gqa4_w100": Workload("c", 107, 1, 512, 4, 1, 128, "f32", 64, "diag", 4, 100, 4, "total"),
    "f32_full_gqa2_d64_b128": Workload("c", 108, 1, 768, 2, 1, 64, "f32", 128, "full", 2, 64, 2, "total"),
    # sub-block summaries (max-pooled block scores): 32-key units from 64- and
    # 128-key blocks, 64-key units at d = 64, float32 full and diagonal
    "bf16_gqa4_d128_b64_s2": Workload("c", 117, 1, 1280, 8, 2, 128, "bf16", 64, "diag", 8, 128, 6, "total",
                                      clustered=True, subblocks=2),
    "bf16_gqa8_d128_b128_s4": Workload("c", 118, 1, 2304, 8, 1, 128, "bf16", 128, "diag", 8, 256, 8, "total",
                                       subblocks=4),
    "bf16_mha_d64_b128_s2": Workload("c", 119, 1, 1024, 2, 2, 64, "bf16", 128, "diag", 4, 128, 4, "per_head",
                                     subblocks=2),
    "f32_full_d64_s2": Workload("c", 120, 1, 768, 1, 1, 64, "f32", 64, "full", 4, 64, 4, "total", subblocks=2),
    "f32_diag_gqa2_d128_b128_s4": Workload("c", 121, 1, 512, 2, 1, 128, "f32", 128, "diag", 2, 100, 2, "total",
                                           subblocks=4),
    # windows of several chunks on the block-major path: two 128-key chunks
    # (G = 1) and three 256-key chunks (G = 8)
    "bf16_mha_d128_b64_w200": Workload("c", 123, 1, 1536, 2, 2, 128, "bf16", 64, "diag", 8, 200, 4, "per_head"),
    "bf16_gqa8_d128_b64_w600": Workload("c", 124, 1, 2048, 16, 2, 128, "bf16", 64, "diag", 8, 600, 4, "total",
                                        clustered=True),
    # the largest windows: 1985 keys (32 window blocks of 64, the most the
    # block-major path takes: 8 window chunks) and 4032 keys (the API's limit,
    # 64 window tiles, per-row gather)
    "bf16_gqa4_d128_b64_w1985": Workload("c", 125, 1, 4096, 8, 2, 128, "bf16", 64, "diag", 8, 1985, 4, "total",
                                         clustered=True),
    "bf16_gqa4_d128_b64_w4032": Workload("c", 126, 1, 5120, 8, 2, 128, "bf16", 64, "diag", 8, 4032, 4, "total"),
    # routing temperatures other than 2: beta = 0 (centroid routing: the
    # variance half of every feature is zero), beta = 1 and beta = 3 (the
    # (beta/2) multiply of the squared sum is then not the identity), on the
    # tiled and row-wise routers, the block-major attention and float32
    "bf16_gqa4_d128_b64_beta0": Workload("c", 127, 1, 1536, 8, 2, 128, "bf16", 64, "diag", 16, 256, 6, "total",
                                         clustered=True, beta=0.0),
    "bf16_mha_d128_b64_beta1": Workload("c", 128, 1, 1280, 2, 2, 128, "bf16", 64, "diag", 8, 128, 4, "per_head",
                                        beta=1.0),
    "bf16_gqa8_d128_b128_beta3": Workload("c", 129, 1, 2048, 8, 1, 128, "bf16", 128, "diag", 8, 256, 6, "total",
                                          clustered=True, beta=3.0),
    "bf16_gqa4_d64_b64_beta3": Workload("c", 130, 1, 1024, 8, 2, 64, "bf16", 64, "diag", 8, 64, 4, "total",
                                        beta=3.0),
    "f32_full_d64_beta3": Workload("c", 131, 1, 768, 2, 1, 64, "f32", 64, "full", 4, 64, 2, "total", beta=3.0),
    "f32_diag_d128_beta0": Workload("c", 132, 1, 512, 4, 2, 128, "f32", 64, "diag", 4, 64, 2, "total", beta=0.0),
    # the outlier channel: a second summary row per block (its largest-norm
    # key, zero covariance), max-pooled with the block's cumulant score, on
    # the tiled and row-wise bf16 routers and the float32 routers
    "bf16_gqa4_d128_b64_outlier": Workload("c", 133, 1, 1536, 8, 2, 128, "bf16", 64, "diag", 8, 256, 6, "total",
                                           clustered=True, outlier=True),
    "bf16_gqa8_d128_b128_outlier": Workload("c", 134, 1, 2048, 8, 1, 128, "bf16", 128, "diag", 8, 256, 6,
                                            "total", outlier=True),
    "bf16_mha_d64_b64_outlier_beta0": Workload("c", 135, 1, 1024, 2, 2, 64, "bf16", 64, "diag", 4, 64, 4,
                                               "per_head", outlier=True, beta=0.0),
    "f32_diag_d128_outlier": Workload("c", 136, 1, 512, 4, 2, 128, "f32", 64, "diag", 4, 64, 2, "total",
                                      outlier=True),
    "f32_full_d64_outlier": Workload("c", 137, 1, 768, 2, 1, 64, "f32", 64, "full", 4, 64, 2, "total",
                                     outlier=True),
    # paired slots at their edges: k = 1 (every tile a single block, its
    # second half masked) and k = 2 (one pair or two singles per row), with
    # 64-key blocks (128-key tiles) and 128-key blocks (256-key tiles)
    "bf16_gqa4_d128_b64_k1": Workload("c", 138, 1, 2048, 8, 2, 128, "bf16", 64, "diag", 1, 128, 4, "total",
                                      clustered=True),
    "bf16_gqa8_d128_b128_k1": Workload("c", 139, 1, 3072, 8, 1, 128, "bf16", 128, "diag", 1, 256, 6, "total",
                                       clustered=True),
    "bf16_gqa4_d128_b128_k2": Workload("c", 140, 1, 3072, 8, 2, 128, "bf16", 128, "diag", 2, 256, 6, "total",
                                       clustered=True),
    # float32 routing takes runs of 32 (query, head) pairs per CTA unless a
    # row's 1024 block scores do not fit beside them: then one CTA per row
    "f32_diag_d64_decode_64k": Workload("c", 122, 1, 65536, 1, 1, 64, "f32", 64, "diag", 8, 64, 2, "per_seq",
                                        decode=True),
}

_cache = {}


def case(name):
    if name not in _cache:
        w = CASES[name]
        Q, K, V, plan = make_inputs(w, "cpu")
        pd = problem_dict(w)
        op = O.Problem(**pd)
        Qn, Kn, Vn = Q.float().numpy(), K.float().numpy(), V.float().numpy()
        ref = O.forward(Qn, Kn, Vn, op)
        _cache[name] = dict(w=w, pd=pd, op=op, Q=Q, K=K, V=V, Qn=Qn, Kn=Kn, Vn=Vn, ref=ref)
    return _cache[name]


def to_dev(*ts):
    return [t.cuda() for t in ts]


@pytest.mark.parametrize("name", list(CASES))
def test_summary_bit_exact(name):
    c = case(name)
    p = params(c["pd"])
    (K,) = to_dev(c["K"])
    mu, sig, tab = gpu_summary(p, K)
    check_no_device_error()
    mu32, sig32, table = c["ref"]["stored"]
    assert np.array_equal(mu.cpu().numpy().astype(np.float64), mu32)
    g = sig.cpu().numpy()
    r = sig32.astype(np.float32)
    ulp = np.abs(g.view(np.int32).astype(np.int64) - r.view(np.int32).astype(np.int64))
    assert ulp.max() <= 1 and np.mean(ulp > 0) < 1e-4
    if tab is not None:
        assert np.array_equal(tab.float().cpu().numpy().astype(np.float64), table)


def _stored_on_device(c):
    # the oracle's arrays may keep the strides of a permuted source: the C ABI
    # reads dense row-major buffers
    mu32, sig32, table = c["ref"]["stored"]
    mu = torch.from_numpy(np.ascontiguousarray(mu32, dtype=np.float32)).cuda()
    sig = torch.from_numpy(np.ascontiguousarray(sig32, dtype=np.float32)).cuda()
    tab = torch.from_numpy(np.ascontiguousarray(table)).to(torch.bfloat16).cuda() if table is not None else None
    return mu, sig, tab


ROUTE_IMPLS = [(n, impl) for n in CASES for impl in
               ((ssa.SSA_ROUTE_TILED, ssa.SSA_ROUTE_ROWWISE) if CASES[n].dtype == "bf16" else (ssa.SSA_ROUTE_AUTO,))]


IMPL_NAME = {ssa.SSA_ROUTE_AUTO: "auto", ssa.SSA_ROUTE_TILED: "tiled", ssa.SSA_ROUTE_ROWWISE: "rowwise"}


@pytest.mark.parametrize("name,impl", ROUTE_IMPLS, ids=[f"{n}-{IMPL_NAME[i]}" for n, i in ROUTE_IMPLS])
def test_route_matches_oracle_selection(name, impl):
    c = case(name)
    p = params(c["pd"], impl)
    (Q,) = to_dev(c["Q"])
    mu, sig, tab = _stored_on_device(c)
    idx, sc = gpu_route(p, Q, mu, sig, tab)
    check_no_device_error()
    gi = idx.cpu().numpy()
    n, strict, literal, in_band = compare_idx(gi, c["ref"]["block_idx"], c["ref"]["gaps"])
    assert strict == 0, f"{strict} of {n} rows differ outside the {NEAR_TIE_BAND} near-tie band"
    # scores of the selected blocks agree with the oracle's to float32 accumulation error
    stored = c["ref"]["stored"]
    op = c["op"]
    gs = sc.cpu().numpy()
    rng = np.random.default_rng(0)
    for bi in range(op.batch):
        for g in range(op.h_kv):
            S = O.route_scores(c["Qn"], stored, op, bi, g)
            for i in rng.choice(op.n_q, size=min(64, op.n_q), replace=False):
                for j in range(op.topk):
                    blk = gi[bi, i, g, j]
                    if blk >= 0:
                        assert abs(gs[bi, i, g, j] - S[i, blk]) <= 2e-5 * abs(S[i, blk]) + 1e-4
                    else:
                        assert gs[bi, i, g, j] == -np.inf
    # rows with fewer visible blocks than k keep all of them, then -1
    for i in range(min(op.n_q, 3 * op.block)):
        nv = O.visible_blocks(op.q_offset + i, op)
        if nv <= op.topk:
            assert list(gi[0, i, 0, :nv]) == list(range(nv))
            assert np.all(gi[0, i, 0, nv:] == -1)


@pytest.mark.parametrize("impl", [ssa.SSA_ROUTE_TILED, ssa.SSA_ROUTE_ROWWISE], ids=["tiled", "rowwise"])
def test_bf16_features_read_back_equal_golden_rounding(impl):
    """The GPU's routing features on the hand-derived rounding case
    (tests/golden/feature_rounding.json: beta = 3, eight query heads whose
    float32 head-order sums, (beta/2) multiply and bf16 rounding each decide
    a feature).  A routing table of unit rows e_t turns every score into one
    feature, f . e_t = f_t, and with all 8 blocks selected top_scores returns
    them in block order."""
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "feature_rounding.json")) as fh:
        g = json.load(fh)
    dg, G, d, B = g["d"], g["G"], 64, 64
    nb = 2 * dg
    n = nb * B
    q = torch.zeros(G, d, dtype=torch.float64)
    q[:, :dg] = torch.tensor(g["q_heads_by_dim"], dtype=torch.float64).T
    assert torch.equal(q.to(torch.bfloat16).double(), q)          # every input is a bf16 value
    Q = q.to(torch.bfloat16).expand(1, n, G, d).contiguous().cuda()
    tab = torch.zeros(1, 1, nb, 2 * d, dtype=torch.bfloat16)
    for t in range(dg):
        tab[0, 0, t, t] = 1.0                 # block t reads f_s[t]
        tab[0, 0, dg + t, d + t] = 1.0        # block dg + t reads f_q[t]
    tab = tab.cuda()
    p = ssa.make_params(batch=1, n_q=n, n_kv=n, h_q=G, h_kv=1, d=d, block=B, topk=nb, window=B,
                        beta=g["beta"], route_impl=impl)
    idx, sc = gpu_route(p, Q, None, None, tab)
    check_no_device_error()
    last = n - 1                                # the one row that sees all nb blocks
    assert idx[0, last, 0].tolist() == list(range(nb))
    assert sc[0, last, 0].double().cpu().tolist() == g["features"]


@pytest.mark.parametrize("impl", [ssa.SSA_ROUTE_TILED, ssa.SSA_ROUTE_ROWWISE], ids=["tiled", "rowwise"])
def test_route_all_blocks_equal_takes_the_first_k(impl):
    """Every block holds the same keys, so every visible block scores the
    same: the selection is the k lowest visible blocks.  With the tile
    router's seeds the seed bound equals the k-th best score exactly here,
    so this also checks that a block scoring exactly the bound is kept."""
    B, n, k = 64, 64 * 96, 16
    blk = torch.randn(B, 2, 128, generator=torch.Generator().manual_seed(9)).to(torch.bfloat16)
    K = blk.repeat(n // B, 1, 1).unsqueeze(0).contiguous()
    Q = torch.randn(1, n, 8, 128, generator=torch.Generator().manual_seed(10)).to(torch.bfloat16)
    p = ssa.make_params(batch=1, n_q=n, n_kv=n, h_q=8, h_kv=2, d=128, block=B, topk=k, window=B,
                        route_impl=impl)
    (Qd, Kd) = to_dev(Q, K)
    _, _, tab = gpu_summary(p, Kd)
    assert torch.equal(tab[0, :, :1].expand_as(tab[0]), tab[0])   # identical rows
    idx, sc = gpu_route(p, Qd, None, None, tab)
    check_no_device_error()
    gi = idx.cpu().numpy()
    for i in (63, 64 * 16 - 1, 64 * 40, n - 1):
        nv = min(n // B, (i + 1) // B)
        want = list(range(min(k, nv))) + [-1] * (k - min(k, nv))
        for g in range(2):
            assert gi[0, i, g].tolist() == want, (i, g)
            s = sc[0, i, g, :min(k, nv)].cpu()
            assert torch.all(s == s[0])


@pytest.mark.parametrize("name", list(CASES))
def test_attention_matches_oracle_on_oracle_selection(name):
    c = case(name)
    p = params(c["pd"])
    Q, K, V = to_dev(c["Q"], c["K"], c["V"])
    idx = torch.from_numpy(c["ref"]["block_idx"].astype(np.int32)).cuda()
    O_, lse, bad = gpu_attn(p, Q, K, V, idx)
    check_no_device_error()
    assert int(bad.item()) == 0
    max_abs, rel, ok = compare_out(as_np(O_), c["ref"]["O"], c["w"].dtype)
    assert ok, (max_abs, rel)
    np.testing.assert_allclose(lse.cpu().numpy(), c["ref"]["lse"], rtol=0, atol=2e-3 if c["w"].dtype == "bf16" else 1e-4)


@pytest.mark.parametrize("name", list(CASES))
def test_forward_end_to_end(name):
    c = case(name)
    p = params(c["pd"])
    Q, K, V = to_dev(c["Q"], c["K"], c["V"])
    ws = ssa.byte_buffer(ssa.ssa_workspace_size(p))
    O_ = torch.empty_like(Q)
    lse = torch.empty(Q.shape[:3], dtype=torch.float32, device="cuda")
    ssa.ssa_forward(p, Q, K, V, O_, lse, ws)
    check_no_device_error()
    gaps = c["ref"]["gaps"]                      # [b, n_q, h_kv]
    keep = np.all(gaps >= NEAR_TIE_BAND, axis=2)   # rows with no near-tie in any kv-head
    got = as_np(O_)
    max_abs, rel, ok = compare_out(got[keep], c["ref"]["O"][keep], c["w"].dtype)
    assert ok, (max_abs, rel)
    # the staged calls run the same kernels: identical bytes
    mu, sig, tab = gpu_summary(p, K)
    idx, _ = gpu_route(p, Q, mu, sig, tab)
    O2, lse2, _ = gpu_attn(p, Q, K, V, idx)
    assert torch.equal(O_, O2) and torch.equal(lse, lse2)


def test_hostio_matches_device_forward():
    c = case("bf16_gqa4_d128_b64")
    p = params(c["pd"])
    Q, K, V = to_dev(c["Q"], c["K"], c["V"])
    ws = ssa.byte_buffer(ssa.ssa_workspace_size(p))
    O_ = torch.empty_like(Q)
    ssa.ssa_forward(p, Q, K, V, O_, None, ws)
    hQ, hK, hV = (t.pin_memory() for t in (c["Q"], c["K"], c["V"]))
    hO = torch.empty_like(c["Q"]).pin_memory()
    hl = torch.empty(c["Q"].shape[:3], dtype=torch.float32).pin_memory()
    buf = ssa.byte_buffer(ssa.ssa_hostio_buffer_size(p))
    ssa.ssa_forward_hostio(p, hQ, hK, hV, hO, hl, buf)
    torch.cuda.synchronize()
    assert torch.equal(hO, O_.cpu())


def test_decode_row_equals_last_prefill_row():
    w = Workload("c", 110, 3, 2048, 8, 2, 128, "bf16", 64, "diag", 8, 256, 4, "per_seq", decode=True)
    Q, K, V, _ = make_inputs(w, "cpu")
    pd = problem_dict(w)
    op = O.Problem(**pd)
    ref = O.forward(Q.float().numpy(), K.float().numpy(), V.float().numpy(), op)
    p = params(pd)
    Qd, Kd, Vd = to_dev(Q, K, V)
    mu, sig, tab = gpu_summary(p, Kd)
    idx, _ = gpu_route(p, Qd, mu, sig, tab)
    O_, lse, _ = gpu_attn(p, Qd, Kd, Vd, idx)
    check_no_device_error()
    n, strict, _, _ = compare_idx(idx.cpu().numpy(), ref["block_idx"], ref["gaps"])
    assert strict == 0
    _, _, ok = compare_out(as_np(O_), ref["O"], "bf16")
    assert ok
    # the decode row is the prefill definition's last row
    pp = O.Problem(**{**pd, "n_q": w.n, "q_offset": 0})
    Qfull = np.zeros((w.batch, w.n, w.h_q, w.d))
    Qfull[:, -1] = Q.float().numpy()[:, 0]
    last = O.forward(Qfull, K.float().numpy(), V.float().numpy(), pp, rows=[(b, w.n - 1) for b in range(w.batch)])
    np.testing.assert_allclose(last["O"][:, -1], ref["O"][:, 0], atol=1e-12)


def test_full_budget_is_dense_causal_attention():
    w = Workload("c", 111, 1, 1024, 8, 2, 128, "bf16", 64, "diag", 16, 64, 0, "total")
    Q, K, V, _ = make_inputs(w, "cpu")
    pd = problem_dict(w)
    op = O.Problem(**pd)
    Od, _ = O.dense_causal_attention(Q.float().numpy(), K.float().numpy(), V.float().numpy(), op)
    p = params(pd)
    Qd, Kd, Vd = to_dev(Q, K, V)
    ws = ssa.byte_buffer(ssa.ssa_workspace_size(p))
    O_ = torch.empty_like(Qd)
    ssa.ssa_forward(p, Qd, Kd, Vd, O_, None, ws)
    check_no_device_error()
    _, _, ok = compare_out(as_np(O_), Od, "bf16")
    assert ok


def _clean_row(row, nvis):
    out, run = [], -1
    for v in row:
        if 0 <= v < nvis:
            if v > run:
                out.append(v)
            run = max(run, v)
    return out


def test_invalid_block_indices_are_skipped_and_counted():
    c = case("bf16_gqa4_d128_b64")
    op = c["op"]
    p = params(c["pd"])
    rng = np.random.default_rng(5)
    idx = c["ref"]["block_idx"].copy()
    n_bad = 0
    for _ in range(300):
        b, i, g = rng.integers(0, op.batch), rng.integers(0, op.n_q), rng.integers(0, op.h_kv)
        j = rng.integers(0, op.topk)
        idx[b, i, g, j] = rng.choice([op.nb + 3, -5, 10 ** 6, idx[b, i, g, max(j - 1, 0)], 0])
    expect_bad = 0
    clean = np.full_like(idx, -1)
    for b in range(op.batch):
        for i in range(op.n_q):
            nv = O.visible_blocks(i, op)
            for g in range(op.h_kv):
                row = list(idx[b, i, g])
                kept = _clean_row(row, nv)
                expect_bad += sum(1 for v in row if v != -1) - len(kept)
                clean[b, i, g, :len(kept)] = kept
    Q, K, V = to_dev(c["Q"], c["K"], c["V"])
    O_, _, bad = gpu_attn(p, Q, K, V, torch.from_numpy(idx.astype(np.int32)).cuda())
    check_no_device_error()
    assert int(bad.item()) == expect_bad and expect_bad > 0
    rows = [(b, i) for b in range(op.batch) for i in range(0, op.n_q, 7)]
    Oref, _ = O.attention(c["Qn"], c["Kn"], c["Vn"], clean, op, rows=rows)
    got = as_np(O_)
    for b, i in rows:
        assert np.abs(got[b, i] - Oref[b, i]).max() < 2e-2
    del n_bad


def test_window_of_one_key_and_early_rows():
    w = Workload("c", 112, 1, 640, 4, 4, 64, "bf16", 64, "diag", 4, 1, 0, "total")
    Q, K, V, _ = make_inputs(w, "cpu")
    pd = problem_dict(w)
    op = O.Problem(**pd)
    ref = O.forward(Q.float().numpy(), K.float().numpy(), V.float().numpy(), op)
    p = params(pd)
    Qd, Kd, Vd = to_dev(Q, K, V)
    ws = ssa.byte_buffer(ssa.ssa_workspace_size(p))
    O_ = torch.empty_like(Qd)
    ssa.ssa_forward(p, Qd, Kd, Vd, O_, None, ws)
    check_no_device_error()
    keep = np.all(ref["gaps"] >= NEAR_TIE_BAND, axis=2)
    _, _, ok = compare_out(as_np(O_)[keep], ref["O"][keep], "bf16")
    assert ok
    # rows before the first full block attend only to themselves: o = v_pos
    got = as_np(O_)
    for i in range(63):
        np.testing.assert_allclose(got[0, i], np.repeat(V.float().numpy()[0, i], 1, axis=0), atol=1e-2)


def test_empty_problem_launches_nothing_and_small_workspace_is_rejected():
    before = ssa.ssa_launch_count()
    p = ssa.make_params(0, 128, 128, 2, 2, 128, 64, 4, 64)
    ssa.ssa_forward(p, None, None, None, None, None, None)
    assert ssa.ssa_launch_count() == before
    c = case("bf16_gqa4_d128_b64")
    p = params(c["pd"])
    Q, K, V = to_dev(c["Q"], c["K"], c["V"])
    O_ = torch.empty_like(Q)
    small = ssa.byte_buffer(ssa.ssa_workspace_size(p) - 4096)
    with pytest.raises(ssa.SSAError) as e:
        ssa.ssa_forward(p, Q, K, V, O_, None, small)
    assert e.value.status == ssa.SSA_ERR_WORKSPACE
    assert ssa.ssa_launch_count() == before


# Problems the block-major attention takes (bf16, d = 128, G in {1, 2, 4, 8},
# k * G <= 128, at least 1024 query rows, a window over at most 32 key
# blocks) when it is given its workspace.
BLOCK_MAJOR = [n for n, w in CASES.items()
               if w.dtype == "bf16" and w.d == 128 and w.h_q // w.h_kv in (1, 2, 4, 8)
               and w.topk * (w.h_q // w.h_kv) <= 128 and w.n_q >= 1024
               and (w.window + w.block - 2) // w.block + 1 <= 32]


def test_block_major_cases_exist():
    assert len(BLOCK_MAJOR) >= 3
    assert "bf16_mha_d128_b64_k32" in BLOCK_MAJOR          # G = 1: 128 queries per tile
    for n in BLOCK_MAJOR:
        assert ssa.ssa_attn_workspace_size(params(problem_dict(CASES[n]))) > 0
    assert ssa.ssa_attn_workspace_size(params(problem_dict(CASES["bf16_gqa2_d64_b64"]))) == 0   # d = 64
    assert "bf16_gqa4_d128_b64_w1985" in BLOCK_MAJOR                # 32 window blocks
    assert ssa.ssa_attn_workspace_size(params(problem_dict(CASES["bf16_gqa4_d128_b64_w4032"]))) == 0


@pytest.mark.parametrize("name", BLOCK_MAJOR)
def test_block_major_attention_matches_oracle_and_gather(name):
    c = case(name)
    p = params(c["pd"])
    Q, K, V = to_dev(c["Q"], c["K"], c["V"])
    idx = torch.from_numpy(c["ref"]["block_idx"].astype(np.int32)).cuda()
    n0 = ssa.ssa_launch_count()
    Ob, lb, bad_b = gpu_attn(p, Q, K, V, idx, workspace=True)
    n1 = ssa.ssa_launch_count()
    Og, lg, bad_g = gpu_attn(p, Q, K, V, idx, workspace=False)
    n2 = ssa.ssa_launch_count()
    check_no_device_error()
    assert n2 - n1 == 1 and n1 - n0 > 1        # gather: one kernel; block-major: plan, tiles, merge
    assert int(bad_b.item()) == 0 and int(bad_g.item()) == 0
    for got, lse in ((Ob, lb), (Og, lg)):
        max_abs, rel, ok = compare_out(as_np(got), c["ref"]["O"], "bf16")
        assert ok, (max_abs, rel)
        np.testing.assert_allclose(lse.cpu().numpy(), c["ref"]["lse"], rtol=0, atol=2e-3)
    # each path is within the bf16 bound of the oracle, so the two are within twice it
    assert float((Ob.float() - Og.float()).abs().max()) <= 2 * 2e-2


def test_block_major_with_query_offset():
    """A chunk of query rows [n - 1024, n) at q_offset = n - 1024 gives the
    full problem's last 1024 rows."""
    c = case("bf16_gqa4_d128_b64_k32_b2")
    w = c["w"]
    m = 1024
    pd = {**c["pd"], "n_q": m, "q_offset": w.n - m}
    p = params(pd)
    Q = c["Q"][:, w.n - m:].contiguous()
    Qd, K, V = to_dev(Q, c["K"], c["V"])
    idx = torch.from_numpy(np.ascontiguousarray(c["ref"]["block_idx"][:, w.n - m:]).astype(np.int32)).cuda()
    assert ssa.ssa_attn_workspace_size(p) > 0
    O_, lse, bad = gpu_attn(p, Qd, K, V, idx)
    check_no_device_error()
    assert int(bad.item()) == 0
    max_abs, rel, ok = compare_out(as_np(O_), c["ref"]["O"][:, w.n - m:], "bf16")
    assert ok, (max_abs, rel)
    np.testing.assert_allclose(lse.cpu().numpy(), c["ref"]["lse"][:, w.n - m:], rtol=0, atol=2e-3)


def test_block_major_without_selections_is_window_attention():
    """Every block_idx entry -1: no block tile runs and each row attends to
    its causal window alone."""
    c = case("bf16_gqa8_d128_b128_k16")
    op = c["op"]
    p = params(c["pd"])
    Q, K, V = to_dev(c["Q"], c["K"], c["V"])
    none = np.full(c["ref"]["block_idx"].shape, -1, dtype=np.int32)
    O_, lse, bad = gpu_attn(p, Q, K, V, torch.from_numpy(none).cuda())
    check_no_device_error()
    assert int(bad.item()) == 0
    rows = [(0, i) for i in range(0, op.n_q, 5)]
    Oref, Lref = O.attention(c["Qn"], c["Kn"], c["Vn"], none, op, rows=rows)
    got = as_np(O_)
    ri = [i for _, i in rows]
    max_abs, rel, ok = compare_out(got[0, ri], Oref[0, ri], "bf16")
    assert ok, (max_abs, rel)


def test_block_major_stages_equal_single_call():
    c = case("bf16_gqa4_d128_b64_k32_b2")
    p = params(c["pd"])
    Q, K, V = to_dev(c["Q"], c["K"], c["V"])
    idx = torch.from_numpy(c["ref"]["block_idx"].astype(np.int32)).cuda()
    O1, l1, b1 = gpu_attn(p, Q, K, V, idx)
    ws = ssa.byte_buffer(ssa.ssa_attn_workspace_size(p))
    O2 = torch.empty_like(Q)
    l2 = torch.empty(Q.shape[:3], dtype=torch.float32, device="cuda")
    b2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    ssa.ssa_attn_plan(p, idx, ws)
    ssa.ssa_attn_blocks(p, Q, K, V, ws)
    ssa.ssa_attn_window(p, Q, K, V, ws)
    ssa.ssa_attn_merge(p, idx, O2, l2, b2, ws)
    check_no_device_error()
    assert torch.equal(O1, O2) and torch.equal(l1, l2) and int(b2.item()) == int(b1.item()) == 0


def test_block_major_one_key_window_and_single_block():
    """W = 1 and k = 1 on the block-major path: every row's window slot is
    masked down to its own key, rows before the first full block attend to
    themselves alone, and the rest add one selected block."""
    w = Workload("c", 117, 1, 1536, 8, 2, 128, "bf16", 64, "diag", 1, 1, 4, "total", clustered=True)
    Q, K, V, _ = make_inputs(w, "cpu")
    pd = problem_dict(w)
    op = O.Problem(**pd)
    ref = O.forward(Q.float().numpy(), K.float().numpy(), V.float().numpy(), op)
    p = params(pd)
    assert ssa.ssa_attn_workspace_size(p) > 0
    Qd, Kd, Vd = to_dev(Q, K, V)
    idx = torch.from_numpy(ref["block_idx"].astype(np.int32)).cuda()
    O_, lse, bad = gpu_attn(p, Qd, Kd, Vd, idx)
    check_no_device_error()
    assert int(bad.item()) == 0
    max_abs, rel, ok = compare_out(as_np(O_), ref["O"], "bf16")
    assert ok, (max_abs, rel)
    np.testing.assert_allclose(lse.cpu().numpy(), ref["lse"], rtol=0, atol=2e-3)
    got = as_np(O_)
    Vn = V.float().numpy()
    for i in range(63):                          # no full block yet: o = v_i for every head
        for h in range(w.h_q):
            np.testing.assert_allclose(got[0, i, h], Vn[0, i, h // (w.h_q // w.h_kv)], atol=1e-2)


def test_pair_tiles_when_one_block_of_the_pair_dominates():
    """256-key pair tiles (128-key blocks, G = 8) where one block's logits
    stand far above the other's: keys of one block of every pair are scaled
    by 8 (exact in bf16).  When the second block dominates, the softmax of
    the tile's second 128-key sub-tile must raise the running maximum and
    rescale the first sub-tile's O and row sum; when the first dominates,
    the second sub-tile's P stays far below 1.  Both against the oracle."""
    w = Workload("c", 141, 1, 3072, 8, 1, 128, "bf16", 128, "diag", 2, 256, 4, "total")
    Q, K, V, _ = make_inputs(w, "cpu")
    pd = problem_dict(w)
    op = O.Problem(**pd)
    nb = w.n // w.block
    Kf = K.float()
    for c in range(nb):
        # pairs (2j, 2j + 1): the second block dominates in the first half of
        # the sequence, the first block in the second half
        big = (c % 2 == 1) if c < nb // 2 else (c % 2 == 0)
        if big:
            Kf[:, c * w.block:(c + 1) * w.block] *= 8.0
    K = Kf.to(torch.bfloat16)
    idx = np.full((1, w.n, 1, 2), -1, dtype=np.int32)
    for i in range(w.n):
        npair = ((i + 1) // w.block) // 2          # fully visible pairs
        if npair:
            j = (i * 7) % npair
            idx[0, i, 0] = (2 * j, 2 * j + 1)
    Qn, Kn, Vn = Q.float().numpy(), K.float().numpy(), V.float().numpy()
    # the rescale is really exercised: for many rows the second block's
    # largest logit is more than 8 powers of two above the first block's
    log2e = 1.0 / np.log(2.0)
    up = down = rows = 0
    for i in range(0, w.n, 16):
        c1, c2 = idx[0, i, 0]
        if c1 < 0:
            continue
        s1 = Qn[0, i] @ Kn[0, c1 * w.block:(c1 + 1) * w.block, 0].T * op.scale * log2e
        s2 = Qn[0, i] @ Kn[0, c2 * w.block:(c2 + 1) * w.block, 0].T * op.scale * log2e
        jump = s2.max(axis=1) - s1.max(axis=1)       # per head
        rows += 1
        up += bool(jump.max() > 8)
        down += bool(jump.min() < -8)
    assert up > 0.25 * rows and down > 0.05 * rows, (up, down, rows)
    Oref, Lref = O.attention(Qn, Kn, Vn, idx, op)
    p = params(pd)
    assert ssa.ssa_attn_workspace_size(p) > 0
    Qd, Kd, Vd = to_dev(Q, K, V)
    O_, lse, bad = gpu_attn(p, Qd, Kd, Vd, torch.from_numpy(idx).cuda())
    check_no_device_error()
    assert int(bad.item()) == 0
    max_abs, rel, ok = compare_out(as_np(O_), Oref, "bf16")
    assert ok, (max_abs, rel)
    np.testing.assert_allclose(lse.cpu().numpy(), Lref, rtol=0, atol=2e-3)


def test_bounded_wait_gives_up_reports_its_site_and_leaves_the_context_usable():
    """A wait that nothing completes (the library's self-test kernel) gives up
    after the 1 s limit, names its site in the failure word, which reading
    clears, and the layer still runs correctly on the same context."""
    import time
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0
    t0 = time.perf_counter()
    ssa.ssa_selftest_wait_timeout()
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert 0.9 < dt < 60, dt
    assert ssa.ssa_device_error() == ssa.SITE_SELFTEST
    assert ssa.ssa_device_error() == 0
    c = case("bf16_gqa4_d128_b64")
    p = params(c["pd"])
    Q, K, V = to_dev(c["Q"], c["K"], c["V"])
    ws = ssa.byte_buffer(ssa.ssa_workspace_size(p))
    O_ = torch.empty_like(Q)
    ssa.ssa_forward(p, Q, K, V, O_, None, ws)
    check_no_device_error()
    keep = np.all(c["ref"]["gaps"] >= NEAR_TIE_BAND, axis=2)
    max_abs, rel, ok = compare_out(as_np(O_)[keep], c["ref"]["O"][keep], "bf16")
    assert ok, (max_abs, rel)
