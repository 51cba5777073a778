"""GPU parity of the hierarchical router (node summaries, probe,
certificates, escalation) against the CPU oracle, through the C ABI.

Comparison rules: node rows are bit-exact and radii and bounds agree to a
float32 ulp; a row's kept blocks and its certificate are compared where
neither side's float32 rounding can decide them (the node ranking's p-th /
(p+1)-th gap, the kept set's k-th / (k+1)-th gap and the certificate's
margin all at least HIER_BAND * ||f|| T*, T* the largest row norm); a
certified row always holds the flat top-k; with escalation every row holds
it, compared like the flat router.
"""
import numpy as np
import pytest
import torch

from content_routed_block_ssa_b200 import ssa
from content_routed_block_ssa_b200.workload import Workload, make_inputs, problem_dict
from oracle import ssa_oracle as O
from parity_util import check_no_device_error, compare_idx, params

pytestmark = pytest.mark.gpu

HIER_BAND = 4e-5

# name: (workload, fanout, probe)
CASES = {
    # keys alike over runs of 16 blocks: certificates fire on many rows
    "gqa4_d128_b64_span16_M16_p2": (Workload("h", 131, 1, 4096, 8, 2, 128, "bf16", 64, "diag", 8, 256, 6,
                                             "total", clustered=True, cluster_span=16), 16, 2),
    # a centroid per block (the 128K workload's recipe): the bound is loose
    "gqa4_d128_b64_blockclusters_M8_p3": (Workload("h", 132, 1, 3072, 8, 2, 128, "bf16", 64, "diag", 16, 128, 6,
                                                   "total", clustered=True), 8, 3),
    "gqa8_d128_b128_span8_M8_p1": (Workload("h", 133, 1, 4096, 8, 1, 128, "bf16", 128, "diag", 8, 256, 8,
                                            "total", clustered=True, cluster_span=8), 8, 1),
    "mha_d64_b64_span4_M4_p2": (Workload("h", 134, 1, 2048, 2, 2, 64, "bf16", 64, "diag", 4, 64, 4, "per_head",
                                         clustered=True, cluster_span=4), 4, 2),
    # 67 blocks: 4 complete nodes of 16 and 3 trailing blocks
    "gqa4_d128_b64_ragged_M16_p1": (Workload("h", 136, 1, 4288, 8, 2, 128, "bf16", 64, "diag", 8, 256, 4,
                                             "total", clustered=True, cluster_span=16), 16, 1),
    # one query per sequence at the end of a 16K cache
    "decode_gqa4_d128_span16_M16_p2": (Workload("h", 135, 4, 16384, 8, 2, 128, "bf16", 64, "diag", 16, 256, 2,
                                                "per_seq", clustered=True, cluster_span=16, decode=True), 16, 2),
}

_cache = {}


def case(name):
    if name not in _cache:
        w, M, probe = CASES[name]
        Q, K, V, _plan = make_inputs(w, "cpu")
        pd = problem_dict(w)
        op = O.Problem(**pd)
        Qn, Kn = Q.float().numpy(), K.float().numpy()
        stored = O.stored_summaries(*O.block_summaries(Kn, op), op)
        flat, gaps = O.route_topk(Qn, stored, op)
        hb, hc, info = O.hier_route(Qn, stored, op, M, probe)
        _cache[name] = dict(w=w, M=M, probe=probe, pd=pd, op=op, Q=Q, Qn=Qn, stored=stored, flat=flat,
                            gaps=gaps, hb=hb, hc=hc, info=info, nodes=O.hier_nodes(stored[2], M))
    return _cache[name]


def impls(name):
    return (ssa.SSA_ROUTE_ROWWISE,) if CASES[name][0].decode else (ssa.SSA_ROUTE_TILED, ssa.SSA_ROUTE_ROWWISE)


PAIRS = [(n, i) for n in CASES for i in impls(n)]
IDS = [f"{n}-{'tiled' if i == ssa.SSA_ROUTE_TILED else 'rowwise'}" for n, i in PAIRS]


def gpu_nodes(c, p, hp):
    tab = torch.from_numpy(c["stored"][2]).to(torch.bfloat16).cuda()
    nodes = ssa.byte_buffer(ssa.ssa_hier_nodes_size(p, hp), "cuda")
    nodes.fill_(0xAB)
    ssa.ssa_hier_nodes(p, hp, tab, nodes)
    return tab, nodes


def gpu_hier(c, p, hp, tab, nodes):
    Q = c["Q"].cuda()
    idx = torch.full(ssa.idx_shape(p), -7, dtype=torch.int32, device="cuda")
    cert = torch.full(idx.shape[:3], 7, dtype=torch.uint8, device="cuda")
    ws = ssa.byte_buffer(ssa.ssa_route_hier_workspace_size(p, hp), "cuda")
    ssa.ssa_route_hier(p, hp, Q, tab, nodes, idx, cert, ws)
    check_no_device_error()
    return idx.cpu().numpy(), cert.cpu().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_hier_nodes_match_oracle(name):
    c = case(name)
    p = params(c["pd"])
    hp = ssa.make_hier_params(c["M"], c["probe"])
    _tab, nodes = gpu_nodes(c, p, hp)
    check_no_device_error()
    rows, rad, bnd = ssa.hier_node_views(p, hp, nodes)
    nt, radius, r_star, t_star = c["nodes"]
    assert np.array_equal(rows.float().cpu().numpy().astype(np.float64), nt)

    def ulps(a, b):
        a = np.asarray(a, np.float32)
        b = np.asarray(b, np.float32)
        return np.abs(a.view(np.int32).astype(np.int64) - b.view(np.int32).astype(np.int64))
    assert ulps(rad.cpu().numpy(), radius).max(initial=0) <= 1
    g = bnd.cpu().numpy()
    assert ulps(g[..., 0], r_star).max() <= 1 and ulps(g[..., 1], t_star).max() <= 1
    assert np.all(rad.cpu().numpy() >= 0)


def _decidable(c, bi, i, g):
    inf = c["info"][(bi, i, g)]
    band = HIER_BAND * inf["scale"]
    return (inf["node_gap"] >= band and inf["kept_gap"] >= band
            and (not np.isfinite(inf["bound"]) or abs(inf["tau"] - inf["bound"]) >= band))


@pytest.mark.parametrize("name,impl", PAIRS, ids=IDS)
def test_hier_probe_and_certificates_match_oracle(name, impl):
    c = case(name)
    op = c["op"]
    p = params(c["pd"], impl)
    hp = ssa.make_hier_params(c["M"], c["probe"], escalate=False)
    tab, nodes = gpu_nodes(c, p, hp)
    gi, gc = gpu_hier(c, p, hp, tab, nodes)
    assert set(np.unique(gc)) <= {0, 1}
    checked = mism = cmis = 0
    for bi in range(op.batch):
        for i in range(op.n_q):
            for g in range(op.h_kv):
                if gc[bi, i, g]:   # a certified row holds the flat top-k (outside flat near-ties)
                    if c["gaps"][bi, i, g] >= 1e-5:
                        assert np.array_equal(gi[bi, i, g], c["flat"][bi, i, g]), (bi, i, g)
                if not _decidable(c, bi, i, g):
                    continue
                checked += 1
                mism += int(not np.array_equal(gi[bi, i, g], c["hb"][bi, i, g]))
                cmis += int(bool(gc[bi, i, g]) != bool(c["hc"][bi, i, g]))
    total = op.batch * op.n_q * op.h_kv
    assert checked >= 0.8 * total, (checked, total)
    assert mism == 0 and cmis == 0, (mism, cmis, checked)


@pytest.mark.parametrize("name,impl", PAIRS, ids=IDS)
def test_hier_escalation_gives_the_flat_selection(name, impl):
    c = case(name)
    p = params(c["pd"], impl)
    hp = ssa.make_hier_params(c["M"], c["probe"], escalate=True)
    tab, nodes = gpu_nodes(c, p, hp)
    gi, gc = gpu_hier(c, p, hp, tab, nodes)
    n, strict, _lit, _band = compare_idx(gi, c["flat"], c["gaps"])
    assert strict == 0, f"{strict} of {n} rows differ from the flat top-k outside the near-tie band"


def test_hier_certificates_fire_on_alike_blocks_and_not_on_block_clusters():
    fired = {}
    for name in ("gqa4_d128_b64_span16_M16_p2", "gqa4_d128_b64_blockclusters_M8_p3"):
        c = case(name)
        p = params(c["pd"], ssa.SSA_ROUTE_TILED)
        hp = ssa.make_hier_params(c["M"], c["probe"])
        tab, nodes = gpu_nodes(c, p, hp)
        _gi, gc = gpu_hier(c, p, hp, tab, nodes)
        late = gc[:, c["op"].n_q // 2:]          # rows that see many nodes
        fired[name] = float(late.mean())
    assert fired["gqa4_d128_b64_span16_M16_p2"] > 0.3
    assert fired["gqa4_d128_b64_blockclusters_M8_p3"] < fired["gqa4_d128_b64_span16_M16_p2"]


# ------------------------------------------------------------------ two levels

# name: (workload, fanout, probe); nodes of M blocks, super-nodes of M nodes
CASES2 = {
    # keys alike over runs of 16 blocks: a super-node of 4 x 4 blocks is one run
    "gqa4_d128_b64_span16_M4_p2": (Workload("h", 141, 1, 4096, 8, 2, 128, "bf16", 64, "diag", 8, 256, 6,
                                            "total", clustered=True, cluster_span=16), 4, 2),
    # a centroid per block: loose bounds at both levels
    "gqa4_d128_b64_blockclusters_M4_p3": (Workload("h", 142, 1, 3072, 8, 2, 128, "bf16", 64, "diag", 16, 128, 6,
                                                   "total", clustered=True), 4, 3),
    # 70 blocks of 128 keys at M = 2: 35 nodes, 17 super-nodes and a trailing node
    "gqa8_d128_b128_ragged_M2_p2": (Workload("h", 143, 1, 8960, 8, 1, 128, "bf16", 128, "diag", 8, 256, 8,
                                             "total", clustered=True, cluster_span=4), 2, 2),
    "decode_gqa4_d128_span16_M4_p2": (Workload("h", 144, 4, 16384, 8, 2, 128, "bf16", 64, "diag", 16, 256, 2,
                                               "per_seq", clustered=True, cluster_span=16, decode=True), 4, 2),
}

_cache2 = {}


def case2(name):
    if name not in _cache2:
        w, M, probe = CASES2[name]
        Q, K, V, _plan = make_inputs(w, "cpu")
        pd = problem_dict(w)
        op = O.Problem(**pd)
        Qn, Kn = Q.float().numpy(), K.float().numpy()
        stored = O.stored_summaries(*O.block_summaries(Kn, op), op)
        flat, gaps = O.route_topk(Qn, stored, op)
        hb, hc, info = O.hier_route(Qn, stored, op, M, probe, levels=2)
        nodes = O.hier_nodes(stored[2], M)
        _cache2[name] = dict(w=w, M=M, probe=probe, pd=pd, op=op, Q=Q, Qn=Qn, stored=stored, flat=flat,
                             gaps=gaps, hb=hb, hc=hc, info=info, nodes=nodes,
                             supers=O.hier_super_nodes(nodes[0], nodes[1], nodes[3], M))
    return _cache2[name]


def impls2(name):
    return (ssa.SSA_ROUTE_ROWWISE,) if CASES2[name][0].decode else (ssa.SSA_ROUTE_TILED, ssa.SSA_ROUTE_ROWWISE)


PAIRS2 = [(n, i) for n in CASES2 for i in impls2(n)]
IDS2 = [f"{n}-{'tiled' if i == ssa.SSA_ROUTE_TILED else 'rowwise'}" for n, i in PAIRS2]


def _ulps(a, b):
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    return np.abs(a.view(np.int32).astype(np.int64) - b.view(np.int32).astype(np.int64))


@pytest.mark.parametrize("name", list(CASES2))
def test_hier_super_nodes_match_oracle(name):
    """Second level: super-node rows bit-exact; recursive radii, the largest
    radius and the row-norm bound (now over the super-node rows too) within a
    float32 ulp; the node level is unchanged by the second."""
    c = case2(name)
    p = params(c["pd"])
    hp = ssa.make_hier_params(c["M"], c["probe"], levels=2)
    _tab, nodes = gpu_nodes(c, p, hp)
    check_no_device_error()
    rows, rad, bnd = ssa.hier_node_views(p, hp, nodes)
    nt, radius, r_star, _t1 = c["nodes"]
    st, srad, r2, t2 = c["supers"]
    assert np.array_equal(rows.float().cpu().numpy().astype(np.float64), nt)
    assert _ulps(rad.cpu().numpy(), radius).max(initial=0) <= 1
    g = bnd.cpu().numpy()
    assert _ulps(g[..., 0], r_star).max() <= 1 and _ulps(g[..., 1], t2).max() <= 1
    srows, sr, sb = ssa.hier_super_views(p, hp, nodes)
    assert np.array_equal(srows.float().cpu().numpy().astype(np.float64), st)
    assert _ulps(sr.cpu().numpy(), srad).max(initial=0) <= 1
    assert _ulps(sb.cpu().numpy(), r2).max() <= 1


def _decidable2(c, bi, i, g):
    inf = c["info"][(bi, i, g)]
    band = HIER_BAND * inf["scale"]
    return (inf["super_gap"] >= band and inf["node_gap"] >= band and inf["kept_gap"] >= band
            and all(not np.isfinite(b) or abs(inf["tau"] - b) >= band for b in inf["bounds"]))


@pytest.mark.parametrize("name,impl", PAIRS2, ids=IDS2)
def test_hier_two_levels_probe_and_certificates_match_oracle(name, impl):
    c = case2(name)
    op = c["op"]
    p = params(c["pd"], impl)
    hp = ssa.make_hier_params(c["M"], c["probe"], escalate=False, levels=2)
    tab, nodes = gpu_nodes(c, p, hp)
    gi, gc = gpu_hier(c, p, hp, tab, nodes)
    assert set(np.unique(gc)) <= {0, 1}
    checked = mism = cmis = 0
    for bi in range(op.batch):
        for i in range(op.n_q):
            for g in range(op.h_kv):
                if gc[bi, i, g] and c["gaps"][bi, i, g] >= 1e-5:   # a certified row holds the flat top-k
                    assert np.array_equal(gi[bi, i, g], c["flat"][bi, i, g]), (bi, i, g)
                if not _decidable2(c, bi, i, g):
                    continue
                checked += 1
                mism += int(not np.array_equal(gi[bi, i, g], c["hb"][bi, i, g]))
                cmis += int(bool(gc[bi, i, g]) != bool(c["hc"][bi, i, g]))
    total = op.batch * op.n_q * op.h_kv
    assert checked >= 0.8 * total, (checked, total)
    assert mism == 0 and cmis == 0, (mism, cmis, checked)


@pytest.mark.parametrize("name,impl", PAIRS2, ids=IDS2)
def test_hier_two_levels_escalation_gives_the_flat_selection(name, impl):
    c = case2(name)
    p = params(c["pd"], impl)
    hp = ssa.make_hier_params(c["M"], c["probe"], escalate=True, levels=2)
    tab, nodes = gpu_nodes(c, p, hp)
    gi, _gc = gpu_hier(c, p, hp, tab, nodes)
    n, strict, _lit, _band = compare_idx(gi, c["flat"], c["gaps"])
    assert strict == 0, f"{strict} of {n} rows differ from the flat top-k outside the near-tie band"
