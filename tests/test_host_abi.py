"""Host-side checks of the C ABI: no kernel is launched here.

The library must load, export every entry point ``include/ssa.h`` declares,
lay ``ssa_params`` out as the header says, and reject invalid or unsupported
arguments with the documented status codes before touching the GPU.
"""
import ctypes as C
import os
import re

import pytest

from content_routed_block_ssa_b200 import ssa

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "ssa.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SSA_API\s+[\w\s\*]+?\b(ssa_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 12
    lib = C.CDLL(ssa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(ssa.EXPORTED) == names


def test_params_layout_matches_header():
    assert C.sizeof(ssa.ssa_params) == 72
    assert ssa.ssa_params.q_offset.offset == 48
    assert ssa.ssa_params.beta.offset == 56
    assert ssa.ssa_params.scale.offset == 60
    assert ssa.ssa_params.subblocks.offset == 64
    assert ssa.ssa_params.outlier.offset == 68
    text = open(HEADER).read()
    body = text[text.index("typedef struct {"):text.index("} ssa_params;")]
    fields = re.findall(r"\b(int32_t|int64_t|float)\s+(\w+);", body)
    assert [f for _, f in fields] == [f for f, _ in ssa.ssa_params._fields_]


def test_status_strings():
    assert ssa.status_string(0) == "SSA_OK"
    assert ssa.status_string(3) == "SSA_ERR_WORKSPACE"
    assert ssa.status_string(99) == "SSA_ERR_UNKNOWN"
    assert ssa.lib.ssa_version() == 1000


def good(**kw):
    base = dict(batch=1, n_q=256, n_kv=256, h_q=4, h_kv=2, d=128, block=64, topk=4, window=64)
    base.update(kw)
    return ssa.make_params(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(n_kv=250), ssa.SSA_ERR_INVALID_ARG),              # n_kv % block
    (dict(h_q=3), ssa.SSA_ERR_INVALID_ARG),                 # h_q % h_kv
    (dict(topk=0), ssa.SSA_ERR_INVALID_ARG),
    (dict(window=0), ssa.SSA_ERR_INVALID_ARG),
    (dict(q_offset=1), ssa.SSA_ERR_INVALID_ARG),            # queries past the last key
    (dict(q_offset=-1), ssa.SSA_ERR_INVALID_ARG),
    (dict(batch=-1), ssa.SSA_ERR_INVALID_ARG),
    (dict(scale=0.0), ssa.SSA_ERR_INVALID_ARG),
    (dict(beta=float("nan")), ssa.SSA_ERR_INVALID_ARG),
    (dict(dtype=7), ssa.SSA_ERR_INVALID_ARG),
    (dict(route_impl=5), ssa.SSA_ERR_INVALID_ARG),
    (dict(d=96), ssa.SSA_ERR_UNSUPPORTED),
    (dict(block=32, n_kv=256), ssa.SSA_ERR_UNSUPPORTED),
    (dict(h_q=6, h_kv=2), ssa.SSA_ERR_UNSUPPORTED),         # G = 3
    (dict(topk=33), ssa.SSA_ERR_UNSUPPORTED),
    (dict(window=5000), ssa.SSA_ERR_UNSUPPORTED),
    (dict(sigma="full"), ssa.SSA_ERR_UNSUPPORTED),          # bf16 routes on a diagonal Sigma
    (dict(subblocks=0), ssa.SSA_ERR_INVALID_ARG),
    (dict(subblocks=3), ssa.SSA_ERR_INVALID_ARG),           # does not divide the block
    (dict(subblocks=4), ssa.SSA_ERR_UNSUPPORTED),           # 16-key sub-blocks
    (dict(subblocks=8, block=128), ssa.SSA_ERR_UNSUPPORTED),
    (dict(subblocks=64), ssa.SSA_ERR_UNSUPPORTED),
])
def test_invalid_and_unsupported_params(kw, code):
    p = good(**kw)
    dummy = 256   # any non-null, 16-byte-aligned value: validation fails first
    assert ssa.lib.ssa_block_summary(C.byref(p), dummy, None, None, dummy, None) == code
    assert ssa.lib.ssa_forward(C.byref(p), dummy, dummy, dummy, dummy, None, dummy, 1 << 30, None) == code
    assert ssa.lib.ssa_sparse_attn(C.byref(p), dummy, dummy, dummy, dummy, dummy, None, None, None, 0, None) == code
    assert ssa.lib.ssa_workspace_size(C.byref(p)) == 0


def test_outlier_field_is_a_flag():
    dummy = 256
    for v in (2, -1):
        p = good()
        p.outlier = v
        assert ssa.lib.ssa_block_summary(C.byref(p), dummy, None, None, dummy, None) == ssa.SSA_ERR_INVALID_ARG
        assert ssa.ssa_workspace_size(p) == 0
    # the outlier row is not combined with sub-block summaries, nor with the
    # hierarchical router
    p = good(subblocks=2, outlier=True)
    assert ssa.lib.ssa_block_summary(C.byref(p), dummy, None, None, dummy, None) == ssa.SSA_ERR_UNSUPPORTED
    p = good(outlier=True)
    assert ssa.ssa_hier_nodes_size(p, ssa.make_hier_params()) == 0
    # two summary rows per block
    mu, sig, tab = ssa.summary_shapes(p)
    assert mu == (1, 2, 2 * (256 // 64), 128) and tab == (1, 2, 2 * (256 // 64), 256)


def test_null_and_misaligned_pointers_rejected():
    p = good()
    assert ssa.lib.ssa_block_summary(None, 256, None, None, None, None) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.lib.ssa_block_summary(C.byref(p), None, None, None, 256, None) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.lib.ssa_block_summary(C.byref(p), 258, None, None, 256, None) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.lib.ssa_route_topk(C.byref(p), 256, None, None, None, 256, None, None, 0, None) == \
        ssa.SSA_ERR_INVALID_ARG                           # bf16 needs the route table
    assert ssa.lib.ssa_sparse_attn(C.byref(p), 256, 256, 256, None, 256, None, None, None, 0, None) == \
        ssa.SSA_ERR_INVALID_ARG
    assert ssa.lib.ssa_forward(C.byref(p), 256, 256, 264, 256, None, 256, 1 << 30, None) == \
        ssa.SSA_ERR_INVALID_ARG
    f32 = good(dtype="f32")
    assert ssa.lib.ssa_block_summary(C.byref(f32), 256, 256, 256, 256, None) == ssa.SSA_ERR_INVALID_ARG


def test_empty_problems_are_valid_noops():
    for kw in (dict(batch=0), dict(n_q=0, q_offset=0)):
        p = good(**kw)
        assert ssa.lib.ssa_forward(C.byref(p), None, None, None, None, None, None, 0, None) == ssa.SSA_OK
        assert ssa.lib.ssa_sparse_attn(C.byref(p), None, None, None, None, None, None, None, None, 0, None) == ssa.SSA_OK
        assert ssa.lib.ssa_route_topk(C.byref(p), None, None, None, None, None, None, None, 0, None) == ssa.SSA_OK


def test_workspace_sizes():
    p = good(n_q=1000, n_kv=1024)
    nb = 1024 // 64
    tab = 1 * 2 * nb * 256 * 2
    feat = 1 * 2 * 1000 * 256 * 2
    idx = 1 * 1000 * 2 * 4 * 4
    rnd = lambda x: (x + 255) // 256 * 256
    assert ssa.ssa_route_workspace_size(p) == rnd(feat)
    assert ssa.ssa_workspace_size(p) == rnd(tab) + rnd(feat) + rnd(idx)
    # with at least 32 blocks the tiled router also takes its seed arrays:
    # variance sums [bgs, nb] f32, seed blocks [bgs, nb/32, 128] i32 and the
    # seed rows [bgs * nb/32 * 128, 2d] bf16
    sp = good(n_q=1000, n_kv=4096)
    feat4 = 1 * 2 * 1000 * 256 * 2
    assert ssa.ssa_route_workspace_size(sp) == (rnd(feat4) + rnd(2 * 64 * 4) + rnd(2 * 2 * 128 * 4)
                                                + rnd(2 * 2 * 128 * 256 * 2))
    row = good(n_q=1, n_kv=1024, q_offset=1023)           # decode routes per row: no features
    assert ssa.ssa_route_workspace_size(row) == 0
    f32 = good(dtype="f32", sigma="full", d=64, h_q=2, n_q=128, n_kv=128)
    nb = 2
    assert ssa.ssa_workspace_size(f32) == rnd(2 * nb * 64 * 4) + rnd(2 * nb * 64 * 64 * 4) + rnd(128 * 2 * 4 * 4)
    h = ssa.ssa_hostio_buffer_size(p)
    assert h > ssa.ssa_workspace_size(p)
    # sub-block summaries: S route-table rows per block
    s2 = good(n_q=1000, n_kv=1024, subblocks=2)
    assert ssa.ssa_workspace_size(s2) == rnd(2 * tab) + rnd(feat) + rnd(idx)
    mu, sig, t = ssa.summary_shapes(s2)
    assert mu == (1, 2, 2 * 16, 128) and t == (1, 2, 2 * 16, 256)
    f4 = good(dtype="f32", sigma="full", d=64, h_q=2, n_q=128, n_kv=128, block=128, subblocks=4)
    assert ssa.ssa_workspace_size(f4) == rnd(2 * 4 * 64 * 4) + rnd(2 * 4 * 64 * 64 * 4) + rnd(128 * 2 * 4 * 4)


def test_block_major_workspace_and_stage_checks():
    # qualifies: bf16, d = 128, G = 4, k * G = 32, n_q >= 1024
    p = good(n_q=2048, n_kv=2048, topk=8, h_q=8, h_kv=2)
    aw = ssa.ssa_attn_workspace_size(p)
    assert aw > 0
    base = ssa.ssa_workspace_size(good(n_q=2048, n_kv=2048, topk=8, h_q=8, h_kv=2, d=64))
    assert ssa.ssa_workspace_size(p) >= aw
    # the partial outputs dominate: one bf16 row of d per (query, kv-head, slot, head)
    assert aw >= 2048 * 2 * 8 * 4 * 128 * 2
    del base
    # does not qualify: too few rows, d = 64, k * G > 128, float32
    for kw in (dict(n_q=1000, n_kv=1024), dict(d=64),
               dict(topk=32, h_q=16, h_kv=2), dict(dtype="f32", h_q=2, h_kv=1)):
        q = good(**{**dict(n_q=2048, n_kv=2048), **kw})
        assert ssa.ssa_attn_workspace_size(q) == 0, kw
        assert ssa.lib.ssa_attn_plan(C.byref(q), 256, 256, 1 << 40, None) == ssa.SSA_ERR_UNSUPPORTED
    # staged calls without (or with too little) workspace are refused before any launch
    before = ssa.ssa_launch_count()
    assert ssa.lib.ssa_attn_plan(C.byref(p), 256, None, 0, None) == ssa.SSA_ERR_WORKSPACE
    assert ssa.lib.ssa_attn_blocks(C.byref(p), 256, 256, 256, 256, aw - 16, None) == ssa.SSA_ERR_WORKSPACE
    assert ssa.lib.ssa_attn_merge(C.byref(p), 256, 256, None, None, 264, aw, None) == \
        ssa.SSA_ERR_WORKSPACE                                  # misaligned
    assert ssa.lib.ssa_attn_plan(C.byref(p), None, 256, aw, None) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.ssa_launch_count() == before
    # empty problems are no-ops for every stage
    e = good(n_q=0, q_offset=0)
    assert ssa.lib.ssa_attn_merge(C.byref(e), None, None, None, None, None, 0, None) == ssa.SSA_OK


def test_hier_params_layout_and_checks():
    assert C.sizeof(ssa.ssa_hier_params) == 16
    assert ssa.ssa_hier_params.escalate.offset == 8
    p = good(n_q=1000, n_kv=4096)
    dummy = 256
    ok = ssa.make_hier_params(fanout=8, probe=2, escalate=True)
    nb, nn, bgs = 4096 // 64, 4096 // 64 // 8, 2
    rnd = lambda x: (x + 255) // 256 * 256
    assert ssa.ssa_hier_nodes_size(p, ok) == rnd(bgs * nn * 256 * 2) + rnd(bgs * nn * 4) + rnd(bgs * 8)
    rows = 1000 * 2
    tiles = (1000 + 255) // 256
    assert ssa.ssa_route_hier_workspace_size(p, ok) == (rnd(rows * 256 * 2) + 2 * rnd(rows * 3 * 4) + rnd(rows)
                                                        + rnd(bgs * tiles * 4))
    no_esc = ssa.make_hier_params(fanout=8, probe=2, escalate=False)
    assert ssa.ssa_route_hier_workspace_size(p, ok) - ssa.ssa_route_hier_workspace_size(p, no_esc) == \
        rnd(bgs * tiles * 4)
    # two levels: the super-node rows, radii and largest radius after the
    # nodes; per row the super-node list (probe+1 entries and scores), the
    # candidate-node count and the best unexpanded super-node score
    two = ssa.make_hier_params(fanout=8, probe=2, escalate=True, levels=2)
    ns = nn // 8
    assert ssa.ssa_hier_nodes_size(p, two) == (ssa.ssa_hier_nodes_size(p, ok) + rnd(bgs * ns * 256 * 2)
                                               + rnd(bgs * ns * 4) + rnd(bgs * 4))
    assert ssa.ssa_route_hier_workspace_size(p, two) == (ssa.ssa_route_hier_workspace_size(p, ok)
                                                         + 2 * rnd(rows * 3 * 4) + 2 * rnd(rows * 4))
    assert ssa.ssa_hier_nodes_size(p, ssa.make_hier_params(fanout=8, probe=2, levels=0)) == \
        ssa.ssa_hier_nodes_size(p, ssa.make_hier_params(fanout=8, probe=2, levels=1))
    for hp, code in ((ssa.make_hier_params(fanout=3), ssa.SSA_ERR_INVALID_ARG),      # not a power of two
                     (ssa.make_hier_params(fanout=128), ssa.SSA_ERR_INVALID_ARG),
                     (ssa.make_hier_params(probe=0), ssa.SSA_ERR_INVALID_ARG),
                     (ssa.make_hier_params(probe=32), ssa.SSA_ERR_INVALID_ARG),
                     (ssa.ssa_hier_params(fanout=8, probe=2, escalate=2, levels=0), ssa.SSA_ERR_INVALID_ARG),
                     (ssa.ssa_hier_params(fanout=8, probe=2, escalate=0, levels=3), ssa.SSA_ERR_INVALID_ARG),
                     (ssa.ssa_hier_params(fanout=8, probe=2, escalate=0, levels=-1), ssa.SSA_ERR_INVALID_ARG),
                     (ssa.make_hier_params(fanout=64, probe=8), ssa.SSA_ERR_UNSUPPORTED)):   # 576 candidates
        assert ssa.ssa_hier_nodes_size(p, hp) == 0
        assert ssa.lib.ssa_hier_nodes(C.byref(p), C.byref(hp), dummy, dummy, None) == code
        assert ssa.lib.ssa_route_hier(C.byref(p), C.byref(hp), dummy, dummy, dummy, dummy, None, dummy,
                                      1 << 30, None) == code
    for kw in (dict(dtype="f32", sigma="diag"), dict(subblocks=2)):
        q = good(**kw)
        assert ssa.lib.ssa_hier_nodes(C.byref(q), C.byref(ok), dummy, dummy, None) == ssa.SSA_ERR_UNSUPPORTED
    assert ssa.lib.ssa_hier_nodes(C.byref(p), None, dummy, dummy, None) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.lib.ssa_hier_nodes(C.byref(p), C.byref(ok), 258, dummy, None) == ssa.SSA_ERR_INVALID_ARG
    assert ssa.lib.ssa_route_hier(C.byref(p), C.byref(ok), dummy, dummy, dummy, dummy, None, dummy, 16,
                                  None) == ssa.SSA_ERR_WORKSPACE
    e = good(batch=0)
    assert ssa.lib.ssa_route_hier(C.byref(e), C.byref(ok), None, None, None, None, None, None, 0, None) == ssa.SSA_OK


def test_hier_node_views_match_the_node_store_layout():
    """The binding's views of a node store (rows, radii, bounds) tile the
    buffer the size call asks for, at the documented 256-byte-aligned offsets."""
    import torch
    for kw, M in ((dict(n_q=1000, n_kv=4096), 8), (dict(batch=2, n_kv=4288, n_q=4288, h_q=8, h_kv=2), 16),
                  (dict(n_kv=8192, n_q=1, q_offset=8191, d=64), 4)):
        p = good(**kw)
        hp = ssa.make_hier_params(fanout=M, probe=2)
        size = ssa.ssa_hier_nodes_size(p, hp)
        buf = torch.zeros(size, dtype=torch.uint8)
        rows, rad, bnd = ssa.hier_node_views(p, hp, buf)
        nn = (p.n_kv // p.block) // M
        assert rows.shape == (p.batch, p.h_kv, nn, 2 * p.d) and rad.shape == (p.batch, p.h_kv, nn)
        base = buf.data_ptr()
        assert rows.data_ptr() == base
        assert (rad.data_ptr() - base) % 256 == 0 and rad.data_ptr() - base >= rows.numel() * 2
        assert (bnd.data_ptr() - base) % 256 == 0 and bnd.data_ptr() - base >= rad.data_ptr() - base + rad.numel() * 4
        assert bnd.data_ptr() - base + bnd.numel() * 4 <= size


def test_binding_refuses_strided_tensors_before_calling_the_library():
    """The C ABI reads dense row-major buffers.  A tensor whose memory is in
    another order (here [b, nb, h_kv, d] memory viewed as [b, h_kv, nb, d],
    what a reduction over a transposed NumPy array gives) is refused by the
    binding; nothing reaches the library."""
    import numpy as np
    import torch
    p = good(dtype="f32")
    mem = torch.zeros(1, 4, 2, 128)                  # [b, nb, h_kv, d] in memory
    mu = mem.transpose(1, 2)                         # viewed as [b, h_kv, nb, d]
    assert not mu.is_contiguous()
    before = ssa.ssa_launch_count()
    with pytest.raises(ValueError, match="dense row-major"):
        ssa.ssa_route_topk(p, torch.zeros(1, 256, 4, 128), mu, mu.contiguous(), None,
                           torch.zeros(1, 256, 2, 4, dtype=torch.int32))
    assert ssa.ssa_launch_count() == before
    # the oracle's summaries are such arrays: a reduction keeps the source's order
    K = np.zeros((1, 256, 2, 128))
    m = K.reshape(1, 4, 64, 2, 128).transpose(0, 3, 1, 2, 4).sum(axis=3)
    assert not torch.from_numpy(m).is_contiguous()
