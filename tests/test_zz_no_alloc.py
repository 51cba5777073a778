"""ssa_route_topk_static: routing without a caller workspace.

Some callers cannot allocate device memory when they route (a host framework
whose allocator owns the whole device pool, or a loop that cannot afford
cudaMalloc's implicit synchronisation).  For them the library keeps the
router's feature scratch in a fixed device array.  This file checks, through
the C ABI, that the static variant selects exactly what the workspace variant
selects on two calls in a row (different problems, so the second call runs
over the first call's leftover scratch), and that a problem too large for
the array is refused before anything is launched.  It is named to be
collected last and works alone in a fresh process or after the other tests.
"""
import ctypes as C

import pytest
import torch

from content_routed_block_ssa_b200 import ssa
from content_routed_block_ssa_b200.workload import Workload, make_inputs, problem_dict

pytestmark = pytest.mark.gpu


def _route_both(w):
    Q, K, V, _ = make_inputs(w, "cpu")
    p = ssa.make_params(**problem_dict(w))
    Qd, Kd = Q.cuda(), K.cuda()
    _, _, tab_s = ssa.summary_shapes(p)
    tab = torch.empty(tab_s, dtype=torch.bfloat16, device="cuda")
    ssa.ssa_block_summary(p, Kd, None, None, tab)
    ref_idx = torch.empty(ssa.idx_shape(p), dtype=torch.int32, device="cuda")
    ref_sc = torch.empty(ssa.idx_shape(p), dtype=torch.float32, device="cuda")
    ws = ssa.byte_buffer(ssa.ssa_route_workspace_size(p))
    ssa.ssa_route_topk(p, Qd, None, None, tab, ref_idx, ref_sc, ws)
    idx = torch.full(ssa.idx_shape(p), -7, dtype=torch.int32, device="cuda")
    sc = torch.full(ssa.idx_shape(p), 7.0, dtype=torch.float32, device="cuda")
    st = ssa.lib.ssa_route_topk_static(C.byref(p), Qd.data_ptr(), None, None, tab.data_ptr(),
                                       idx.data_ptr(), sc.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == ssa.SSA_OK, ssa.status_string(st)
    torch.cuda.synchronize()
    assert ssa.ssa_device_error() == 0
    assert ssa.ssa_route_workspace_size(p) > 0          # the tiled router uses scratch
    return ref_idx, ref_sc, idx, sc


def test_static_scratch_route_matches_workspace_route_twice():
    w1 = Workload("z", 201, 1, 2048, 8, 2, 128, "bf16", 64, "diag", 16, 256, 8, "total", clustered=True)
    w2 = Workload("z", 202, 2, 1152, 4, 4, 64, "bf16", 128, "diag", 8, 128, 4, "total")
    for w in (w1, w2):
        ref_idx, ref_sc, idx, sc = _route_both(w)
        # same kernels on the same inputs: identical selections and scores
        assert torch.equal(idx, ref_idx)
        assert torch.equal(sc, ref_sc)


def test_static_scratch_route_at_exactly_its_size():
    # 4 kv-heads x 8192 rows x 256 bf16 features: exactly 16 MiB of feature rows
    w = Workload("z", 203, 1, 8192, 16, 4, 128, "bf16", 64, "diag", 8, 128, 4, "total", clustered=True)
    assert w.batch * w.h_kv * w.n * 2 * w.d * 2 == ssa.ROUTE_STATIC_SCRATCH_BYTES
    ref_idx, ref_sc, idx, sc = _route_both(w)
    assert torch.equal(idx, ref_idx)
    assert torch.equal(sc, ref_sc)


def test_static_scratch_rejects_problems_beyond_its_size():
    # one (query row, kv-head) pair more than fits: 4 x 8193 rows x 512 bytes
    p1 = ssa.make_params(1, 8193, 8256, 16, 4, 128, 64, 8, 128)
    assert 4 * 8193 * 2 * 128 * 2 == ssa.ROUTE_STATIC_SCRATCH_BYTES + 4 * 512
    before = ssa.ssa_launch_count()
    st = ssa.lib.ssa_route_topk_static(C.byref(p1), 256, None, None, 256, 256, None, None)
    assert st == ssa.SSA_ERR_WORKSPACE
    assert ssa.ssa_launch_count() == before
    # 8 kv-heads x 8192 rows x 256 bf16 features = 32 MiB of feature rows > 16 MiB
    p = ssa.make_params(1, 8192, 8192, 8, 8, 128, 64, 8, 64)
    assert ssa.ssa_route_workspace_size(p) > ssa.ROUTE_STATIC_SCRATCH_BYTES
    before = ssa.ssa_launch_count()
    st = ssa.lib.ssa_route_topk_static(C.byref(p), 256, None, None, 256, 256, None, None)
    assert st == ssa.SSA_ERR_WORKSPACE
    assert ssa.ssa_launch_count() == before
