"""ctypes binding of libssa (include/ssa.h): argument marshalling only.

Every function takes torch tensors (device or, for ``ssa_forward_hostio``,
host) or None, passes their data pointers and the CUDA stream to the C ABI,
and raises ``SSAError`` on a non-zero status.  All computation happens in the
CUDA kernels behind the ABI; there is no other implementation to fall back
to, and importing this module fails if ``libssa.so`` has not been built.
"""
from __future__ import annotations

import ctypes as C
import math
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libssa.so")

SSA_OK, SSA_ERR_INVALID_ARG, SSA_ERR_UNSUPPORTED, SSA_ERR_WORKSPACE, SSA_ERR_CUDA, SSA_ERR_DEVICE = range(6)
SSA_F32, SSA_BF16 = 0, 1
SSA_SIGMA_DIAG, SSA_SIGMA_FULL = 0, 1
SSA_ROUTE_AUTO, SSA_ROUTE_TILED, SSA_ROUTE_ROWWISE = 0, 1, 2


class SSAError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


class ssa_params(C.Structure):
    _fields_ = [("batch", C.c_int32), ("n_q", C.c_int32), ("n_kv", C.c_int32), ("h_q", C.c_int32),
                ("h_kv", C.c_int32), ("d", C.c_int32), ("block", C.c_int32), ("topk", C.c_int32),
                ("window", C.c_int32), ("dtype", C.c_int32), ("sigma", C.c_int32),
                ("route_impl", C.c_int32), ("q_offset", C.c_int64), ("beta", C.c_float),
                ("scale", C.c_float), ("subblocks", C.c_int32), ("outlier", C.c_int32)]


assert C.sizeof(ssa_params) == 72


class ssa_hier_params(C.Structure):
    _fields_ = [("fanout", C.c_int32), ("probe", C.c_int32), ("escalate", C.c_int32), ("levels", C.c_int32)]


assert C.sizeof(ssa_hier_params) == 16


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"{_LIB_PATH} is missing: build it with "
                          "`python -m content_routed_block_ssa_b200.build` (nvcc, sm_100a)")
    lib = C.CDLL(_LIB_PATH)
    P = C.POINTER(ssa_params)
    H = C.POINTER(ssa_hier_params)
    vp, sz, i32 = C.c_void_p, C.c_size_t, C.c_int32
    sig = {
        "ssa_status_string": (C.c_char_p, [i32]),
        "ssa_version": (i32, []),
        "ssa_launch_count": (C.c_uint64, []),
        "ssa_device_error": (i32, [C.POINTER(C.c_uint32)]),
        "ssa_block_summary": (i32, [P, vp, vp, vp, vp, vp]),
        "ssa_route_workspace_size": (sz, [P]),
        "ssa_route_topk": (i32, [P, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "ssa_route_topk_static": (i32, [P, vp, vp, vp, vp, vp, vp, vp]),
        "ssa_attn_workspace_size": (sz, [P]),
        "ssa_attn_plan": (i32, [P, vp, vp, sz, vp]),
        "ssa_attn_blocks": (i32, [P, vp, vp, vp, vp, sz, vp]),
        "ssa_attn_window": (i32, [P, vp, vp, vp, vp, sz, vp]),
        "ssa_attn_merge": (i32, [P, vp, vp, vp, vp, vp, sz, vp]),
        "ssa_sparse_attn": (i32, [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "ssa_workspace_size": (sz, [P]),
        "ssa_forward": (i32, [P, vp, vp, vp, vp, vp, vp, sz, vp]),
        "ssa_hostio_buffer_size": (sz, [P]),
        "ssa_forward_hostio": (i32, [P, vp, vp, vp, vp, vp, vp, sz, vp]),
        "ssa_hier_nodes_size": (sz, [P, H]),
        "ssa_hier_nodes": (i32, [P, H, vp, vp, vp]),
        "ssa_route_hier_workspace_size": (sz, [P, H]),
        "ssa_route_hier": (i32, [P, H, vp, vp, vp, vp, vp, vp, sz, vp]),
        "ssa_selftest_wait_timeout": (i32, [vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()
LIB_PATH = _LIB_PATH
EXPORTED = ("ssa_status_string", "ssa_version", "ssa_launch_count", "ssa_device_error",
            "ssa_block_summary", "ssa_route_workspace_size", "ssa_route_topk", "ssa_route_topk_static",
            "ssa_attn_workspace_size", "ssa_sparse_attn", "ssa_attn_plan", "ssa_attn_blocks",
            "ssa_attn_window", "ssa_attn_merge",
            "ssa_workspace_size", "ssa_forward", "ssa_hostio_buffer_size", "ssa_forward_hostio",
            "ssa_hier_nodes_size", "ssa_hier_nodes", "ssa_route_hier_workspace_size", "ssa_route_hier",
            "ssa_selftest_wait_timeout")


def status_string(s: int) -> str:
    return lib.ssa_status_string(int(s)).decode()


def make_params(batch, n_q, n_kv, h_q, h_kv, d, block, topk, window, q_offset=0, beta=2.0,
                scale=None, dtype="bf16", sigma="diag", route_impl=SSA_ROUTE_AUTO, subblocks=1,
                outlier=False) -> ssa_params:
    """An ssa_params struct from plain values (dtype 'f32'|'bf16', sigma 'diag'|'full';
    outlier: add the outlier-channel row to every block's summaries)."""
    return ssa_params(batch=batch, n_q=n_q, n_kv=n_kv, h_q=h_q, h_kv=h_kv, d=d, block=block, topk=topk,
                      window=window, dtype={"f32": SSA_F32, "bf16": SSA_BF16}.get(dtype, dtype),
                      sigma={"diag": SSA_SIGMA_DIAG, "full": SSA_SIGMA_FULL}.get(sigma, sigma),
                      route_impl=route_impl, q_offset=q_offset, beta=beta,
                      scale=(1.0 / math.sqrt(d)) if scale is None else scale, subblocks=subblocks,
                      outlier=1 if outlier else 0)


def _ptr(t):
    """Address of a tensor's first element.  The C ABI reads every buffer as
    dense row-major memory, so a strided view (a transpose, a slice with a
    step, an array whose strides NumPy or torch kept from a permuted source)
    is refused rather than read in the wrong order."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError(f"libssa needs dense row-major buffers; got a tensor of shape {tuple(t.shape)} "
                         f"with strides {t.stride()} (call .contiguous() first)")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status, what):
    if status != SSA_OK:
        raise SSAError(status, what)


def ssa_launch_count() -> int:
    return int(lib.ssa_launch_count())


def ssa_device_error() -> int:
    code = C.c_uint32(0)
    st = lib.ssa_device_error(C.byref(code))
    if st not in (SSA_OK, SSA_ERR_DEVICE):
        raise SSAError(st, "ssa_device_error")
    return int(code.value)


def ssa_block_summary(p, K, mu=None, sigma=None, route_table=None, stream=None):
    _check(lib.ssa_block_summary(C.byref(p), _ptr(K), _ptr(mu), _ptr(sigma), _ptr(route_table),
                                 _stream(stream)), "ssa_block_summary")


def ssa_route_workspace_size(p) -> int:
    return int(lib.ssa_route_workspace_size(C.byref(p)))


def ssa_route_topk(p, Q, mu, sigma, route_table, block_idx, top_scores=None, ws=None, stream=None):
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib.ssa_route_topk(C.byref(p), _ptr(Q), _ptr(mu), _ptr(sigma), _ptr(route_table),
                              _ptr(block_idx), _ptr(top_scores), _ptr(ws), nbytes, _stream(stream)),
           "ssa_route_topk")


ROUTE_STATIC_SCRATCH_BYTES = 16 << 20


def ssa_route_topk_static(p, Q, mu, sigma, route_table, block_idx, top_scores=None, stream=None):
    """ssa_route_topk with the library's fixed scratch array instead of a workspace."""
    _check(lib.ssa_route_topk_static(C.byref(p), _ptr(Q), _ptr(mu), _ptr(sigma), _ptr(route_table),
                                     _ptr(block_idx), _ptr(top_scores), _stream(stream)),
           "ssa_route_topk_static")


def ssa_attn_workspace_size(p) -> int:
    return int(lib.ssa_attn_workspace_size(C.byref(p)))


def _nbytes(t):
    return t.numel() * t.element_size() if t is not None else 0


def ssa_attn_plan(p, block_idx, ws, stream=None):
    _check(lib.ssa_attn_plan(C.byref(p), _ptr(block_idx), _ptr(ws), _nbytes(ws), _stream(stream)), "ssa_attn_plan")


def ssa_attn_blocks(p, Q, K, V, ws, stream=None):
    _check(lib.ssa_attn_blocks(C.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(ws), _nbytes(ws), _stream(stream)),
           "ssa_attn_blocks")


def ssa_attn_window(p, Q, K, V, ws, stream=None):
    _check(lib.ssa_attn_window(C.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(ws), _nbytes(ws), _stream(stream)),
           "ssa_attn_window")


def ssa_attn_merge(p, block_idx, O, lse, bad_index_count, ws, stream=None):
    _check(lib.ssa_attn_merge(C.byref(p), _ptr(block_idx), _ptr(O), _ptr(lse), _ptr(bad_index_count), _ptr(ws),
                              _nbytes(ws), _stream(stream)), "ssa_attn_merge")


def ssa_sparse_attn(p, Q, K, V, block_idx, O, lse=None, bad_index_count=None, ws=None, stream=None):
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib.ssa_sparse_attn(C.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(block_idx), _ptr(O),
                               _ptr(lse), _ptr(bad_index_count), _ptr(ws), nbytes, _stream(stream)),
           "ssa_sparse_attn")


def ssa_workspace_size(p) -> int:
    return int(lib.ssa_workspace_size(C.byref(p)))


def ssa_forward(p, Q, K, V, O, lse=None, ws=None, stream=None):
    nbytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib.ssa_forward(C.byref(p), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse), _ptr(ws), nbytes,
                           _stream(stream)), "ssa_forward")


def ssa_hostio_buffer_size(p) -> int:
    return int(lib.ssa_hostio_buffer_size(C.byref(p)))


def ssa_forward_hostio(p, hQ, hK, hV, hO, hlse=None, dev_buf=None, stream=None):
    nbytes = dev_buf.numel() * dev_buf.element_size() if dev_buf is not None else 0
    _check(lib.ssa_forward_hostio(C.byref(p), _ptr(hQ), _ptr(hK), _ptr(hV), _ptr(hO), _ptr(hlse),
                                  _ptr(dev_buf), nbytes, _stream(stream)), "ssa_forward_hostio")


# ---------------------------------------------------------------- buffers

def summary_shapes(p):
    """Shapes of mu, Sigma and the route table: one row per sub-block (and
    one more per block with the outlier channel)."""
    rows = (p.n_kv // p.block) * (max(p.subblocks, 1) + (1 if p.outlier else 0))
    mu = (p.batch, p.h_kv, rows, p.d)
    sig = mu + ((p.d,) if p.sigma == SSA_SIGMA_FULL else ())
    tab = (p.batch, p.h_kv, rows, 2 * p.d)
    return mu, sig, tab


def idx_shape(p):
    return (p.batch, p.n_q, p.h_kv, p.topk)


def byte_buffer(nbytes: int, device="cuda"):
    """A caller-owned uint8 buffer (workspaces are allocated by the caller)."""
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def make_hier_params(fanout=16, probe=2, escalate=False, levels=1) -> ssa_hier_params:
    """An ssa_hier_params struct: nodes of `fanout` blocks (and with levels=2
    super-nodes of `fanout` nodes), `probe` entries expanded per row and level."""
    return ssa_hier_params(fanout=fanout, probe=probe, escalate=1 if escalate else 0, levels=levels)


def ssa_hier_nodes_size(p, hp) -> int:
    return int(lib.ssa_hier_nodes_size(C.byref(p), C.byref(hp)))


def ssa_hier_nodes(p, hp, route_table, nodes, stream=None):
    _check(lib.ssa_hier_nodes(C.byref(p), C.byref(hp), _ptr(route_table), _ptr(nodes), _stream(stream)),
           "ssa_hier_nodes")


def ssa_route_hier_workspace_size(p, hp) -> int:
    return int(lib.ssa_route_hier_workspace_size(C.byref(p), C.byref(hp)))


def ssa_route_hier(p, hp, Q, route_table, nodes, block_idx, certified=None, ws=None, stream=None):
    _check(lib.ssa_route_hier(C.byref(p), C.byref(hp), _ptr(Q), _ptr(route_table), _ptr(nodes), _ptr(block_idx),
                              _ptr(certified), _ptr(ws), _nbytes(ws), _stream(stream)), "ssa_route_hier")


def hier_node_views(p, hp, nodes):
    """(node rows [b, h_kv, nn, 2d] bf16, radii [b, h_kv, nn] f32, bounds [b, h_kv, 2] f32) views of a
    node store (a uint8 device tensor of ssa_hier_nodes_size bytes)."""
    nn = (p.n_kv // p.block) // hp.fanout
    bgs = p.batch * p.h_kv

    def ru(x):
        return (x + 255) // 256 * 256
    t_bytes = bgs * nn * 2 * p.d * 2
    r_off = ru(t_bytes)
    b_off = r_off + ru(bgs * nn * 4)
    rows = nodes[:t_bytes].view(torch.bfloat16).view(p.batch, p.h_kv, nn, 2 * p.d)
    rad = nodes[r_off:r_off + bgs * nn * 4].view(torch.float32).view(p.batch, p.h_kv, nn)
    bnd = nodes[b_off:b_off + bgs * 8].view(torch.float32).view(p.batch, p.h_kv, 2)
    return rows, rad, bnd


def hier_super_views(p, hp, nodes):
    """(super-node rows [b, h_kv, ns, 2d] bf16, radii [b, h_kv, ns] f32, largest radius [b, h_kv] f32)
    views of a two-level node store."""
    nn = (p.n_kv // p.block) // hp.fanout
    ns = nn // hp.fanout
    bgs = p.batch * p.h_kv

    def ru(x):
        return (x + 255) // 256 * 256
    off = ru(bgs * nn * 2 * p.d * 2) + ru(bgs * nn * 4) + ru(bgs * 8)
    t_bytes = bgs * ns * 2 * p.d * 2
    r_off = off + ru(t_bytes)
    b_off = r_off + ru(bgs * ns * 4)
    rows = nodes[off:off + t_bytes].view(torch.bfloat16).view(p.batch, p.h_kv, ns, 2 * p.d)
    rad = nodes[r_off:r_off + bgs * ns * 4].view(torch.float32).view(p.batch, p.h_kv, ns)
    bnd = nodes[b_off:b_off + bgs * 4].view(torch.float32).view(p.batch, p.h_kv)
    return rows, rad, bnd


SITE_SELFTEST = 0x7F1


def ssa_selftest_wait_timeout(stream=None):
    """Launches the failure-path self-test kernel (a wait that times out after 1 s)."""
    _check(lib.ssa_selftest_wait_timeout(_stream(stream)), "ssa_selftest_wait_timeout")
