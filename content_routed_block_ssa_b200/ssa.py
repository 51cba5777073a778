"""Public Python entry points (re-exported from the ctypes binding)."""
from ._lib import *  # noqa: F401,F403
from ._lib import (SSAError, lib, make_params, ssa_block_summary, ssa_device_error, ssa_forward,  # noqa: F401
                   ssa_forward_hostio, ssa_hostio_buffer_size, ssa_launch_count, ssa_params,
                   ssa_route_topk, ssa_route_topk_static, ssa_route_workspace_size, ssa_sparse_attn,
                   ssa_attn_workspace_size, ssa_attn_plan, ssa_attn_blocks, ssa_attn_window, ssa_attn_merge,
                   ssa_workspace_size, status_string, ssa_hier_params, make_hier_params,
                   ssa_hier_nodes_size, ssa_hier_nodes, ssa_route_hier_workspace_size, ssa_route_hier,
                   hier_node_views, ssa_selftest_wait_timeout, SITE_SELFTEST, summary_shapes, idx_shape, byte_buffer, EXPORTED, LIB_PATH)
