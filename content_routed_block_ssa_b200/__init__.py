"""B200-native forward pass of one content-routed block-sparse attention layer.

The compute path is the CUDA library ``libssa.so`` (C ABI in include/ssa.h),
reached through the ctypes binding in ``content_routed_block_ssa_b200.ssa``
(import it explicitly: importing the package itself loads nothing, so the
seeded workload generator in ``.workload`` is usable without a GPU).
"""
