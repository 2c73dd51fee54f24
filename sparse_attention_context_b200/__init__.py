"""B200-native (sm_100a) In-context Sparse Attention (ISA) forward.

The four ISA stages (context pre-selection, query sharpness and routing,
full attention for routed queries, 0-th order Taylor attention for the rest)
and an in-house dense flash-attention baseline run as hand-written CUDA
kernels in ``libisa.so`` behind the C ABI of ``include/isa.h``; this package
binds that ABI for torch tensors (``api``) and splits problems over ranks
by heads (``sharding``).
"""
from ._lib import IsaError, IsaShape, LIB_PATH, lib  # noqa: F401
from .api import (  # noqa: F401
    dense_workspace, isa_attn_fwd, isa_dense_attn_fwd, isa_forward, isa_forward_blocks, isa_forward_static,
    isa_forward_taylor1, isa_full_attn_fwd, isa_full_attn_rows_fwd, isa_n_keep, isa_n_route, isa_n_route_blocks,
    isa_preselect_ctx, isa_read_device_status, isa_route_blocks_taylor_fwd, isa_route_queries,
    isa_route_taylor_fwd, isa_selftest_umma, isa_taylor1_attn_fwd, isa_taylor_attn_fwd, isa_workspace_size,
    make_shape, new_workspace, taylor1_workspace,
)
