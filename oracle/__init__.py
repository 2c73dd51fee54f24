"""Float64 CPU oracle of the ISA attention forward (test infrastructure only)."""
from .isa_oracle import (  # noqa: F401
    block_layout, block_mean_sharpness, correction_matrices, block_means, block_saliency, dense, dense_head, full_rows, isa_fwd,
    guarded_count, isa_head, kept_blocks, kept_tokens, kth_value, n_keep_of, n_route_blocks_of, n_route_of,
    route_query_blocks, sharpness,
    taylor1_rows, taylor_rows, topk_ascending,
)
