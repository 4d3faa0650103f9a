"""CPU fp64 oracle for NABLA block-sparse video attention (nabla.py) and for
the Token Radius Attention block mask (tra.py).

TEST INFRASTRUCTURE ONLY: the reference the CUDA path is checked against.
Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import it; the library never does, and the two share no code.
"""
from .nabla import (  # noqa: F401
    widen_bf16, fractal_order, flatten, unflatten, pool, reduced_map, cdf_keep,
    block_coords, sta_keep, pooled_head, nabla_mask, masked_attention,
    attention_head, nabla_attention, tile_shape, block_heatmap, block_heatmap_rows, heat_recall,
    masked_attention_backward, masked_attention_backward_blocks, attention_backward_head,
)
from .tra import (  # noqa: F401
    token_entropy, entropy_budget, budget_radius2, radius_support, radius_block_mask, tra_mask,
)
