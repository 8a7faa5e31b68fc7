"""fp64 CPU oracle of the ISA forward pass (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does.
"""
from .isa_oracle import *  # noqa: F401,F403
from .isa_oracle import (Params, HeadPlan, segment_blocks, pool, coarse_scores,
                         context_importance, topk_lower_index, softmax_rows, sharpness,
                         split_sharp_flat, plan_head, forward_head, dense_attention,
                         isa_forward, n_select, n_flat_blocks, n_exact_blocks,
                         sharp_block, flat_block, rope_decoupled,
                         backward_head, isa_backward, coarse_output,
                         coarse_residual, coarse_residual_backward)
