"""fp64 CPU oracle of the BPT layer: test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA path never does.
"""
from .bpt_oracle import (  # noqa: F401
    LN_EPS, attention_rows, attention_stats_rows, ffn_residual, gelu, layer_blockwise,
    layer_intermediates,
    layer_norm, layer_rows, layer_unfused, online_softmax_init,
    online_softmax_update, softmax_rows,
)
from .bpt_backward import (  # noqa: F401
    GRAD_NAMES, attention_backward, gelu_grad, layer_backward, layer_backward_blockwise,
    layer_norm_backward,
)
from .bsfa import (  # noqa: F401
    attention_gated, block_max, calibrate_thresholds, head_scores, keep_mask, layer_block_max,
    layer_gated,
)
