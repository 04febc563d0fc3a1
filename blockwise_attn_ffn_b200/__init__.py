"""B200-native forward pass of one pre-LN Blockwise Parallel Transformer layer.

The layer runs in libbpt.so (hand-written sm_100a CUDA kernels behind a C
ABI, ``include/bpt.h``).  This package is the thin Python side: the ctypes
binding (``bpt_*`` functions with the C names), a torch-tensor convenience
call, the seeded input generator and the FLOP/byte accountant.
"""
from ._lib import (  # noqa: F401
    BPT_BF16, BPT_ERR_CUDA, BPT_ERR_INVALID_ARG, BPT_ERR_RANGE, BPT_ERR_TIMEOUT, BPT_ERR_UNSUPPORTED,
    BPT_ERR_WORKSPACE, BPT_F32, BPT_OK, BPT_SCHEDULE_FUSED, BPT_SCHEDULE_WAVES,
    BPT_STATIC_WORKSPACE_BYTES, BPT_TAIL_MAX_PAIRS, BPT_WAVE_BLOCKS, EXPORTED, KINDS, LIB_PATH,
    BptError, Options, bpt_layer_backward, bpt_layer_backward_keep_o, bpt_layer_backward_opt,
    bpt_layer_backward_workspace_size, bpt_layer_backward_workspace_size_opt,
    bpt_layer_forward, bpt_layer_forward_bsfa, bpt_layer_forward_bsfa_opt, bpt_layer_forward_opt,
    bpt_layer_forward_static, bpt_layer_forward_train, bpt_layer_forward_train_keep_o,
    bpt_layer_launch_count,
    bpt_layer_launch_count_opt, bpt_layer_shard_forward, bpt_layer_shard_project,
    bpt_layer_shard_workspace_size, bpt_layer_tail_plan, bpt_layer_workspace_size,
    bpt_layer_workspace_size_opt,
    bpt_profile_enable, bpt_profile_read, bpt_read_device_error, bpt_status_string, load,
    make_options, status_string,
)
from .layer import (  # noqa: F401
    GRAD_SHAPES, PARAM_NAMES, layer_backward, layer_forward, layer_forward_bsfa,
    layer_forward_train, to_device, workspace_for,
)
