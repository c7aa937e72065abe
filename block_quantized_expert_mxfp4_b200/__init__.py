"""B200-native routed-expert FFN with block-quantized (MXFP4 / NVFP4 / FP8
block-128) weights: a C-ABI CUDA library (libqk.so, sm_100a) and its thin
Python binding.  See include/qk.h for the ABI."""
from ._lib import (  # noqa: F401
    LIB_PATH, QK_ACT_E4M3, QK_ACT_MXFP4, QK_ACT_NONE, QK_ERR_CUDA, QK_ERR_INVALID_ARG,
    QK_ERR_NAN_SCALE, QK_ERR_NONFINITE, QK_ERR_TIMEOUT, QK_ERR_UNSUPPORTED, QK_ERR_WORKSPACE, QK_FMT_MXFP4,
    QK_FMT_NVFP4, QK_OK, QkError, fp8_block_linear, fp8_shared_expert_forward,
    fp8_shared_expert_workspace_size, load, make_layer, make_weight, moe_expert_forward,
    moe_expert_forward_noalloc,
    moe_expert_workspace_size, moe_route_topk, qk_debug_set_wait_limit_ns, qk_last_device_status,
    qk_moe_layer, qk_weight, quant_convert_mxfp4_to_nvfp4, quant_convert_nvfp4_to_mxfp4,
    status_string,
)
