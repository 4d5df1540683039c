"""B200-native (sm_100a) routed mixture-of-experts FFN layer over MXFP4 experts.

The computation lives in libmoe_b200.so (C ABI in include/moe.h, CUDA kernels
in csrc/); ``moe`` is its ctypes binding, ``synth`` draws seeded inputs.
"""
from . import moe  # noqa: F401
from .moe import (  # noqa: F401
    EXPORTS, Experts, MoeError, load_library, make_workspace, moe_act_quant_mxfp4,
    moe_bucket, moe_combine, moe_decode_mxfp4, moe_expert_ffn_mxfp4, moe_get_error,
    moe_get_error_static, moe_layer_forward, moe_layer_forward_static, moe_route_topk,
    moe_version, moe_workspace_bytes, moe_workspace_init, moe_workspace_set_limits, shape_of,
)
