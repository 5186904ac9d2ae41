"""Routed-expert MoE MLP forward pass on B200 (sm_100a).

The product is libmoe.so (C ABI in include/moe.h); ``_capi`` is its thin Python binding
(argument marshalling only; tensors are torch CUDA tensors the caller allocates), ``build``
compiles the library for sm_100a, and ``inputs`` holds the seeded synthetic workload
generators.
"""
from ._capi import (MOE_DTYPE_BF16, MOE_DTYPE_FP8_MXFP4, MOE_SCORE_SIGMOID, MOE_SCORE_SOFTMAX,  # noqa: F401
                    MoeError, MoeShape, load, moe_combine, moe_debug_inject_stall,
                    moe_debug_set_wait_limit_ns, moe_forward, moe_get_device_status,
                    moe_grouped_gemm1_swiglu, moe_grouped_gemm2, moe_last_launch_count,
                    moe_permute, moe_quantize_weights_mxfp4, moe_quantize_x, moe_route,
                    moe_status_string, moe_workspace_init, moe_workspace_region,
                    moe_workspace_size)
