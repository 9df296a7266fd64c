"""B200-native (sm_100a) NF4 grouped mixture-of-experts layer.

The compute lives in ``libmoenf4.so`` (C ABI, ``include/moe_nf4.h``); this
package is its thin Python binding.  See ``_lib`` for the calls.
"""

from ._lib import (  # noqa: F401
    LIB_PATH,
    MoEError,
    DEVERR_BAD_INDEX,
    DEVERR_BAD_OFFSETS,
    DEVERR_NONFINITE,
    DEVERR_TIMEOUT,
    DEVERR_RANGE,
    load,
    nf4_levels,
    nf4_quantize,
    nf4_dequantize,
    route_permute_workspace_size,
    route_permute,
    nf4_grouped_gemm,
    int4_quantize,
    int4_grouped_gemm,
    lora_delta,
    nf4_grouped_gemm_t,
    nf4_down_backward,
    swiglu_backward,
    combine_backward,
    route_backward,
    mxfp4_quantize,
    mxfp4_grouped_gemm,
    permute_rows,
    swiglu,
    unpermute_combine,
    layer_workspace_size,
    layer_forward,
)
