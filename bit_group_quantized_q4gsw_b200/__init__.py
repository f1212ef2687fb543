"""q4gsw: 4-bit group-symmetric weight-quantized linear layer for B200 (sm_100a).

The public functions carry the names of the C ABI in ``include/q4gsw.h`` and
take torch tensors; all arithmetic runs in the CUDA library ``libq4gsw.so``.
"""
from .binding import (  # noqa: F401
    Q4gswError, library, q4gsw_dq8ca_quantize, q4gsw_linear_dq8ca_fwd, q4gsw_adapter_bwd_input, q4gsw_adapter_fwd, q4gsw_debug_pin_routes, q4gsw_debug_wait_timeout, q4gsw_dequant, q4gsw_device_error_check, q4gsw_embedding, q4gsw_last_route,
    q4gsw_layout_version, q4gsw_linear_bwd_input,
    q4gsw_linear_fwd, q4gsw_packed_bytes, q4gsw_prepack, q4gsw_prepack_f32s, q4gsw_qkv_fwd, q4gsw_status_str, q4gsw_unpack,
)
