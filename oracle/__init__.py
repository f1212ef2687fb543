"""CPU oracle for the q4gsw linear layer (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
legs may import this package.  It shares no code with the CUDA library.
``q4gsw_variants`` holds the fp32-scale (packed layout version 2) and the
frozen-base adapter variants.
"""
from .q4gsw_oracle import *  # noqa: F401,F403
from .q4gsw_oracle import (  # noqa: F401
    LAYOUT_VERSION, ZERO_POINT, packed_layout, codes_byte_offset, trailer_words, pack, pack_fast, unpack_codes,
    unpack_codes_fast, unpack_scale_bits, fp16_bits_to_float, float_to_fp16_bits_rne,
    dequant_w32, dequant_w16_bits, dequant_w16_bits_fast, linear_fwd, linear_bwd_input,
    qkv_fwd, linear_fwd_rows, linear_bwd_input_rows, embedding,
)
from . import q4gsw_variants  # noqa: F401,E402
