"""q4gsw: 4-bit group-symmetric weight-quantized linear layer for B200 (sm_100a)."""
