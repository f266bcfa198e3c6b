"""SageAttention-style quantized attention forward for B200 (sm_100a)."""
