"""BitNet b1.58 BitLinear forward (W1.58A8) for NVIDIA B200 (sm_100a)."""
