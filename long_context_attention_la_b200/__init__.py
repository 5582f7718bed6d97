"""Lightning Attention layer kernel for NVIDIA B200 (sm_100a): Python binding of the C ABI."""
