"""HyperQuant tile codec for NVIDIA B200 (sm_100a): Python binding over the C-ABI library."""
