"""FP6 (e3m2) x FP16 weight-only linear layer for NVIDIA B200 (sm_100a)."""
