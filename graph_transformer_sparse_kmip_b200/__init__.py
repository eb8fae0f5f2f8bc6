"""k-MIP attention for graph transformers on NVIDIA B200 (sm_100a)."""
