"""Local MoE expert forward on the non-expand routed layout, for NVIDIA B200 (sm_100a)."""
