"""MoE expert-MLP + Split-LoRA layer for NVIDIA B200 (sm_100a)."""
