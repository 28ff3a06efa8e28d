"""fp64 CPU oracle for the MoE + Split-LoRA layer.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check in
__graft_entry__.py and by the CPU-baseline leg of bench.py, never by the CUDA
library or its Python binding.
"""
from .moe_lora_oracle import *  # noqa: F401,F403
from .moe_lora_oracle import __all__  # noqa: F401
