"""Gated ReLU linear attention (RoPE after ReLU, sigmoid output gate) for B200."""
from . import workloads  # noqa: F401
