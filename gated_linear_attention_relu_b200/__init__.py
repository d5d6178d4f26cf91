"""Gated ReLU linear attention with RoPE after ReLU and a sigmoid output gate, for B200.

Per (batch, head): S = sum_n RoPE3D(ReLU(K_n))^T V_n, z = sum_n ReLU(K_n),
O_n = (RoPE3D(ReLU(Q_n)) S) / (ReLU(Q_n) . z + eps) * sigmoid(G_n); bidirectional or
block-causal over blocks of latent frames.  The compute runs in ``liblinattn.so`` (CUDA,
sm_100a); this package only marshals arguments.
"""
from . import workloads  # noqa: F401
from .binding import (  # noqa: F401
    LaError, Problem, apply, backward, backward_bidir, block_step, device_error, forward, forward_bidir, forward_blockcausal, forward_gated,
    forward_marked, forward_tokencausal,
    last_launch_count, load, state_reduce, state_scan, state_update, status_string, workspace,
    workspace_bytes,
)
