"""Seeded synthetic workloads for the gated ReLU linear-attention token mixer.

This module only describes problem shapes and draws seeded random inputs.  It
holds none of the method's arithmetic, so the CUDA path and the fp64 oracle can
both be fed from it without sharing any computation.

Shapes follow the latent grids of the video DiT described in "SANA-Video 2.0:
Hybrid Linear Attention with Attention Residuals for Efficient Video
Generation" (Sec. 2, Eq. 1; Appendix B: head dimension 128) and the block-causal
cache of "SANA-Video: Efficient Video Generation with Block Linear Diffusion
Transformer" (Sec. 3.4).  A 720p/5 s clip maps to a 21 x 45 x 80 latent grid,
i.e. 75,600 tokens (the ">75,000 tokens" of that page's Sec. 1.1).  No dataset
is used: every input is drawn from a seeded torch generator.

Token order inside a head is row-major over the grid, time slowest:
n = (t * Hh + h) * W + w.  Layout of every activation is [B, H, N, d].
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Optional, Sequence, Tuple


@dataclass(frozen=True)
class Workload:
    """One synthetic problem: grid, heads, RoPE bands, dtype and value recipe."""

    name: str
    B: int
    H: int
    T: int
    Hh: int
    W: int
    d: int
    bands: Tuple[int, int, int]  # channels rotated by t, h, w (in that order)
    dtype: str  # "bf16" or "f32": dtype of Q, K, V, G and O
    seed: int
    qkv_scale: float = 1.0  # Q, K, V ~ N(0, 1) * qkv_scale
    k_shift: float = 0.0  # added to K after scaling
    block_frames: int = 0  # 0: bidirectional; >0: latent frames per causal block
    rope_base: float = 10000.0
    eps: float = 1e-6

    @property
    def N(self) -> int:
        return self.T * self.Hh * self.W

    @property
    def nblk(self) -> int:
        if self.block_frames <= 0:
            return 1
        return -(-self.T // self.block_frames)

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    @property
    def token_heads(self) -> int:
        return self.B * self.H * self.N

    @property
    def min_bytes(self) -> int:
        """Read Q, K, V, G once and write O once."""
        return 5 * self.B * self.H * self.N * self.d * self.elem_bytes

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


_INV_SQRT_128 = 1.0 / math.sqrt(128.0)

WORKLOADS = {
    # Tiny fp32 case that the oracle (and its O(N^2) brute form) finish instantly.
    "tiny_f32": Workload("tiny_f32", B=1, H=2, T=2, Hh=4, W=4, d=32, bands=(8, 12, 12),
                         dtype="f32", seed=0),
    # 480p-shaped, 81 frames: 21 x 30 x 52 latent grid.
    "480p": Workload("480p", B=1, H=24, T=21, Hh=30, W=52, d=128, bands=(32, 48, 48),
                     dtype="bf16", seed=1, qkv_scale=_INV_SQRT_128),
    # 720p/5s-shaped: 21 x 45 x 80 latent grid.
    "720p_5s": Workload("720p_5s", B=1, H=32, T=21, Hh=45, W=80, d=128, bands=(32, 48, 48),
                        dtype="bf16", seed=2, qkv_scale=_INV_SQRT_128),
    # Same with a batch of two (classifier-free-guidance pair).
    "720p_5s_b2": Workload("720p_5s_b2", B=2, H=32, T=21, Hh=45, W=80, d=128,
                           bands=(32, 48, 48), dtype="bf16", seed=2, qkv_scale=_INV_SQRT_128),
    # 720p/60s-shaped long sequence: 241 x 45 x 80 latent grid.
    "720p_60s": Workload("720p_60s", B=1, H=32, T=241, Hh=45, W=80, d=128, bands=(32, 48, 48),
                         dtype="bf16", seed=3, qkv_scale=_INV_SQRT_128),
    # Block-causal: 81 x 45 x 80 grid, 27 blocks of 3 latent frames (10,800 tokens each).
    # K is shifted by -0.5 so about 69% of ReLU(K) entries are zero.
    "blockcausal": Workload("blockcausal", B=1, H=32, T=81, Hh=45, W=80, d=128,
                            bands=(32, 48, 48), dtype="bf16", seed=4, k_shift=-0.5,
                            block_frames=3),
}

# Order in which the workloads are listed (smallest first).
ORDER = ["tiny_f32", "480p", "720p_5s", "720p_5s_b2", "720p_60s", "blockcausal"]


def _torch_dtype(name: str):
    import torch

    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def generate(w: Workload, device="cpu", seed: Optional[int] = None,
             heads: Optional[Sequence[int]] = None):
    """Draw (Q, K, V, G) for workload ``w`` on ``device``.

    Each tensor is drawn in fp32 from one generator seeded with ``w.seed`` (or
    ``seed``), in the order Q, K, V, G and one (b, h) head at a time, then
    Q, K and V are scaled by ``qkv_scale``, ``k_shift`` is added to K, and the
    result is rounded to ``w.dtype``.  G is N(0, 1) and is never scaled.
    Drawing head by head keeps the fp32 temporaries to one head.

    ``heads`` restricts the output to the listed flat head indices b*H + h
    (the draw still walks every head so the values do not depend on
    ``heads``); the result then has shape [1, len(heads), N, d].
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    dt = _torch_dtype(w.dtype)
    BH = w.B * w.H
    keep = list(range(BH)) if heads is None else list(heads)
    keep_set = {h: i for i, h in enumerate(keep)}
    out = []
    for which in range(4):  # Q, K, V, G
        if heads is None:
            t = torch.empty((w.B, w.H, w.N, w.d), dtype=dt, device=device)
            flat = t.view(BH, w.N, w.d)
        else:
            t = torch.empty((1, len(keep), w.N, w.d), dtype=dt, device=device)
            flat = t.view(len(keep), w.N, w.d)
        for bh in range(BH):
            x = torch.randn((w.N, w.d), generator=g, device=device, dtype=torch.float32)
            if bh not in keep_set:
                continue
            if which < 3:
                x = x * w.qkv_scale
            if which == 1 and w.k_shift != 0.0:
                x = x + w.k_shift
            flat[keep_set[bh]].copy_(x.to(dt))
        out.append(t)
    return tuple(out)



def generate_gates(w: Workload, device="cpu", seed: Optional[int] = None):
    """Draw the optional inputs of the full gated form for workload ``w``: the write gate beta
    [B, H, N] uniform in [0, 1) (rounded to ``w.dtype``) and an RMSNorm weight gamma [d] fp32,
    1 + 0.1 N(0, 1).  Seeded with ``w.seed + 7`` (or ``seed``), independent of ``generate``."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed((w.seed + 7) if seed is None else seed)
    beta = torch.rand((w.B, w.H, w.N), generator=g, device=device, dtype=torch.float32)
    gamma = 1.0 + 0.1 * torch.randn((w.d,), generator=g, device=device, dtype=torch.float32)
    return beta.to(_torch_dtype(w.dtype)).contiguous(), gamma.contiguous()



def generate_grad(w: Workload, device="cpu", seed: Optional[int] = None):
    """An output gradient dO [B, H, N, d] for workload ``w``: N(0, 1) rounded to ``w.dtype``, seeded
    with ``w.seed + 11`` (or ``seed``), independent of ``generate``."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed((w.seed + 11) if seed is None else seed)
    x = torch.randn((w.B, w.H, w.N, w.d), generator=g, device=device, dtype=torch.float32)
    return x.to(_torch_dtype(w.dtype)).contiguous()


def custom(name: str, B: int, H: int, T: int, Hh: int, W: int, d: int = 128,
           bands: Optional[Tuple[int, int, int]] = None, dtype: str = "bf16", seed: int = 7,
           qkv_scale: Optional[float] = None, k_shift: float = 0.0, block_frames: int = 0,
           rope_base: float = 10000.0, eps: float = 1e-6) -> Workload:
    """A workload of any shape, with the default band split d/4, 3d/8, 3d/8."""
    if bands is None:
        bands = (d // 4, 3 * d // 8, d - d // 4 - 3 * d // 8)
    if qkv_scale is None:
        qkv_scale = 1.0 / math.sqrt(d) if dtype == "bf16" else 1.0
    return Workload(name, B=B, H=H, T=T, Hh=Hh, W=W, d=d, bands=tuple(bands), dtype=dtype,
                    seed=seed, qkv_scale=qkv_scale, k_shift=k_shift,
                    block_frames=block_frames, rope_base=rope_base, eps=eps)
