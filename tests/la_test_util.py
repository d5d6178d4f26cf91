"""Helpers shared by the GPU tests: run the oracle on selected heads of GPU-generated inputs."""
from __future__ import annotations

import numpy as np

import oracle as orc

# Tolerances on max |O - O_ref| / max |O_ref| over the compared elements.
TOL_BF16 = 2e-2
TOL_F32 = 1e-5


def tol_for(dtype: str) -> float:
    return TOL_BF16 if dtype == "bf16" else TOL_F32


def to64(t) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    scale = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / (scale if scale > 0 else 1.0)


def oracle_head(w, q, k, v, g, tokens=None, beta=None, rms=None):
    """Oracle output rows (all, or the listed token indices) and the per-block inclusive states
    of one head.  q, k, v, g: (N, d) float64 arrays of that head; ``beta`` (N,) and ``rms``
    (gamma, norm_eps) are the optional terms of the full gated form."""
    pos = orc.grid_positions(w.T, w.Hh, w.W)
    if w.block_frames <= 0:
        S, z = orc.head_state(k, v, pos, w.bands, w.rope_base, beta)
        Sinc, zinc = S[None], z[None]
        blk = np.zeros(w.N, dtype=np.int64)
    else:
        Sb, zb = orc.block_states(k, v, pos, w.bands, w.rope_base, w.block_frames, beta)
        Sinc, zinc = np.cumsum(Sb, axis=0), np.cumsum(zb, axis=0)
        blk = orc.block_of_tokens(pos, w.block_frames)
    idx = np.arange(w.N) if tokens is None else np.asarray(tokens)
    out = np.empty((len(idx), w.d))
    for b in np.unique(blk[idx]):
        sel = blk[idx] == b
        rows = idx[sel]
        out[sel] = orc.head_apply(q[rows], g[rows], Sinc[b], zinc[b], pos[rows], w.bands, w.rope_base, w.eps,
                                  rms)
    return out, Sinc, zinc


def sample_tokens(w, count: int, seed: int = 0) -> np.ndarray:
    """Sampled token indices: random ones plus the first/last tokens of every 128-token tile edge
    region near block ends, so ragged tails are always compared."""
    rng = np.random.default_rng(seed)
    n = w.N
    pick = set(rng.choice(n, size=min(count, n), replace=False).tolist())
    pick.update(range(min(n, 130)))
    pick.update(range(max(0, n - 130), n))
    if w.block_frames > 0:
        L = w.block_frames * w.Hh * w.W
        for b in range(1, w.nblk):
            pick.update(range(max(0, b * L - 3), min(n, b * L + 3)))
    return np.array(sorted(pick), dtype=np.int64)
