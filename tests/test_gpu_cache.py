"""Block-autoregressive cache (la_state_update + la_apply with a frame offset) against the oracle.

A generator that produces one block of latent frames at a time keeps a constant-size cache
(S, z) (SANA-Video, Sec. 3.4, Algorithm 1): after each block it folds the block's keys and values
into the cache, and the block's outputs read the cache including the block itself.  Driving the
library that way, one call per block with `t0` = the block's first global frame, must reproduce
the block-causal operator on the whole video.
"""
import numpy as np
import pytest
import torch

import gated_linear_attention_relu_b200 as la
from gated_linear_attention_relu_b200 import workloads as wl
from la_test_util import oracle_head, rel_err, to64, tol_for

pytestmark = pytest.mark.gpu


def _stream_blocks(w, Q, K, V, G, simt=False):
    HW = w.Hh * w.W
    S = torch.zeros((w.B, w.H, 1, w.d, w.d), dtype=torch.float32, device=Q.device)
    z = torch.zeros((w.B, w.H, 1, w.d), dtype=torch.float32, device=Q.device)
    outs, caches = [], []
    for t0 in range(0, w.T, w.block_frames):
        t1 = min(w.T, t0 + w.block_frames)
        sl = slice(t0 * HW, t1 * HW)
        pb = la.Problem.from_workload(w, T=t1 - t0, block_frames=0, t0=t0, force_simt=simt)
        blk = [x[:, :, sl].contiguous() for x in (Q, K, V, G)]
        la.state_update(pb, blk[1], blk[2], S, z)
        outs.append(la.apply(pb, blk[0], blk[3], S, z))
        caches.append((S.clone(), z.clone()))
    torch.cuda.synchronize()
    assert la.device_error() == 0
    return torch.cat(outs, dim=2), caches


CASES = [
    wl.custom("cache_ragged", B=1, H=2, T=7, Hh=6, W=10, block_frames=2),        # last block 1 frame
    wl.custom("cache_b2", B=2, H=2, T=6, Hh=5, W=30, block_frames=3),
    wl.custom("cache_sparse", B=1, H=3, T=5, Hh=4, W=33, block_frames=1, k_shift=-0.5, qkv_scale=1.0),
    wl.custom("cache_f32_d64", B=1, H=2, T=4, Hh=3, W=11, d=64, bands=(16, 24, 24), dtype="f32",
              block_frames=2),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_streaming_cache_matches_oracle_block_causal(w):
    Q, K, V, G = wl.generate(w, "cuda")
    O, caches = _stream_blocks(w, Q, K, V, G)
    tol = tol_for(w.dtype)
    for b in range(w.B):
        for h in range(w.H):
            ref, Sinc, zinc = oracle_head(w, to64(Q[b, h]), to64(K[b, h]), to64(V[b, h]), to64(G[b, h]))
            assert rel_err(to64(O[b, h]), ref) <= tol
            for j, (S, z) in enumerate(caches):
                assert rel_err(to64(S[b, h, 0]), Sinc[j]) <= tol
                assert rel_err(to64(z[b, h, 0]), zinc[j]) <= tol


def test_streaming_cache_matches_whole_video_forward():
    w = CASES[0]
    Q, K, V, G = wl.generate(w, "cuda")
    O, caches = _stream_blocks(w, Q, K, V, G)
    p = la.Problem.from_workload(w)
    O_all, S_incl, z_incl = la.forward_blockcausal(p, Q, K, V, G, return_states=True)
    S_last, z_last = caches[-1]
    torch.cuda.synchronize()
    scale = O_all.float().abs().max().item()
    assert (O.float() - O_all.float()).abs().max().item() <= 1e-2 * scale
    assert torch.allclose(S_last[:, :, 0], S_incl[:, :, -1], rtol=1e-4, atol=1e-4)
    assert torch.allclose(z_last[:, :, 0], z_incl[:, :, -1], rtol=1e-5, atol=1e-5)


def test_streaming_cache_cuda_core_path():
    w = CASES[0]
    Q, K, V, G = wl.generate(w, "cuda")
    O, _ = _stream_blocks(w, Q, K, V, G, simt=True)
    for h in range(w.H):
        ref, _, _ = oracle_head(w, to64(Q[0, h]), to64(K[0, h]), to64(V[0, h]), to64(G[0, h]))
        assert rel_err(to64(O[0, h]), ref) <= tol_for(w.dtype)


def test_frame_offset_shifts_positions():
    """A bidirectional call on frames [t0, t0 + T) of a longer video with t0 set equals the oracle
    with global positions, and differs from the t0 = 0 call."""
    w = wl.custom("offset", B=1, H=2, T=3, Hh=5, W=16)
    Q, K, V, G = wl.generate(w, "cuda")
    p5 = la.Problem.from_workload(w, t0=5)
    O5 = la.forward_bidir(p5, Q, K, V, G)
    O0 = la.forward_bidir(la.Problem.from_workload(w), Q, K, V, G)
    torch.cuda.synchronize()
    import oracle as orc

    pos = orc.grid_positions(w.T, w.Hh, w.W)
    pos[:, 0] += 5
    for h in range(w.H):
        ref = orc.forward_positions(to64(Q[0, h]), to64(K[0, h]), to64(V[0, h]), to64(G[0, h]), pos,
                                    w.bands, w.rope_base, w.eps)
        assert rel_err(to64(O5[0, h]), ref) <= tol_for(w.dtype)
    assert not torch.equal(O5, O0)


@pytest.mark.parametrize("w", CASES[:3], ids=lambda w: w.name)
def test_block_step_matches_two_call_path(w):
    """la_block_step (one call per block) computes what la_state_update + la_apply compute."""
    Q, K, V, G = wl.generate(w, "cuda")
    O_two, caches = _stream_blocks(w, Q, K, V, G)
    HW = w.Hh * w.W
    S = torch.zeros((w.B, w.H, w.d, w.d), dtype=torch.float32, device="cuda")
    z = torch.zeros((w.B, w.H, w.d), dtype=torch.float32, device="cuda")
    outs = []
    for t0 in range(0, w.T, w.block_frames):
        t1 = min(w.T, t0 + w.block_frames)
        sl = slice(t0 * HW, t1 * HW)
        pb = la.Problem.from_workload(w, T=t1 - t0, block_frames=0, t0=t0)
        qb, kb, vb, gb = (x[:, :, sl].contiguous() for x in (Q, K, V, G))
        outs.append(la.block_step(pb, qb, kb, vb, gb, S, z))
        assert la.last_launch_count() == (4 if w.d == 128 and w.dtype == "bf16" else 3)
    O = torch.cat(outs, dim=2)
    torch.cuda.synchronize()
    assert la.device_error() == 0
    # Same kernels, same order of every sum: identical results.
    assert torch.equal(O, O_two)
    assert torch.equal(S, caches[-1][0][:, :, 0]) and torch.equal(z, caches[-1][1][:, :, 0])
