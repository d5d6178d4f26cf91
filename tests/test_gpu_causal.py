"""Token-causal operator (la_forward_tokencausal) against the fp64 oracle.

Token n reads the states of tokens 0..n of its head.  The kernel walks contiguous tile ranges
per CTA and carries the state across them, so the cases include heads split over many CTAs
(carried start states), CTAs that span several heads, ragged last tiles and N < one tile.
"""
import numpy as np
import pytest
import torch

import gated_linear_attention_relu_b200 as la
import oracle as orc
from gated_linear_attention_relu_b200 import workloads as wl
from la_test_util import rel_err, sample_tokens, to64, tol_for

pytestmark = pytest.mark.gpu

CASES = [
    wl.custom("tc_ragged", B=1, H=3, T=3, Hh=5, W=37),                  # N = 555: 4 full tiles + 43
    wl.custom("tc_many_heads", B=3, H=70, T=1, Hh=2, W=64),             # CTAs span several heads
    wl.custom("tc_split_heads", B=1, H=2, T=20, Hh=20, W=40),           # 125 tiles per head over ~74 CTAs
    wl.custom("tc_one_partial", B=1, H=2, T=1, Hh=1, W=50),
    wl.custom("tc_single", B=1, H=2, T=1, Hh=1, W=1),
    wl.custom("tc_sparse", B=1, H=2, T=4, Hh=7, W=23, k_shift=-0.5, qkv_scale=1.0),
    wl.custom("tc_bands", B=1, H=2, T=3, Hh=6, W=20, bands=(0, 64, 64)),
    # 74 tiles per head (ragged), 3 per CTA: four CTAs carry one head's start state into its
    # ragged last tile and then begin the next head with z and S from zero
    wl.custom("tc_cross", B=1, H=6, T=14, Hh=11, W=61),
]


def _oracle(w, Q, K, V, G, b, h, rows=None):
    pos = orc.grid_positions(w.T, w.Hh, w.W)
    return orc.tokencausal_rows(to64(Q[b, h]), to64(K[b, h]), to64(V[b, h]), to64(G[b, h]), pos, w.bands,
                                w.rope_base, w.eps, rows=rows)


SIMT_CASES = [
    # CUDA-core kernels: fp32 (the tiny fp32 config's tolerance), small head dimensions, and the
    # bf16 d = 128 problem forced onto them; heads split over many CTAs and ragged tiles
    wl.WORKLOADS["tiny_f32"],
    wl.custom("tcs_f32_d64", B=1, H=2, T=3, Hh=5, W=37, d=64, bands=(16, 24, 24), dtype="f32"),
    wl.custom("tcs_f32_split", B=2, H=2, T=8, Hh=10, W=40, d=32, bands=(8, 12, 12), dtype="f32"),
    wl.custom("tcs_bf16_d32", B=1, H=3, T=3, Hh=5, W=37, d=32, bands=(8, 12, 12)),
    wl.custom("tcs_forced", B=1, H=2, T=3, Hh=5, W=37),
]


@pytest.mark.parametrize("w", CASES + SIMT_CASES, ids=lambda w: w.name)
def test_tokencausal_all_elements(w):
    Q, K, V, G = wl.generate(w, "cuda")
    p = la.Problem.from_workload(w, force_simt=w.name == "tcs_forced")
    O = la.forward_tokencausal(p, Q, K, V, G)
    torch.cuda.synchronize()
    assert la.device_error() == 0
    heads = range(w.B * w.H) if w.B * w.H <= 8 else [0, 1, 69, 70, 139, w.B * w.H - 1]
    for flat in heads:
        b, h = divmod(flat, w.H)
        ref = _oracle(w, Q, K, V, G, b, h)
        e = rel_err(to64(O[b, h]), ref)
        assert e <= tol_for(w.dtype), (w.name, flat, e)


@pytest.mark.parametrize("name,heads", [("720p_5s", (0, 31)), ("720p_5s_b2", (0, 63)), ("720p_60s", (0, 31))])
def test_tokencausal_full_size_sampled(name, heads):
    w = wl.WORKLOADS[name]
    Q, K, V, G = wl.generate(w, "cuda")
    p = la.Problem.from_workload(w)
    O = la.forward_tokencausal(p, Q, K, V, G)
    torch.cuda.synchronize()
    assert la.device_error() == 0
    assert torch.isfinite(O).all()
    for flat in heads:
        b, h = divmod(flat, w.H)
        toks = sample_tokens(w, 2000, seed=flat)
        ref = _oracle(w, Q, K, V, G, b, h, rows=toks)
        got = to64(O[b, h][torch.as_tensor(toks, device=O.device)])
        e = rel_err(got, ref)
        print(f"token-causal {name} head {flat}: O {e:.2e}")
        assert e <= tol_for(w.dtype)
    del Q, K, V, G, O
    torch.cuda.empty_cache()


def test_tokencausal_deterministic_and_last_token_bidirectional():
    w = CASES[2]
    Q, K, V, G = wl.generate(w, "cuda")
    p = la.Problem.from_workload(w)
    ws, _ = la.workspace(p)
    O1 = la.forward_tokencausal(p, Q, K, V, G, ws=ws).clone()
    O2 = la.forward_tokencausal(p, Q, K, V, G, ws=ws)
    assert la.last_launch_count() == 4
    Ob = la.forward_bidir(p, Q, K, V, G)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2)
    # the last token of every head sees the whole head
    scale = Ob[:, :, -1].float().abs().max().item()
    assert (O1[:, :, -1].float() - Ob[:, :, -1].float()).abs().max().item() <= 2e-2 * scale
