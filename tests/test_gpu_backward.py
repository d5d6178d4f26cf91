"""Gradients of the bidirectional operator (la_backward_bidir) against the fp64 oracle's chain
rule (itself pinned to finite differences of the forward oracle)."""
import numpy as np
import pytest
import torch

import gated_linear_attention_relu_b200 as la
import oracle as orc
from gated_linear_attention_relu_b200 import workloads as wl
from la_test_util import rel_err, to64, tol_for

pytestmark = pytest.mark.gpu

CASES = [
    wl.custom("bw_ragged", B=1, H=2, T=3, Hh=5, W=37),               # N = 555, ragged last tile
    wl.custom("bw_heads", B=2, H=3, T=2, Hh=3, W=40),                # CTAs span several heads
    wl.custom("bw_split", B=1, H=2, T=8, Hh=10, W=40),               # 25 tiles per head over many CTAs
    wl.custom("bw_sparse", B=1, H=2, T=4, Hh=7, W=23, k_shift=-0.5, qkv_scale=1.0),
    wl.custom("bw_bands", B=1, H=2, T=3, Hh=6, W=20, bands=(0, 64, 64)),
    wl.custom("bw_many_heads", B=1, H=160, T=1, Hh=2, W=64),        # one-tile heads, 12 CTAs hold two
    # 74 tiles per head (ragged), 3 per CTA: four CTAs end one head and start the next, so the
    # state image and z (two slots by unit parity) change inside a CTA
    wl.custom("bw_cross", B=1, H=6, T=14, Hh=11, W=61),
]
NAMES = ("dQ", "dK", "dV", "dG")


def _run(w):
    Q, K, V, G = wl.generate(w, "cuda")
    dO = wl.generate_grad(w, "cuda")
    p = la.Problem.from_workload(w)
    grads = la.backward_bidir(p, Q, K, V, G, dO)
    torch.cuda.synchronize()
    assert la.device_error() == 0
    return (Q, K, V, G, dO), grads


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_all_elements(w):
    (Q, K, V, G, dO), grads = _run(w)
    pos = orc.grid_positions(w.T, w.Hh, w.W)
    for flat in range(w.B * w.H):
        b, h = divmod(flat, w.H)
        refs = orc.head_backward(to64(Q[b, h]), to64(K[b, h]), to64(V[b, h]), to64(G[b, h]), to64(dO[b, h]), pos,
                                 w.bands, w.rope_base, w.eps)
        for name, got, ref in zip(NAMES, grads, refs):
            e = rel_err(to64(got[b, h]), ref)
            assert e <= tol_for(w.dtype), (w.name, flat, name, e)


@pytest.mark.parametrize("wname,heads", [("720p_5s", (0, 31)), ("720p_5s_b2", (0, 63))])
def test_backward_full_size_sampled_rows(wname, heads):
    w = wl.WORKLOADS[wname]
    (Q, K, V, G, dO), grads = _run(w)
    pos = orc.grid_positions(w.T, w.Hh, w.W)
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([rng.choice(w.N, 3000, replace=False), np.arange(130), np.arange(w.N - 130, w.N)]))
    for flat in heads:
        b, h = divmod(flat, w.H)
        refs = orc.head_backward(to64(Q[b, h]), to64(K[b, h]), to64(V[b, h]), to64(G[b, h]), to64(dO[b, h]), pos,
                                 w.bands, w.rope_base, w.eps)
        idx = torch.as_tensor(rows, device="cuda")
        for name, got, ref in zip(NAMES, grads, refs):
            e = rel_err(to64(got[b, h][idx]), ref[rows])
            print(f"backward {wname} head {flat} {name}: {e:.2e}")
            assert e <= tol_for(w.dtype), (flat, name, e)


def test_backward_deterministic():
    w = CASES[2]
    Q, K, V, G = wl.generate(w, "cuda")
    dO = wl.generate_grad(w, "cuda")
    p = la.Problem.from_workload(w)
    ws, _ = la.workspace(p)
    a = [t.clone() for t in la.backward_bidir(p, Q, K, V, G, dO, ws=ws)]
    b = la.backward_bidir(p, Q, K, V, G, dO, ws=ws)
    torch.cuda.synchronize()
    assert la.last_launch_count() == 6
    for x, y in zip(a, b):
        assert torch.equal(x, y)
