"""The full gated form (write gate beta, RMSNorm before the output gate; SANA-Video 2.0, Eq. (1))
through la_forward_gated, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gated_linear_attention_relu_b200 as la
from gated_linear_attention_relu_b200 import workloads as wl
from la_test_util import oracle_head, rel_err, sample_tokens, to64, tol_for

pytestmark = pytest.mark.gpu

CASES = [
    wl.custom("g_ragged", B=1, H=3, T=3, Hh=5, W=37),
    wl.custom("g_heads", B=2, H=3, T=2, Hh=3, W=40),
    wl.custom("g_bc", B=1, H=2, T=7, Hh=6, W=10, block_frames=2),
    wl.custom("g_bc_sparse", B=1, H=2, T=5, Hh=4, W=33, block_frames=1, k_shift=-0.5, qkv_scale=1.0),
    wl.custom("g_d64_f32", B=1, H=2, T=3, Hh=4, W=11, d=64, bands=(16, 24, 24), dtype="f32"),
    wl.custom("g_tiny", B=1, H=2, T=2, Hh=4, W=4, d=32, bands=(8, 12, 12), dtype="f32", block_frames=1),
]


def _check(w, use_beta, use_rms, use_gamma=True, simt=False, tokens=None, heads=None):
    Q, K, V, G = wl.generate(w, "cuda")
    beta, gamma = wl.generate_gates(w, "cuda")
    p = la.Problem.from_workload(w, force_simt=simt)
    b = beta if use_beta else None
    gm = gamma if (use_rms and use_gamma) else None
    kw = dict(beta=b, gamma=gm, rms_norm=use_rms, norm_eps=1e-6)
    if w.block_frames > 0:
        O, S, z = la.forward_gated(p, Q, K, V, G, return_states=True, **kw)
    else:
        O = la.forward_gated(p, Q, K, V, G, **kw)
        S = z = None
    torch.cuda.synchronize()
    assert la.device_error() == 0
    tol = tol_for(w.dtype)
    rms = (to64(gm) if gm is not None else None, 1e-6) if use_rms else None
    for flat in (range(w.B * w.H) if heads is None else heads):
        bb, h = divmod(flat, w.H)
        toks = None if tokens is None else sample_tokens(w, tokens, seed=flat)
        ref, Sinc, zinc = oracle_head(w, to64(Q[bb, h]), to64(K[bb, h]), to64(V[bb, h]), to64(G[bb, h]), toks,
                                      beta=to64(beta[bb, h]) if use_beta else None, rms=rms)
        got = to64(O[bb, h]) if toks is None else to64(O[bb, h][torch.as_tensor(toks, device=O.device)])
        e = rel_err(got, ref)
        assert e <= tol, (w.name, flat, e)
        if S is not None:
            assert rel_err(to64(S[bb, h]), Sinc) <= tol and rel_err(to64(z[bb, h]), zinc) <= tol


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("use_beta,use_rms", [(True, False), (False, True), (True, True)])
def test_gated_forms_small(w, use_beta, use_rms):
    _check(w, use_beta, use_rms)


@pytest.mark.parametrize("w", CASES[:3], ids=lambda w: w.name)
def test_gated_cuda_core_path(w):
    _check(w, True, True, simt=True)


def test_rms_without_weight():
    _check(CASES[0], True, True, use_gamma=False)


def test_no_gates_is_the_plain_operator_bitwise():
    for w in (CASES[0], CASES[2]):
        Q, K, V, G = wl.generate(w, "cuda")
        p = la.Problem.from_workload(w)
        a = la.forward(p, Q, K, V, G)
        b = la.forward_gated(p, Q, K, V, G)
        torch.cuda.synchronize()
        assert torch.equal(a, b)


def test_gated_720p_5s_sampled():
    w = wl.WORKLOADS["720p_5s"]
    _check(w, True, True, tokens=2000, heads=[0, w.H - 1])


def test_gated_720p_60s_sampled():
    w = wl.WORKLOADS["720p_60s"]
    _check(w, True, True, tokens=3000, heads=[0, w.H - 1])
    torch.cuda.empty_cache()


def test_gated_blockcausal_sampled():
    w = wl.WORKLOADS["blockcausal"]
    _check(w, True, True, tokens=3000, heads=[5])
