"""Gradients of every form of the operator (la_backward): block-causal, the write gate beta and
RMSNorm of SANA-Video 2.0, Eq. (1), and the CUDA-core path (fp32, d = 32 / 64), against the fp64
oracle's chain rule (itself pinned to central differences of the forward oracle)."""
import numpy as np
import pytest
import torch

import gated_linear_attention_relu_b200 as la
import oracle as orc
from gated_linear_attention_relu_b200 import workloads as wl
from la_test_util import rel_err, to64, tol_for

pytestmark = pytest.mark.gpu

NAMES = ("dQ", "dK", "dV", "dG", "dbeta", "dgamma")

CASES = [
    # tensor-core kernels (bf16, d = 128, no gates): block-causal units inside and across CTAs
    (wl.custom("bwg_bc", B=1, H=2, T=7, Hh=6, W=10, block_frames=2), False, False),
    (wl.custom("bwg_bc_ragged", B=2, H=3, T=5, Hh=5, W=37, block_frames=2), False, False),
    (wl.custom("bwg_bc_sparse", B=1, H=2, T=5, Hh=4, W=33, block_frames=1, k_shift=-0.5, qkv_scale=1.0), False,
     False),
    (wl.custom("bwg_bc_long", B=1, H=3, T=12, Hh=9, W=40, block_frames=3), False, False),
    # the gated forms (tensor cores), fp32 and small head dimensions (CUDA cores)
    (wl.custom("bwg_beta", B=1, H=2, T=3, Hh=5, W=37), True, False),
    (wl.custom("bwg_rms", B=1, H=2, T=3, Hh=5, W=37), False, True),
    (wl.custom("bwg_bc_gated", B=1, H=2, T=5, Hh=6, W=10, block_frames=2), True, True),
    (wl.custom("bwg_f32_d64", B=1, H=2, T=3, Hh=4, W=11, d=64, bands=(16, 24, 24), dtype="f32"), False, False),
    (wl.custom("bwg_f32_d32_bc", B=2, H=2, T=4, Hh=3, W=5, d=32, bands=(8, 12, 12), dtype="f32", block_frames=1),
     True, True),
    (wl.custom("bwg_bf16_d64", B=1, H=2, T=2, Hh=5, W=20, d=64, bands=(16, 24, 24)), False, False),
]


def _run(w, use_beta, use_rms, simt=False):
    Q, K, V, G = wl.generate(w, "cuda")
    dO = wl.generate_grad(w, "cuda")
    beta, gamma = wl.generate_gates(w, "cuda")
    p = la.Problem.from_workload(w, force_simt=simt)
    b = beta if use_beta else None
    gm = gamma if use_rms else None
    out = la.backward(p, Q, K, V, G, dO, beta=b, gamma=gm, rms_norm=use_rms, norm_eps=1e-6)
    torch.cuda.synchronize()
    assert la.device_error() == 0
    return (Q, K, V, G, dO, b, gm), out


def _check(w, inputs, out, use_beta, use_rms, heads=None):
    Q, K, V, G, dO, beta, gamma = inputs
    rms = (to64(gamma), 1e-6) if use_rms else None
    tol = tol_for(w.dtype)
    refs = orc.backward_gated(to64(Q), to64(K), to64(V), to64(G), to64(dO), (w.T, w.Hh, w.W), w.bands,
                              w.rope_base, w.eps, block_frames=w.block_frames,
                              beta=to64(beta) if use_beta else None, rms=rms)
    for flat in (range(w.B * w.H) if heads is None else heads):
        b, h = divmod(flat, w.H)
        for i in range(4):
            e = rel_err(to64(out[i][b, h]), refs[i][b, h])
            assert e <= tol, (w.name, flat, NAMES[i], e)
        if use_beta:
            e = rel_err(to64(out[4][b, h]), refs[4][b, h])
            assert e <= tol, (w.name, flat, "dbeta", e)
    if use_rms:
        e = rel_err(to64(out[5]), refs[5])
        assert e <= tol, (w.name, "dgamma", e)
    else:
        assert out[5] is None


@pytest.mark.parametrize("w,use_beta,use_rms", CASES, ids=[c[0].name for c in CASES])
def test_backward_forms_all_elements(w, use_beta, use_rms):
    inputs, out = _run(w, use_beta, use_rms)
    _check(w, inputs, out, use_beta, use_rms)


@pytest.mark.parametrize("w,use_beta,use_rms", [(CASES[1][0], False, False), (CASES[3][0], False, False),
                                                 (CASES[6][0], True, True)], ids=["bc_ragged", "bc_long", "bc_gated"])
def test_backward_cuda_core_path(w, use_beta, use_rms):
    inputs, out = _run(w, use_beta, use_rms, simt=True)
    _check(w, inputs, out, use_beta, use_rms)


def test_backward_gated_forms_agree_across_paths():
    # The tensor-core and CUDA-core kernels give the same gated gradients within the tolerance.
    w = wl.custom("bwg_paths", B=2, H=3, T=5, Hh=5, W=37, block_frames=2)
    _, a = _run(w, True, True)
    _, b = _run(w, True, True, simt=True)
    for i, (x, y) in enumerate(zip(a, b)):
        scale = y.float().abs().max().item()
        assert (x.float() - y.float()).abs().max().item() <= 2e-2 * scale, NAMES[i]


def test_backward_bidirectional_forms_agree():
    # la_backward without gates on a bidirectional problem is la_backward_bidir, bit for bit.
    w = wl.custom("bwg_same", B=1, H=2, T=3, Hh=5, W=37)
    Q, K, V, G = wl.generate(w, "cuda")
    dO = wl.generate_grad(w, "cuda")
    p = la.Problem.from_workload(w)
    a = [t.clone() for t in la.backward_bidir(p, Q, K, V, G, dO)]
    b = la.backward(p, Q, K, V, G, dO)
    torch.cuda.synchronize()
    for x, y in zip(a, b[:4]):
        assert torch.equal(x, y)
    assert b[4] is None and b[5] is None


def test_backward_blockcausal_workload_sampled_heads():
    # The block-causal workload (27 blocks of 10,800 tokens, 69%-sparse ReLU(K)) on the tensor cores.
    w = wl.WORKLOADS["blockcausal"]
    inputs, out = _run(w, False, False)
    Q, K, V, G, dO, _, _ = inputs
    pos = orc.grid_positions(w.T, w.Hh, w.W)
    rng = np.random.default_rng(9)
    rows = np.unique(np.concatenate([rng.choice(w.N, 3000, replace=False), np.arange(130),
                                     np.arange(w.N - 130, w.N)]))
    idx = torch.as_tensor(rows, device="cuda")
    for flat in (0, w.H - 1):
        refs = orc.head_backward_gated(to64(Q[0, flat]), to64(K[0, flat]), to64(V[0, flat]), to64(G[0, flat]),
                                       to64(dO[0, flat]), pos, w.bands, w.rope_base, w.eps,
                                       block_frames=w.block_frames)
        for i in range(4):
            e = rel_err(to64(out[i][0, flat][idx]), refs[i][rows])
            print(f"backward blockcausal head {flat} {NAMES[i]}: {e:.2e}")
            assert e <= tol_for(w.dtype), (flat, NAMES[i], e)


def test_backward_gated_720p_5s_sampled_heads():
    # The full gated form at 720p/5s, two heads checked.
    w = wl.WORKLOADS["720p_5s"]
    inputs, out = _run(w, True, True)
    Q, K, V, G, dO, beta, gamma = inputs
    pos = orc.grid_positions(w.T, w.Hh, w.W)
    for flat in (0, w.H - 1):
        refs = orc.head_backward_gated(to64(Q[0, flat]), to64(K[0, flat]), to64(V[0, flat]), to64(G[0, flat]),
                                       to64(dO[0, flat]), pos, w.bands, w.rope_base, w.eps,
                                       beta=to64(beta[0, flat]), rms=(to64(gamma), 1e-6))
        for i in range(5):
            e = rel_err(to64(out[i][0, flat]), refs[i])
            print(f"gated backward 720p_5s head {flat} {NAMES[i]}: {e:.2e}")
            assert e <= tol_for(w.dtype), (flat, NAMES[i], e)


SAVED = [CASES[0], CASES[1], CASES[4], CASES[5], CASES[6]]


@pytest.mark.parametrize("w,use_beta,use_rms", SAVED, ids=[c[0].name for c in SAVED])
def test_backward_from_saved_states_equals_recompute(w, use_beta, use_rms):
    # la_backward_saved with the states la_forward_gated returned gives la_backward's gradients bit
    # for bit on the tensor cores (the same operand image, built from the same fp32 sums).
    (Q, K, V, G, dO, beta, gamma), ref = _run(w, use_beta, use_rms)
    p = la.Problem.from_workload(w)
    _, S, z = la.forward_gated(p, Q, K, V, G, beta=beta, gamma=gamma, rms_norm=use_rms, norm_eps=1e-6,
                               return_states=True)
    out = la.backward(p, Q, K, V, G, dO, beta=beta, gamma=gamma, rms_norm=use_rms, norm_eps=1e-6, S=S, z=z)
    torch.cuda.synchronize()
    assert la.device_error() == 0
    for i, (x, y) in enumerate(zip(out, ref)):
        assert (x is None) == (y is None), NAMES[i]
        if x is not None:
            assert torch.equal(x, y), NAMES[i]


def test_forward_states_bidirectional_match_oracle():
    # la_forward_gated returns each head's state in bidirectional mode too (beta included, z not).
    w = wl.custom("fwd_states", B=1, H=2, T=3, Hh=5, W=37)
    Q, K, V, G = wl.generate(w, "cuda")
    beta, _ = wl.generate_gates(w, "cuda")
    p = la.Problem.from_workload(w)
    _, S, z = la.forward_gated(p, Q, K, V, G, beta=beta, return_states=True)
    torch.cuda.synchronize()
    pos = orc.grid_positions(w.T, w.Hh, w.W)
    for flat in range(w.B * w.H):
        b, h = divmod(flat, w.H)
        Sr, zr = orc.head_state(to64(K[b, h]), to64(V[b, h]), pos, w.bands, w.rope_base, beta=to64(beta[b, h]))
        assert rel_err(to64(S[b, h, 0]), Sr) <= tol_for(w.dtype)
        assert rel_err(to64(z[b, h, 0]), zr) <= tol_for(w.dtype)


@pytest.mark.parametrize("w,use_beta,use_rms", [CASES[7], CASES[8]], ids=[CASES[7][0].name, CASES[8][0].name])
def test_backward_from_saved_states_cuda_core_path(w, use_beta, use_rms):
    # fp32 and small head dimensions: the saved-state gradients match the oracle.
    Q, K, V, G = wl.generate(w, "cuda")
    dO = wl.generate_grad(w, "cuda")
    beta, gamma = wl.generate_gates(w, "cuda")
    b = beta if use_beta else None
    gm = gamma if use_rms else None
    p = la.Problem.from_workload(w)
    _, S, z = la.forward_gated(p, Q, K, V, G, beta=b, gamma=gm, rms_norm=use_rms, norm_eps=1e-6,
                               return_states=True)
    out = la.backward(p, Q, K, V, G, dO, beta=b, gamma=gm, rms_norm=use_rms, norm_eps=1e-6, S=S, z=z)
    torch.cuda.synchronize()
    assert la.device_error() == 0
    _check(w, (Q, K, V, G, dO, b, gm), out, use_beta, use_rms)


def test_backward_from_saved_states_blockcausal_workload_equals_recompute():
    # The block-causal workload with the inclusive states of its forward pass.
    w = wl.WORKLOADS["blockcausal"]
    Q, K, V, G = wl.generate(w, "cuda")
    dO = wl.generate_grad(w, "cuda")
    p = la.Problem.from_workload(w)
    _, S, z = la.forward_gated(p, Q, K, V, G, return_states=True)
    out = la.backward(p, Q, K, V, G, dO, S=S, z=z)
    ref = la.backward(p, Q, K, V, G, dO)
    torch.cuda.synchronize()
    assert la.device_error() == 0
    for i in range(4):
        assert torch.equal(out[i], ref[i]), NAMES[i]
