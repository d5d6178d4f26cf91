"""CUDA path against the fp64 oracle, element by element, through the C ABI.

Small grids are compared on every output element (several 128-token tiles plus ragged tails,
block ends inside tiles, CTAs whose token range spans many heads).  The full-size workloads
are run in the same configuration the benchmark times and compared on sampled heads and
sampled tokens (the oracle reduces the whole head's state in fp64).
"""
import numpy as np
import pytest
import torch

import gated_linear_attention_relu_b200 as la
from gated_linear_attention_relu_b200 import workloads as wl
from la_test_util import oracle_head, rel_err, sample_tokens, to64, tol_for

pytestmark = pytest.mark.gpu


def _problem(w, simt=False):
    return la.Problem.from_workload(w, force_simt=simt)


def _check_all_heads(w, simt=False, check_states=True):
    Q, K, V, G = wl.generate(w, "cuda")
    p = _problem(w, simt)
    if w.block_frames > 0:
        O, S, z = la.forward_blockcausal(p, Q, K, V, G, return_states=True)
    else:
        O = la.forward_bidir(p, Q, K, V, G)
        S, z = la.state_reduce(p, K, V)
    torch.cuda.synchronize()
    assert la.device_error() == 0
    tol = tol_for(w.dtype)
    worst = 0.0
    for b in range(w.B):
        for h in range(w.H):
            ref, Sref, zref = oracle_head(w, to64(Q[b, h]), to64(K[b, h]), to64(V[b, h]), to64(G[b, h]))
            e = rel_err(to64(O[b, h]), ref)
            worst = max(worst, e)
            assert e <= tol, f"{w.name} b={b} h={h}: O rel err {e:.3e} > {tol}"
            if check_states:
                es = rel_err(to64(S[b, h]), Sref)
                ez = rel_err(to64(z[b, h]), zref)
                assert es <= tol and ez <= tol, f"{w.name} b={b} h={h}: S {es:.3e} z {ez:.3e}"
    return worst


SMALL = [
    wl.custom("ragged", B=1, H=3, T=3, Hh=5, W=37),                 # N = 555: 4 full tiles + 43
    wl.custom("batch2", B=2, H=2, T=2, Hh=9, W=16),                 # N = 288
    wl.custom("one_partial_tile", B=1, H=2, T=1, Hh=1, W=50),       # N = 50 < one tile
    wl.custom("w_is_1", B=1, H=1, T=40, Hh=3, W=1),                 # position stepping wraps every token
    wl.custom("many_heads", B=3, H=70, T=1, Hh=2, W=64),            # 210 heads: CTAs span several heads
    wl.custom("single_token", B=1, H=2, T=1, Hh=1, W=1),            # N = 1
    wl.custom("sparse_k", B=1, H=2, T=4, Hh=7, W=23, k_shift=-0.5, qkv_scale=1.0),
    wl.custom("bands_0_64_64", B=1, H=2, T=3, Hh=6, W=20, bands=(0, 64, 64)),
]

SMALL_BC = [
    wl.custom("bc_ragged", B=1, H=2, T=7, Hh=6, W=10, block_frames=2),     # 120-token blocks, last 60
    wl.custom("bc_big", B=1, H=2, T=5, Hh=9, W=40, block_frames=2),        # 720-token blocks, last 360
    wl.custom("bc_one_block", B=1, H=2, T=4, Hh=5, W=30, block_frames=4),
    wl.custom("bc_bf_gt_T", B=2, H=1, T=3, Hh=5, W=30, block_frames=10),
    wl.custom("bc_bf1_sparse", B=1, H=3, T=6, Hh=4, W=33, block_frames=1, k_shift=-0.5, qkv_scale=1.0),
]


@pytest.mark.parametrize("w", SMALL + SMALL_BC, ids=lambda w: w.name)
def test_bf16_d128_tensor_core_path(w):
    _check_all_heads(w)


@pytest.mark.parametrize("w", SMALL[:3] + SMALL_BC[:2], ids=lambda w: w.name)
def test_bf16_d128_cuda_core_path(w):
    _check_all_heads(w, simt=True)


@pytest.mark.parametrize("d,bands", [(32, (8, 12, 12)), (64, (16, 24, 24))])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("bf", [0, 2])
def test_other_head_dims_and_fp32(d, bands, dtype, bf):
    w = wl.custom(f"d{d}_{dtype}_{bf}", B=2, H=2, T=5, Hh=3, W=11, d=d, bands=bands, dtype=dtype,
                  block_frames=bf)
    _check_all_heads(w)


def test_fp32_d128():
    _check_all_heads(wl.custom("f32_d128", B=1, H=2, T=3, Hh=5, W=19, dtype="f32"))


def test_tiny_f32_workload():
    w = wl.WORKLOADS["tiny_f32"]
    _check_all_heads(w)


# ------------------------------------------------------------------------- full-size workloads

def _check_sampled(w, heads, ntok=3000):
    Q, K, V, G = wl.generate(w, "cuda")
    p = _problem(w)
    ws, _ = la.workspace(p)
    if w.block_frames > 0:
        O, S, z = la.forward_blockcausal(p, Q, K, V, G, ws=ws, return_states=True)
    else:
        O = la.forward_bidir(p, Q, K, V, G, ws=ws)
        S, z = la.state_reduce(p, K, V, ws=ws)
    torch.cuda.synchronize()
    assert la.device_error() == 0
    assert torch.isfinite(O).all()
    tol = tol_for(w.dtype)
    for flat in heads:
        b, h = divmod(flat, w.H)
        toks = sample_tokens(w, ntok, seed=flat)
        ref, Sref, zref = oracle_head(w, to64(Q[b, h]), to64(K[b, h]), to64(V[b, h]), to64(G[b, h]), toks)
        got = to64(O[b, h][torch.as_tensor(toks, device=O.device)])
        e = rel_err(got, ref)
        es, ez = rel_err(to64(S[b, h]), Sref), rel_err(to64(z[b, h]), zref)
        print(f"{w.name} head {flat}: O {e:.2e}  S {es:.2e}  z {ez:.2e}")
        assert e <= tol and es <= tol and ez <= tol
    return Q, K, V, G, O


def test_480p_all_heads_sampled_tokens():
    w = wl.WORKLOADS["480p"]
    _check_sampled(w, heads=range(w.H), ntok=1500)


def test_720p_5s():
    w = wl.WORKLOADS["720p_5s"]
    _check_sampled(w, heads=[0, 17, w.H - 1])


def test_720p_5s_batch2_and_batch_independence():
    w = wl.WORKLOADS["720p_5s_b2"]
    Q, K, V, G, O = _check_sampled(w, heads=[0, w.B * w.H - 1])
    # Batch 1 of the B = 2 run against a separate B = 1 run of the same inputs.
    p1 = la.Problem.from_workload(w, B=1)
    O1 = la.forward_bidir(p1, Q[1:2].contiguous(), K[1:2].contiguous(), V[1:2].contiguous(),
                          G[1:2].contiguous())
    torch.cuda.synchronize()
    scale = O1.float().abs().max().item()
    assert (O[1:2].float() - O1.float()).abs().max().item() <= 1e-2 * scale


def test_720p_60s_long_sequence():
    w = wl.WORKLOADS["720p_60s"]
    _check_sampled(w, heads=[0, w.H - 1], ntok=4000)


def test_blockcausal_workload():
    w = wl.WORKLOADS["blockcausal"]
    _check_sampled(w, heads=[0, w.H - 1], ntok=4000)


# ------------------------------------------------------------------------- composition, determinism

def test_decomposed_calls_match_forward_bitwise():
    w = wl.custom("compose", B=1, H=4, T=6, Hh=9, W=24, block_frames=2)
    Q, K, V, G = wl.generate(w, "cuda")
    for bf in (0, 2):
        p = la.Problem.from_workload(w, block_frames=bf)
        O = la.forward(p, Q, K, V, G)
        S, z = la.state_reduce(p, K, V)
        la.state_scan(p, S, z)
        O2 = la.apply(p, Q, G, S, z)
        torch.cuda.synchronize()
        assert torch.equal(O, O2)


def test_deterministic_runs_bitwise():
    w = wl.WORKLOADS["720p_5s"]
    Q, K, V, G = wl.generate(w, "cuda")
    p = _problem(w)
    ws, _ = la.workspace(p)
    O1 = la.forward_bidir(p, Q, K, V, G, ws=ws).clone()
    S1, z1 = la.state_reduce(p, K, V, ws=ws)
    O2 = la.forward_bidir(p, Q, K, V, G, ws=ws)
    S2, z2 = la.state_reduce(p, K, V, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(O1, O2) and torch.equal(S1, S2) and torch.equal(z1, z2)


def test_launch_counts_and_device_error_word():
    w = wl.custom("launches", B=1, H=2, T=2, Hh=4, W=40)
    Q, K, V, G = wl.generate(w, "cuda")
    p = _problem(w)
    la.forward_bidir(p, Q, K, V, G)
    assert la.last_launch_count() == 4  # cos/sin table, state, combine, apply
    la.state_reduce(p, K, V)
    assert la.last_launch_count() == 3  # cos/sin table, state, combine
    la.forward_bidir(la.Problem.from_workload(w, force_simt=True), Q, K, V, G)
    assert la.last_launch_count() == 3  # state, combine, apply (CUDA cores)
    assert la.device_error() == 0


def test_empty_problems_are_no_ops():
    for kw in (dict(B=0, H=4, T=3, Hh=4, W=4), dict(B=1, H=4, T=0, Hh=4, W=4)):
        p = la.Problem(**kw)
        x = torch.empty((p.B, p.H, p.N, 128), dtype=torch.bfloat16, device="cuda")
        O = la.forward_bidir(p, x, x, x, x)
        assert O.numel() == 0
    # N = 0 in bidirectional mode: the states are zero.
    p = la.Problem(B=1, H=2, T=0, Hh=4, W=4)
    x = torch.empty((1, 2, 0, 128), dtype=torch.bfloat16, device="cuda")
    S, z = la.state_reduce(p, x, x)
    torch.cuda.synchronize()
    assert S.abs().max().item() == 0.0 and z.abs().max().item() == 0.0


def test_rejects_bad_arguments_without_launching():
    w = wl.custom("bad", B=1, H=1, T=1, Hh=2, W=8)
    Q, K, V, G = wl.generate(w, "cuda")
    p = _problem(w)
    with pytest.raises(la.LaError) as e:
        la.forward_bidir(la.Problem.from_workload(w, bands=(32, 48, 40)), Q, K, V, G)
    assert e.value.status == 3
    with pytest.raises(la.LaError) as e:
        la.forward_bidir(p, Q, K, V, G, ws=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 6
    flat = torch.empty(Q.numel() + 8, dtype=torch.bfloat16, device="cuda")
    mis = flat[1:1 + Q.numel()].view_as(Q)  # 2-byte offset: misaligned
    with pytest.raises(la.LaError) as e:
        la.forward_bidir(p, mis, K, V, G)
    assert e.value.status == 4
