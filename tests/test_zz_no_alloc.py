"""The allocation-free entry point (la_forward_bidir_static) against the regular one.

Some callers cannot allocate device memory while they run (a plugin inside a framework that owns
every allocation, or a service that fixes its memory at start-up), so they cannot provide the
workspace la_forward_bidir needs.  la_forward_bidir_static uses the library's fixed device
scratch instead.  This test calls it through the C ABI twice in a row, on two different problems
(so the second call runs on scratch the first one left behind), and checks each output against
la_forward_bidir bit for bit (both run the same kernels on the same work split, with every
reduction in a fixed order, so any difference means stale scratch was read), and the second one
against the fp64 oracle as well, with the tolerance the parity tests use.  It lives in a file of
its own that pytest collects last.
"""
import ctypes

import pytest
import torch

import gated_linear_attention_relu_b200 as la
from gated_linear_attention_relu_b200 import workloads as wl
import oracle as orc
from la_test_util import TOL_BF16, rel_err, to64

pytestmark = pytest.mark.gpu


def _static_call(p, Q, K, V, G, O):
    lib = la.load()
    cp = p.c()
    return lib.la_forward_bidir_static(ctypes.byref(cp), Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                       G.data_ptr(), O.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_static_scratch_forward_matches_workspace_forward_twice():
    cases = [wl.custom("static_a", B=1, H=4, T=5, Hh=9, W=40),        # 1,800 tokens per head
             wl.custom("static_b", B=2, H=3, T=3, Hh=7, W=37)]        # ragged last tile
    for w in cases:
        Q, K, V, G = wl.generate(w, "cuda")
        p = la.Problem.from_workload(w)
        ref = la.forward_bidir(p, Q, K, V, G)
        O = torch.full_like(Q, float("nan"))
        assert _static_call(p, Q, K, V, G, O) == 0
        torch.cuda.synchronize()
        assert la.device_error() == 0
        assert torch.equal(O, ref), (w.name, (O.float() - ref.float()).abs().max().item())
    # the second problem against the oracle too
    o_ref = orc.forward_bidir(to64(Q), to64(K), to64(V), to64(G), (w.T, w.Hh, w.W), w.bands, w.rope_base, w.eps)
    err = rel_err(to64(O), o_ref)
    assert err <= TOL_BF16, (w.name, err)


def test_static_scratch_takes_the_720p_5s_problem():
    # B = 1, H = 32 on the 720p/5s latent grid fits the fixed scratch on a B200 (148 SMs).
    w = wl.WORKLOADS["720p_5s"]
    Q, K, V, G = wl.generate(w, "cuda")
    p = la.Problem.from_workload(w)
    ref = la.forward_bidir(p, Q, K, V, G)
    O = torch.empty_like(Q)
    assert _static_call(p, Q, K, V, G, O) == 0
    torch.cuda.synchronize()
    assert la.device_error() == 0
    assert torch.equal(O, ref)


def test_static_scratch_rejects_problems_that_do_not_fit():
    p = la.Problem(B=8, H=64, T=241, Hh=45, W=80)
    assert la.workspace_bytes(p) > (32 << 20)
    x = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    lib = la.load()
    cp = p.c()
    s = torch.cuda.current_stream().cuda_stream
    ptr = x.data_ptr()
    assert lib.la_forward_bidir_static(ctypes.byref(cp), ptr, ptr, ptr, ptr, ptr, s) == 6  # LA_ERR_WORKSPACE
