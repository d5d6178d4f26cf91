"""The checked build and the bounded-wait abort path, on the GPU, with no fault.

The checked build (LA_CHECKED) tests every index the kernels derive from the work decomposition
against its extent and records a failure in the device error word; run on small shapes it must
give exactly the regular library's outputs and a clean error word.  The same build carries a test
hook (LA_TEST_HOOKS) that makes the state kernel skip one tile's K load, so the waits for that
tile run out after their (here 50 ms) limit: the kernels must wind down and return, the error word
must read LA_ERR_DEVICE, and the next call on the same GPU must be correct again.
"""
import ctypes

import pytest
import torch

import gated_linear_attention_relu_b200 as la
from gated_linear_attention_relu_b200 import binding as bnd
from gated_linear_attention_relu_b200 import build
from gated_linear_attention_relu_b200 import workloads as wl

pytestmark = pytest.mark.gpu

LA_ERR_DEVICE = 8


@pytest.fixture(scope="module")
def checked(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("checked") / "liblinattn_checked.so")
    build.build_variant(out, ["LA_CHECKED", "LA_TEST_HOOKS", "LA_WAIT_LIMIT_NS=50000000ull"])
    lib = ctypes.CDLL(out)
    P, vp, sz = ctypes.POINTER(bnd.LaProblem), ctypes.c_void_p, ctypes.c_size_t
    lib.la_workspace_bytes.restype, lib.la_workspace_bytes.argtypes = sz, [P]
    for name, args in (("la_forward_bidir", [P, vp, vp, vp, vp, vp, vp, sz, vp]),
                       ("la_forward_blockcausal", [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
                       ("la_forward_tokencausal", [P, vp, vp, vp, vp, vp, vp, sz, vp]),
                       ("la_backward_bidir", [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
                       ("la_device_error", [vp]), ("la_test_skip_tile", [ctypes.c_longlong])):
        getattr(lib, name).restype = ctypes.c_int
        getattr(lib, name).argtypes = args
    yield lib
    lib.la_test_skip_tile(-1)


def _ws(lib, p):
    cp = p.c()
    n = lib.la_workspace_bytes(ctypes.byref(cp))
    return torch.empty(max(n, 16), dtype=torch.uint8, device="cuda"), n


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _forward(lib, p, Q, K, V, G):
    O = torch.empty_like(Q)
    ws, n = _ws(lib, p)
    cp = p.c()
    if p.block_frames > 0:
        rc = lib.la_forward_blockcausal(ctypes.byref(cp), Q.data_ptr(), K.data_ptr(), V.data_ptr(), G.data_ptr(),
                                        O.data_ptr(), None, None, ws.data_ptr(), n, _stream())
    else:
        rc = lib.la_forward_bidir(ctypes.byref(cp), Q.data_ptr(), K.data_ptr(), V.data_ptr(), G.data_ptr(),
                                  O.data_ptr(), ws.data_ptr(), n, _stream())
    assert rc == 0
    return O


CASES = [
    wl.custom("chk_ragged", B=1, H=3, T=3, Hh=5, W=37),                # ragged last tile
    wl.custom("chk_heads", B=3, H=70, T=1, Hh=2, W=64),                # CTAs span several heads
    wl.custom("chk_split", B=1, H=2, T=20, Hh=20, W=40),               # heads split over many CTAs
    wl.custom("chk_bc", B=1, H=2, T=7, Hh=6, W=10, block_frames=2),    # blocks end inside tiles
    wl.custom("chk_f32", B=1, H=2, T=3, Hh=4, W=11, d=64, bands=(16, 24, 24), dtype="f32"),
    wl.custom("chk_single", B=1, H=2, T=1, Hh=1, W=1),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_checked_build_matches_regular_build_with_clean_error_word(checked, w):
    Q, K, V, G = wl.generate(w, "cuda")
    p = la.Problem.from_workload(w)
    ref = la.forward(p, Q, K, V, G)
    O = _forward(checked, p, Q, K, V, G)
    assert checked.la_device_error(_stream()) == 0
    assert torch.equal(O, ref)


def test_checked_build_tokencausal_and_backward(checked):
    w = CASES[2]
    Q, K, V, G = wl.generate(w, "cuda")
    dO = wl.generate_grad(w, "cuda")
    p = la.Problem.from_workload(w)
    ws, n = _ws(checked, p)
    cp = p.c()
    O = torch.empty_like(Q)
    assert checked.la_forward_tokencausal(ctypes.byref(cp), Q.data_ptr(), K.data_ptr(), V.data_ptr(),
                                          G.data_ptr(), O.data_ptr(), ws.data_ptr(), n, _stream()) == 0
    grads = [torch.empty_like(Q) for _ in range(4)]
    assert checked.la_backward_bidir(ctypes.byref(cp), Q.data_ptr(), K.data_ptr(), V.data_ptr(), G.data_ptr(),
                                     dO.data_ptr(), *[g.data_ptr() for g in grads], ws.data_ptr(), n,
                                     _stream()) == 0
    assert checked.la_device_error(_stream()) == 0
    assert torch.equal(O, la.forward_tokencausal(p, Q, K, V, G))
    for a, b in zip(grads, la.backward_bidir(p, Q, K, V, G, dO)):
        assert torch.equal(a, b)


def test_lost_arrival_times_out_and_the_next_call_is_correct(checked):
    w = wl.custom("chk_abort", B=1, H=2, T=4, Hh=8, W=40)   # 2,560 tokens: 20 tiles per head
    Q, K, V, G = wl.generate(w, "cuda")
    p = la.Problem.from_workload(w)
    ref = la.forward(p, Q, K, V, G)
    torch.cuda.synchronize()
    # The state kernel never loads tile 3: its waits run out and every kernel of the call returns.
    assert checked.la_test_skip_tile(3) == 0
    _forward(checked, p, Q, K, V, G)
    assert checked.la_device_error(_stream()) == LA_ERR_DEVICE
    assert checked.la_device_error(_stream()) == 0  # reading the word cleared it
    # Same GPU, same process: the next call is correct and clean.
    assert checked.la_test_skip_tile(-1) == 0
    O = _forward(checked, p, Q, K, V, G)
    assert checked.la_device_error(_stream()) == 0
    assert torch.equal(O, ref)
