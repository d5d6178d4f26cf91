"""Host-side checks of the C ABI that need no GPU: the library loads, exports every entry point
the header declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import gated_linear_attention_relu_b200 as la
from gated_linear_attention_relu_b200 import binding as bnd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "la.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(la_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_entry_point():
    lib = la.load()
    names = _declared()
    assert "la_forward_bidir" in names and "la_state_reduce" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) <= set(bnd.EXPORTS)


def test_status_strings():
    for code in range(9):
        assert la.status_string(code) and la.status_string(code) != "unknown status"
    assert la.status_string(99) == "unknown status"


def _call_bidir(p, ptrs=(16, 16, 16, 16, 16)):
    lib = la.load()
    cp = p.c()
    return lib.la_forward_bidir(ctypes.byref(cp), *ptrs, 16, 1 << 30, None)


@pytest.mark.parametrize("kw,status", [
    (dict(d=48, bands=(16, 16, 16)), 5),
    (dict(bands=(32, 48, 40)), 3),
    (dict(bands=(31, 49, 48)), 3),
    (dict(T=-1), 2),
    (dict(eps=float("nan")), 2),
    (dict(rope_base=0.0), 2),
    (dict(block_frames=2), 2),          # la_forward_bidir wants block_frames == 0
    (dict(T=100000, Hh=1000, W=1000), 2),  # N beyond 2^31 tokens
    (dict(t0=-1), 2),                   # frame offset must be >= 0
    (dict(t0=2**31 - 3), 2),            # t0 + T beyond 2^31
])
def test_invalid_problems_rejected_before_cuda(kw, status):
    args = dict(B=1, H=2, T=3, Hh=4, W=5)
    args.update(kw)
    assert _call_bidir(la.Problem(**args)) == status


def test_null_and_misaligned_pointers_rejected_before_cuda():
    p = la.Problem(B=1, H=2, T=3, Hh=4, W=5)
    assert _call_bidir(p, (None, 16, 16, 16, 16)) == 1
    assert _call_bidir(p, (16, 16, 16, 16, 18)) == 4
    lib = la.load()
    cp = p.c()
    assert lib.la_state_reduce(ctypes.byref(cp), 16, 16, None, 16, 16, 1 << 20, None) == 1


def test_invalid_flags_and_dtype():
    lib = la.load()
    cp = la.Problem(B=1, H=1, T=1, Hh=1, W=8).c()
    cp.flags = 8
    assert lib.la_forward_bidir(ctypes.byref(cp), 16, 16, 16, 16, 16, 16, 1, None) == 5
    cp.flags = 0
    cp.dtype = 7
    assert lib.la_forward_bidir(ctypes.byref(cp), 16, 16, 16, 16, 16, 16, 1, None) == 5


def test_workspace_sizes_are_consistent():
    base = la.Problem(B=1, H=32, T=21, Hh=45, W=80)
    ws1 = la.workspace_bytes(base, sm_count=148)
    ws2 = la.workspace_bytes(la.Problem(B=2, H=32, T=21, Hh=45, W=80), sm_count=148)
    assert ws1 > 0 and ws2 > ws1
    # bf16 d=128 uses the tensor-core kernels: partial slots of 128x128 + 8x128 floats, the fp32
    # states and the bf16 operand images.
    units = 32
    assert ws1 >= units * (128 * 128 + 128) * 4 + units * (32768 + 512)
    bc = la.Problem(B=1, H=32, T=81, Hh=45, W=80, block_frames=3)
    assert la.workspace_bytes(bc, sm_count=148) >= 32 * 27 * (32768 + 512)
    assert la.workspace_bytes(la.Problem(B=1, H=1, T=1, Hh=1, W=1, d=40, bands=(8, 16, 16)), 148) == 0
    assert la.workspace_bytes(la.Problem(B=0, H=4, T=2, Hh=2, W=2), sm_count=148) >= 0


def test_host_selftest_of_work_decomposition():
    # Exact fast division and tile/segment bookkeeping, checked on the host by the library itself.
    assert la.load().la_selftest_host() == 0


def test_state_update_rejects_block_causal_problems_before_cuda():
    lib = la.load()
    cp = la.Problem(B=1, H=2, T=3, Hh=4, W=5, block_frames=1).c()
    assert lib.la_state_update(ctypes.byref(cp), 16, 16, 16, 16, 16, 1 << 30, None) == 2
    cp = la.Problem(B=1, H=2, T=3, Hh=4, W=5, t0=-2).c()
    assert lib.la_state_update(ctypes.byref(cp), 16, 16, 16, 16, 16, 1 << 30, None) == 2
    cp = la.Problem(B=1, H=2, T=3, Hh=4, W=5, t0=4).c()
    assert lib.la_state_update(ctypes.byref(cp), None, 16, 16, 16, 16, 1 << 30, None) == 1


def test_tokencausal_rejects_block_causal_problems_before_cuda():
    lib = la.load()
    for kw, status in ((dict(block_frames=1), 2), (dict(dtype="f32", block_frames=2), 2)):
        args = dict(B=1, H=2, T=3, Hh=4, W=5)
        args.update(kw)
        cp = la.Problem(**args).c()
        assert lib.la_forward_tokencausal(ctypes.byref(cp), 16, 16, 16, 16, 16, 16, 1 << 30, None) == status


def test_backward_rejects_bad_arguments_before_cuda():
    lib = la.load()
    for kw, status in ((dict(block_frames=1), 2), (dict(d=48, bands=(16, 16, 16)), 5)):
        args = dict(B=1, H=2, T=3, Hh=4, W=5)
        args.update(kw)
        cp = la.Problem(**args).c()
        assert lib.la_backward_bidir(ctypes.byref(cp), *([16] * 9), 16, 1 << 30, None) == status
    # the general entry point: dbeta is required with a write gate, dgamma with an RMSNorm weight
    cp = la.Problem(B=1, H=2, T=3, Hh=4, W=5, block_frames=1).c()
    g = bnd.LaGates(16, None, 1e-6, 0)
    assert lib.la_backward(ctypes.byref(cp), ctypes.byref(g), *([16] * 9), None, None, 16, 1 << 30, None) == 1
    g = bnd.LaGates(None, 16, 1e-6, 1)
    assert lib.la_backward(ctypes.byref(cp), ctypes.byref(g), *([16] * 9), None, None, 16, 1 << 30, None) == 1
    g = bnd.LaGates(None, 16, 1e-6, 1)
    assert lib.la_backward(ctypes.byref(cp), ctypes.byref(g), *([16] * 9), None, 24, 16, 1 << 30, None) == 4
    g = bnd.LaGates(None, None, 1e-6, 3)
    assert lib.la_backward(ctypes.byref(cp), ctypes.byref(g), *([16] * 9), None, None, 16, 1 << 30, None) == 5
    # with saved states: both states are required and 16-byte aligned; then the same checks
    g = bnd.LaGates(None, None, 1e-6, 0)
    for S, z, status in ((None, 16, 1), (16, None, 1), (24, 16, 4), (16, 40, 4)):
        assert lib.la_backward_saved(ctypes.byref(cp), ctypes.byref(g), S, z, *([16] * 9), None, None, 16, 1 << 30,
                                     None) == status
    assert lib.la_backward_saved(ctypes.byref(cp), ctypes.byref(g), 16, 16, None, *([16] * 8), None, None, 16,
                                 1 << 30, None) == 1
    g = bnd.LaGates(None, None, 1e-6, 3)
    assert lib.la_backward_saved(ctypes.byref(cp), ctypes.byref(g), 16, 16, *([16] * 9), None, None, 16, 1 << 30,
                                 None) == 5


def test_static_entry_point_checks_pointers_before_cuda():
    # A NULL or misaligned tensor is an argument error, reported before the device is queried,
    # even for a problem far too large for the fixed scratch.
    lib = la.load()
    for p in (la.Problem(B=1, H=2, T=3, Hh=4, W=5), la.Problem(B=8, H=64, T=241, Hh=45, W=80)):
        cp = p.c()
        assert lib.la_forward_bidir_static(ctypes.byref(cp), None, 16, 16, 16, 16, None) == 1
        assert lib.la_forward_bidir_static(ctypes.byref(cp), 16, 16, 16, 16, 24, None) == 4
    cp = la.Problem(B=1, H=2, T=3, Hh=4, W=5, block_frames=1).c()
    assert lib.la_forward_bidir_static(ctypes.byref(cp), 16, 16, 16, 16, 16, None) == 2


def test_binding_routes_saved_states_to_la_backward_saved():
    # With S and z the binding calls la_backward_saved, without them la_backward; host tensors and
    # no GPU stop both at their first CUDA call (or, for a misaligned state, at the argument check).
    import torch

    class _Stream:
        cuda_stream = 0

    p = la.Problem(B=1, H=2, T=1, Hh=2, W=8)
    Q, K, V, G, dO = (torch.zeros((1, 2, 16, 128), dtype=torch.bfloat16) for _ in range(5))
    grads = tuple(torch.zeros_like(Q) for _ in range(4))
    ws = torch.zeros(256, dtype=torch.uint8)
    S = torch.zeros((1, 2, 1, 128, 128), dtype=torch.float32)
    z = torch.zeros((1, 2, 1, 128), dtype=torch.float32)
    kw = dict(grads=grads, ws=ws, stream=_Stream())
    with pytest.raises(bnd.LaError, match="la_backward_saved"):
        la.backward(p, Q, K, V, G, dO, S=S, z=z, **kw)
    with pytest.raises(bnd.LaError, match=r"la_backward:"):
        la.backward(p, Q, K, V, G, dO, **kw)
    flat = torch.zeros(2 * 128 * 128 + 1, dtype=torch.float32)
    with pytest.raises(bnd.LaError, match="LA_ERR_ALIGN"):
        la.backward(p, Q, K, V, G, dO, S=flat[1:], z=z, **kw)
