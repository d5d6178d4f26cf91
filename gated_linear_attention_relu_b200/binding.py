"""ctypes binding of ``liblinattn.so`` (the C ABI in include/la.h).

Argument marshalling only: every step of the operator runs in the CUDA library.  PyTorch is
used for device memory (output and workspace tensors) and the current CUDA stream.  If the
library cannot be loaded every call raises; there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblinattn.so")

LA_BF16, LA_F32 = 0, 1
LA_FLAG_FORCE_SIMT = 1
LA_FLAG_TOKEN_CAUSAL = 2

STATUS = {
    0: "LA_OK", 1: "LA_ERR_NULL", 2: "LA_ERR_SHAPE", 3: "LA_ERR_BANDS", 4: "LA_ERR_ALIGN",
    5: "LA_ERR_UNSUPPORTED", 6: "LA_ERR_WORKSPACE", 7: "LA_ERR_CUDA", 8: "LA_ERR_DEVICE",
}

EXPORTS = [
    "la_workspace_bytes", "la_workspace_bytes_for", "la_state_reduce", "la_state_scan", "la_apply",
    "la_forward_bidir", "la_forward_blockcausal", "la_status_string", "la_device_error",
    "la_last_launch_count", "la_forward_marked", "la_selftest_host", "la_forward_bidir_static",
    "la_state_update", "la_forward_gated", "la_block_step", "la_forward_tokencausal", "la_backward_bidir",
    "la_backward", "la_backward_saved",
]


class LaProblem(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int64), ("H", ctypes.c_int64),
        ("T", ctypes.c_int64), ("Hh", ctypes.c_int64), ("W", ctypes.c_int64),
        ("d", ctypes.c_int32), ("dt", ctypes.c_int32), ("dh", ctypes.c_int32), ("dw", ctypes.c_int32),
        ("rope_base", ctypes.c_double), ("eps", ctypes.c_float),
        ("block_frames", ctypes.c_int32), ("dtype", ctypes.c_int32), ("flags", ctypes.c_uint32),
        ("t0", ctypes.c_int64),
    ]


class LaGates(ctypes.Structure):
    _fields_ = [
        ("beta", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("norm_eps", ctypes.c_float),
        ("rms_norm", ctypes.c_int32),
    ]


class LaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status_string(status)})")


_lib = None


def load(path: Optional[str] = None):
    """Load (building first if needed) the CUDA library; raise if that is impossible."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or os.environ.get("LA_LIBRARY") or LIB_PATH
    if not os.path.exists(path) and path == LIB_PATH:
        from . import build as _build

        _build.build()
    try:
        lib = ctypes.CDLL(path)
    except OSError as e:  # no silent fallback: the CUDA library is the product
        raise RuntimeError(f"cannot load the CUDA library {path}: {e}") from e
    P = ctypes.POINTER(LaProblem)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    sig = {
        "la_workspace_bytes": (sz, [P]),
        "la_workspace_bytes_for": (sz, [P, ctypes.c_int]),
        "la_state_reduce": (ctypes.c_int, [P, vp, vp, vp, vp, vp, sz, vp]),
        "la_state_scan": (ctypes.c_int, [P, vp, vp, vp]),
        "la_state_update": (ctypes.c_int, [P, vp, vp, vp, vp, vp, sz, vp]),
        "la_block_step": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "la_forward_tokencausal": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, sz, vp]),
        "la_backward_bidir": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "la_backward": (ctypes.c_int, [P, ctypes.POINTER(LaGates), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                       vp, sz, vp]),
        "la_backward_saved": (ctypes.c_int, [P, ctypes.POINTER(LaGates), vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                             vp, vp, vp, vp, sz, vp]),
        "la_forward_gated": (ctypes.c_int, [P, ctypes.POINTER(LaGates), vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "la_apply": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, sz, vp]),
        "la_forward_bidir": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, sz, vp]),
        "la_forward_blockcausal": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "la_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "la_device_error": (ctypes.c_int, [vp]),
        "la_last_launch_count": (ctypes.c_int, []),
        "la_selftest_host": (ctypes.c_int, []),
        "la_forward_bidir_static": (ctypes.c_int, [P, vp, vp, vp, vp, vp, vp]),
        "la_forward_marked": (ctypes.c_int, [P, ctypes.POINTER(LaGates), vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                             ctypes.POINTER(ctypes.c_void_p), ctypes.c_int]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_string(status: int) -> str:
    lib = load()
    return lib.la_status_string(int(status)).decode()


@dataclass(frozen=True)
class Problem:
    """Sizes and parameters of one call (mirrors ``la_problem``)."""

    B: int
    H: int
    T: int
    Hh: int
    W: int
    d: int = 128
    bands: tuple = (32, 48, 48)
    rope_base: float = 10000.0
    eps: float = 1e-6
    block_frames: int = 0
    dtype: str = "bf16"
    force_simt: bool = False
    t0: int = 0
    token_causal: bool = False  # la_forward_marked runs the token-causal operator  # global index of frame 0 (the t band rotates at t0 + t)

    @property
    def N(self) -> int:
        return self.T * self.Hh * self.W

    @property
    def nblk(self) -> int:
        return 1 if self.block_frames <= 0 else -(-self.T // self.block_frames)

    @classmethod
    def from_workload(cls, w, **kw) -> "Problem":
        args = dict(B=w.B, H=w.H, T=w.T, Hh=w.Hh, W=w.W, d=w.d, bands=tuple(w.bands),
                    rope_base=w.rope_base, eps=w.eps, block_frames=w.block_frames, dtype=w.dtype)
        args.update(kw)
        return cls(**args)

    def c(self) -> LaProblem:
        return LaProblem(self.B, self.H, self.T, self.Hh, self.W, self.d, self.bands[0], self.bands[1],
                         self.bands[2], float(self.rope_base), float(self.eps), int(self.block_frames),
                         LA_BF16 if self.dtype == "bf16" else LA_F32,
                         (LA_FLAG_FORCE_SIMT if self.force_simt else 0) |
                         (LA_FLAG_TOKEN_CAUSAL if self.token_causal else 0), int(self.t0))


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(rc: int, where: str):
    if rc != 0:
        raise LaError(rc, where)


def _torch_dtype(p: Problem):
    import torch

    return torch.bfloat16 if p.dtype == "bf16" else torch.float32


def workspace_bytes(p: Problem, sm_count: Optional[int] = None) -> int:
    lib = load()
    cp = p.c()
    if sm_count is None:
        return int(lib.la_workspace_bytes(ctypes.byref(cp)))
    return int(lib.la_workspace_bytes_for(ctypes.byref(cp), int(sm_count)))


def workspace(p: Problem, device="cuda"):
    import torch

    n = workspace_bytes(p)
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device), n


def state_reduce(p: Problem, K, V, S=None, z=None, ws=None, stream=None):
    """Per-unit states S [B,H,nblk,d,d] and z [B,H,nblk,d] (fp32, not prefixed)."""
    import torch

    lib = load()
    if S is None:
        S = torch.empty((p.B, p.H, p.nblk, p.d, p.d), dtype=torch.float32, device=K.device)
    if z is None:
        z = torch.empty((p.B, p.H, p.nblk, p.d), dtype=torch.float32, device=K.device)
    if ws is None:
        ws, nbytes = workspace(p, K.device)
    else:
        nbytes = ws.numel()
    cp = p.c()
    _check(lib.la_state_reduce(ctypes.byref(cp), _ptr(K), _ptr(V), _ptr(S), _ptr(z), _ptr(ws), nbytes,
                               _stream(stream)), "la_state_reduce")
    return S, z


def state_update(p: Problem, K, V, S, z, ws=None, stream=None):
    """Cache update of block-autoregressive generation: S += sum phi(K)^T V, z += sum ReLU(K)
    over the call's tokens, in place (S [B,H,d,d], z [B,H,d] fp32; ``p.block_frames`` = 0 and
    ``p.t0`` = the block's first global frame)."""
    lib = load()
    if ws is None:
        ws, nbytes = workspace(p, K.device)
    else:
        nbytes = ws.numel()
    cp = p.c()
    _check(lib.la_state_update(ctypes.byref(cp), _ptr(K), _ptr(V), _ptr(S), _ptr(z), _ptr(ws), nbytes,
                               _stream(stream)), "la_state_update")
    return S, z


def block_step(p: Problem, Q, K, V, G, S, z, O=None, ws=None, stream=None):
    """One block of block-autoregressive generation: fold the block into the carried cache
    (S [B,H,d,d], z [B,H,d], in place) and return its outputs against the updated cache."""
    import torch

    lib = load()
    if O is None:
        O = torch.empty_like(Q)
    if ws is None:
        ws, nbytes = workspace(p, Q.device)
    else:
        nbytes = ws.numel()
    cp = p.c()
    _check(lib.la_block_step(ctypes.byref(cp), _ptr(Q), _ptr(K), _ptr(V), _ptr(G), _ptr(O), _ptr(S), _ptr(z),
                             _ptr(ws), nbytes, _stream(stream)), "la_block_step")
    return O


def state_scan(p: Problem, S, z, stream=None):
    lib = load()
    cp = p.c()
    _check(lib.la_state_scan(ctypes.byref(cp), _ptr(S), _ptr(z), _stream(stream)), "la_state_scan")
    return S, z


def apply(p: Problem, Q, G, S, z, O=None, ws=None, stream=None):
    import torch

    lib = load()
    if O is None:
        O = torch.empty_like(Q)
    if ws is None:
        ws, nbytes = workspace(p, Q.device)
    else:
        nbytes = ws.numel()
    cp = p.c()
    _check(lib.la_apply(ctypes.byref(cp), _ptr(Q), _ptr(G), _ptr(S), _ptr(z), _ptr(O), _ptr(ws), nbytes,
                        _stream(stream)), "la_apply")
    return O


def forward_bidir(p: Problem, Q, K, V, G, O=None, ws=None, stream=None):
    import torch

    lib = load()
    if O is None:
        O = torch.empty_like(Q)
    if ws is None:
        ws, nbytes = workspace(p, Q.device)
    else:
        nbytes = ws.numel()
    cp = p.c()
    _check(lib.la_forward_bidir(ctypes.byref(cp), _ptr(Q), _ptr(K), _ptr(V), _ptr(G), _ptr(O), _ptr(ws),
                                nbytes, _stream(stream)), "la_forward_bidir")
    return O


def forward_bidir_static(p: Problem, Q, K, V, G, O, stream=None):
    """la_forward_bidir without a workspace: the library's fixed device scratch is used instead
    (for callers that cannot allocate device memory).  ``O`` must be given; nothing is allocated."""
    lib = load()
    cp = p.c()
    _check(lib.la_forward_bidir_static(ctypes.byref(cp), _ptr(Q), _ptr(K), _ptr(V), _ptr(G), _ptr(O),
                                       _stream(stream)), "la_forward_bidir_static")
    return O


def forward_blockcausal(p: Problem, Q, K, V, G, O=None, S_incl=None, z_incl=None, ws=None,
                        return_states=False, stream=None):
    import torch

    lib = load()
    if O is None:
        O = torch.empty_like(Q)
    if return_states and S_incl is None:
        S_incl = torch.empty((p.B, p.H, p.nblk, p.d, p.d), dtype=torch.float32, device=Q.device)
        z_incl = torch.empty((p.B, p.H, p.nblk, p.d), dtype=torch.float32, device=Q.device)
    if ws is None:
        ws, nbytes = workspace(p, Q.device)
    else:
        nbytes = ws.numel()
    cp = p.c()
    _check(lib.la_forward_blockcausal(ctypes.byref(cp), _ptr(Q), _ptr(K), _ptr(V), _ptr(G), _ptr(O),
                                      _ptr(S_incl), _ptr(z_incl), _ptr(ws), nbytes, _stream(stream)),
           "la_forward_blockcausal")
    if return_states:
        return O, S_incl, z_incl
    return O


def forward_gated(p: Problem, Q, K, V, G, beta=None, gamma=None, rms_norm=False, norm_eps=1e-6, O=None,
                  S_incl=None, z_incl=None, ws=None, return_states=False, stream=None):
    """The full gated form: write gate ``beta`` [B,H,N] (problem dtype) on the state, and RMSNorm
    (weight ``gamma`` [d] fp32, or None) of num/den before the output gate when ``rms_norm``.
    Bidirectional or block-causal as ``p.block_frames`` says."""
    import torch

    lib = load()
    if O is None:
        O = torch.empty_like(Q)
    if return_states and S_incl is None:
        S_incl = torch.empty((p.B, p.H, p.nblk, p.d, p.d), dtype=torch.float32, device=Q.device)
        z_incl = torch.empty((p.B, p.H, p.nblk, p.d), dtype=torch.float32, device=Q.device)
    if ws is None:
        ws, nbytes = workspace(p, Q.device)
    else:
        nbytes = ws.numel()
    cp = p.c()
    gates = LaGates(_ptr(beta), _ptr(gamma), float(norm_eps), 1 if rms_norm else 0)
    _check(lib.la_forward_gated(ctypes.byref(cp), ctypes.byref(gates), _ptr(Q), _ptr(K), _ptr(V), _ptr(G),
                                _ptr(O), _ptr(S_incl), _ptr(z_incl), _ptr(ws), nbytes, _stream(stream)),
           "la_forward_gated")
    if return_states:
        return O, S_incl, z_incl
    return O


def forward_tokencausal(p: Problem, Q, K, V, G, O=None, ws=None, stream=None):
    """Token-causal operator: token n reads the states of tokens 0..n."""
    import torch

    lib = load()
    if O is None:
        O = torch.empty_like(Q)
    if ws is None:
        ws, nbytes = workspace(p, Q.device)
    else:
        nbytes = ws.numel()
    cp = p.c()
    _check(lib.la_forward_tokencausal(ctypes.byref(cp), _ptr(Q), _ptr(K), _ptr(V), _ptr(G), _ptr(O), _ptr(ws),
                                      nbytes, _stream(stream)), "la_forward_tokencausal")
    return O


def backward_bidir(p: Problem, Q, K, V, G, dO, grads=None, ws=None, stream=None):
    """Gradients (dQ, dK, dV, dG) of the bidirectional operator given the output gradient dO."""
    import torch

    lib = load()
    if grads is None:
        grads = tuple(torch.empty_like(Q) for _ in range(4))
    dQ, dK, dV, dG = grads
    if ws is None:
        ws, nbytes = workspace(p, Q.device)
    else:
        nbytes = ws.numel()
    cp = p.c()
    _check(lib.la_backward_bidir(ctypes.byref(cp), _ptr(Q), _ptr(K), _ptr(V), _ptr(G), _ptr(dO), _ptr(dQ), _ptr(dK),
                                 _ptr(dV), _ptr(dG), _ptr(ws), nbytes, _stream(stream)), "la_backward_bidir")
    return dQ, dK, dV, dG


def backward(p: Problem, Q, K, V, G, dO, beta=None, gamma=None, rms_norm=False, norm_eps=1e-6, grads=None,
             ws=None, stream=None, S=None, z=None):
    """Gradients of the operator in any form (bidirectional or block-causal as ``p.block_frames``
    says; write gate ``beta`` and RMSNorm optional): returns (dQ, dK, dV, dG, dbeta, dgamma), with
    dbeta [B,H,N] when ``beta`` is given and dgamma [d] fp32 when RMSNorm has a weight ``gamma``
    (else None).  ``S``, ``z``: the states the forward pass returned (``forward_gated(...,
    return_states=True)``); given, the state is not reduced again (la_backward_saved)."""
    import torch

    lib = load()
    if grads is None:
        grads = tuple(torch.empty_like(Q) for _ in range(4))
    dQ, dK, dV, dG = grads
    dbeta = torch.empty_like(beta) if beta is not None else None
    dgamma = torch.empty_like(gamma) if (rms_norm and gamma is not None) else None
    if ws is None:
        ws, nbytes = workspace(p, Q.device)
    else:
        nbytes = ws.numel()
    cp = p.c()
    gates = LaGates(_ptr(beta), _ptr(gamma), float(norm_eps), 1 if rms_norm else 0)
    if S is not None or z is not None:
        _check(lib.la_backward_saved(ctypes.byref(cp), ctypes.byref(gates), _ptr(S), _ptr(z), _ptr(Q), _ptr(K),
                                     _ptr(V), _ptr(G), _ptr(dO), _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dG),
                                     _ptr(dbeta), _ptr(dgamma), _ptr(ws), nbytes, _stream(stream)),
               "la_backward_saved")
    else:
        _check(lib.la_backward(ctypes.byref(cp), ctypes.byref(gates), _ptr(Q), _ptr(K), _ptr(V), _ptr(G), _ptr(dO),
                               _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dG), _ptr(dbeta), _ptr(dgamma), _ptr(ws), nbytes,
                               _stream(stream)), "la_backward")
    return dQ, dK, dV, dG, dbeta, dgamma


def forward(p: Problem, Q, K, V, G, **kw):
    """Bidirectional or block-causal, as ``p.block_frames`` says."""
    if p.block_frames > 0:
        return forward_blockcausal(p, Q, K, V, G, **kw)
    return forward_bidir(p, Q, K, V, G, **kw)


def forward_marked(p: Problem, Q, K, V, G, O, ws, events, S_incl=None, z_incl=None, stream=None, beta=None,
                   gamma=None, rms_norm=False, norm_eps=1e-6):
    """Forward pass recording ``events[0]`` before the first kernel and ``events[i]`` after kernel i.

    ``events`` are ``torch.cuda.Event(enable_timing=True)`` objects; each is recorded once on
    the stream first so that its CUDA handle exists.
    """
    import torch

    lib = load()
    st = torch.cuda.current_stream() if stream is None else stream
    for e in events:
        if e.cuda_event == 0:
            e.record(st)
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    cp = p.c()
    gates = LaGates(_ptr(beta), _ptr(gamma), float(norm_eps), 1 if rms_norm else 0) if (beta is not None or rms_norm) else None
    _check(lib.la_forward_marked(ctypes.byref(cp), None if gates is None else ctypes.byref(gates), _ptr(Q), _ptr(K), _ptr(V), _ptr(G), _ptr(O),
                                 _ptr(S_incl), _ptr(z_incl), _ptr(ws), ws.numel(), st.cuda_stream,
                                 arr, len(events)), "la_forward_marked")
    return O


def device_error(stream=None) -> int:
    lib = load()
    return int(lib.la_device_error(_stream(stream)))


def last_launch_count() -> int:
    return int(load().la_last_launch_count())
