"""fp64 CPU oracle for the gated ReLU linear-attention token mixer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module: only the tests, the smoke check and the CPU-baseline leg of the
benchmark use it.  It shares no code with the CUDA library.

What it computes, per (batch, head), written out as plainly as possible:

* Feature map and RoPE placement -- "SANA-Video: Efficient Video Generation
  with Block Linear Diffusion Transformer", Sec. 3.2 (the RoPE-after-ReLU
  formula and its pseudocode): RoPE is applied to ReLU(x), and only in the
  numerator; the denominator uses the un-rotated ReLU features.
* State, normaliser, gate -- "SANA-Video 2.0: Hybrid Linear Attention with
  Attention Residuals for Efficient Video Generation", Sec. 2, Eq. (1):
  S = sum_n beta_n k_n^r v_n^T, o_j = RMSNorm((q_j^r S) / (sum_n phi(k_n).phi(q_j)
  + eps)) * sigmoid(g_j).  By default beta = 1 and there is no RMSNorm (the
  operator's main form); both are optional arguments (``beta`` per token,
  ``rms = (gamma, norm_eps)``).  beta scales only the state: the denominator of
  Eq. (1) has none.  RMSNorm sits before the gate, as in Eq. (1) of that page
  (the page's other rendering puts it after the gate); W_o is outside.
* Block-causal mode -- "SANA-Video" Sec. 3.4 (causal linear attention with a
  constant-memory cache, and Algorithm 1's per-block cache update): a token
  in block b reads the sum of the states of blocks 0..b, its own block
  included.
* Token-causal mode -- the same section's causal form, token by token: token n
  reads the states of tokens 0..n (itself included) in the flattened order.

Readings where the pages are silent (each one is listed in the design notes):
3D RoPE splits d into consecutive t / h / w bands; pair i of a band of width D
rotates channels (2i, 2i+1) of that band by angle pos * base**(-2i/D),
counter-clockwise; positions are the integer latent indices starting at 0;
token n sits at grid position (t, h, w) with n = (t*Hh + h)*W + w; eps is added
after the dot product.

Every input is converted to float64 exactly before use, and all arithmetic is
float64.  A matrix product (numpy ``@``) is the only library primitive used.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "band_frequencies", "grid_positions", "relu", "sigmoid", "rope3d",
    "head_state", "head_apply", "forward_positions", "forward_bidir",
    "block_of_tokens", "block_states", "forward_blockcausal", "forward_brute", "rms_norm",
    "tokencausal_rows", "forward_tokencausal", "rope3d_transpose", "head_backward", "backward_bidir",
    "head_backward_gated", "backward_gated",
]


def band_frequencies(D: int, base: float) -> np.ndarray:
    """theta_i = base ** (-2 i / D) for the D/2 pairs of one RoPE band."""
    i = np.arange(D // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / float(D))


def grid_positions(T: int, Hh: int, W: int) -> np.ndarray:
    """(N, 3) integer positions (t, h, w) of the tokens, n = (t*Hh + h)*W + w."""
    t, h, w = np.meshgrid(np.arange(T), np.arange(Hh), np.arange(W), indexing="ij")
    return np.stack([t.reshape(-1), h.reshape(-1), w.reshape(-1)], axis=1).astype(np.int64)


def relu(x: np.ndarray) -> np.ndarray:
    """phi = ReLU ("SANA-Video 2.0", Sec. 2)."""
    return np.maximum(x, 0.0)


def sigmoid(x: np.ndarray) -> np.ndarray:
    """The logistic output gate sigma(g) of Eq. (1)."""
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def rope3d(x: np.ndarray, pos: np.ndarray, bands, base: float) -> np.ndarray:
    """Rotate each channel pair of each band by its position along that band's axis.

    x: (N, d) float64; pos: (N, 3) positions (t, h, w); bands = (dt, dh, dw).
    Channel block [0, dt) follows t, [dt, dt+dh) follows h, [dt+dh, d) follows w.
    """
    x = np.asarray(x, dtype=np.float64)
    y = x.copy()
    off = 0
    for axis, D in enumerate(bands):
        theta = band_frequencies(D, base)
        p = pos[:, axis].astype(np.float64)
        for i in range(D // 2):
            angle = p * theta[i]
            c, s = np.cos(angle), np.sin(angle)
            x0 = x[:, off + 2 * i]
            x1 = x[:, off + 2 * i + 1]
            y[:, off + 2 * i] = x0 * c - x1 * s
            y[:, off + 2 * i + 1] = x0 * s + x1 * c
        off += D
    assert off == x.shape[1], "bands must add up to d"
    return y


def head_state(k: np.ndarray, v: np.ndarray, pos: np.ndarray, bands, base: float, beta=None):
    """S = sum_n beta_n RoPE(ReLU(k_n))^T v_n (d x d) and z = sum_n ReLU(k_n) (d) over the given
    tokens (beta = 1 when None; z is never gated)."""
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    kp = relu(k)
    kr = rope3d(kp, pos, bands, base)
    if beta is not None:
        kr = kr * np.asarray(beta, dtype=np.float64)[:, None]
    S = kr.T @ v
    z = kp.sum(axis=0)
    return S, z


def rms_norm(y: np.ndarray, gamma, norm_eps: float) -> np.ndarray:
    """Row-wise RMSNorm over the channels: y / sqrt(mean(y^2) + norm_eps) * gamma (gamma = 1 if None)."""
    y = np.asarray(y, dtype=np.float64)
    out = y / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + float(norm_eps))
    if gamma is not None:
        out = out * np.asarray(gamma, dtype=np.float64)
    return out


def head_apply(q: np.ndarray, g: np.ndarray, S: np.ndarray, z: np.ndarray, pos: np.ndarray,
               bands, base: float, eps: float, rms=None) -> np.ndarray:
    """o_n = (RoPE(ReLU(q_n)) S) / (ReLU(q_n) . z + eps) * sigmoid(g_n); with ``rms = (gamma,
    norm_eps)`` the quotient is RMS-normalised before the gate."""
    q = np.asarray(q, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    qp = relu(q)
    qr = rope3d(qp, pos, bands, base)
    num = qr @ S
    den = qp @ z + float(eps)
    y = num / den[:, None]
    if rms is not None:
        y = rms_norm(y, rms[0], rms[1])
    return y * sigmoid(g)


def forward_positions(q, k, v, g, pos, bands, base, eps, beta=None, rms=None):
    """Bidirectional output of one head whose tokens sit at explicit positions ``pos``."""
    S, z = head_state(k, v, pos, bands, base, beta)
    return head_apply(q, g, S, z, pos, bands, base, eps, rms)


def _heads(x):
    x = np.asarray(x, dtype=np.float64)
    B, H, N, d = x.shape
    return x.reshape(B * H, N, d)


def forward_bidir(Q, K, V, G, grid, bands, base=10000.0, eps=1e-6, return_state=False, beta=None, rms=None):
    """Bidirectional mixer over [B, H, N, d] inputs on a (T, Hh, W) latent grid (``beta``: [B, H, N])."""
    T, Hh, W = grid
    pos = grid_positions(T, Hh, W)
    B, H, N, d = np.shape(Q)
    assert N == T * Hh * W
    q, k, v, g = _heads(Q), _heads(K), _heads(V), _heads(G)
    O = np.empty((B * H, N, d))
    Ss = np.empty((B * H, d, d))
    zs = np.empty((B * H, d))
    bt = None if beta is None else np.asarray(beta, dtype=np.float64).reshape(B * H, N)
    for u in range(B * H):
        Ss[u], zs[u] = head_state(k[u], v[u], pos, bands, base, None if bt is None else bt[u])
        O[u] = head_apply(q[u], g[u], Ss[u], zs[u], pos, bands, base, eps, rms)
    O = O.reshape(B, H, N, d)
    if return_state:
        return O, Ss.reshape(B, H, d, d), zs.reshape(B, H, d)
    return O


def block_of_tokens(pos: np.ndarray, block_frames: int) -> np.ndarray:
    """Block index of each token: floor(t / block_frames)."""
    return pos[:, 0] // int(block_frames)


def block_states(k, v, pos, bands, base, block_frames, beta=None):
    """Per-block states (not prefixed) of one head: S_b, z_b for b = 0..nblk-1."""
    blk = block_of_tokens(pos, block_frames)
    nblk = int(blk.max()) + 1 if len(blk) else 0
    d = k.shape[1]
    Sb = np.zeros((nblk, d, d))
    zb = np.zeros((nblk, d))
    for b in range(nblk):
        sel = blk == b
        Sb[b], zb[b] = head_state(k[sel], v[sel], pos[sel], bands, base, None if beta is None else beta[sel])
    return Sb, zb


def forward_blockcausal(Q, K, V, G, grid, bands, base=10000.0, eps=1e-6, block_frames=1,
                        return_state=False, beta=None, rms=None):
    """Block-causal mixer: a token of block b reads sum_{b' <= b} (S_b', z_b').

    Returns O and, if asked, the inclusive per-block states [B, H, nblk, d, d] and
    [B, H, nblk, d] (the constant-memory cache after each block).
    """
    T, Hh, W = grid
    pos = grid_positions(T, Hh, W)
    B, H, N, d = np.shape(Q)
    q, k, v, g = _heads(Q), _heads(K), _heads(V), _heads(G)
    blk = block_of_tokens(pos, block_frames)
    nblk = -(-T // block_frames)
    O = np.empty((B * H, N, d))
    Sinc = np.empty((B * H, nblk, d, d))
    zinc = np.empty((B * H, nblk, d))
    bt = None if beta is None else np.asarray(beta, dtype=np.float64).reshape(B * H, N)
    for u in range(B * H):
        Sb, zb = block_states(k[u], v[u], pos, bands, base, block_frames, None if bt is None else bt[u])
        S_run = np.zeros((d, d))
        z_run = np.zeros(d)
        for b in range(nblk):
            S_run = S_run + Sb[b]
            z_run = z_run + zb[b]
            Sinc[u, b], zinc[u, b] = S_run, z_run
            sel = blk == b
            O[u][sel] = head_apply(q[u][sel], g[u][sel], S_run, z_run, pos[sel], bands, base, eps, rms)
    O = O.reshape(B, H, N, d)
    if return_state:
        return O, Sinc.reshape(B, H, nblk, d, d), zinc.reshape(B, H, nblk, d)
    return O


def forward_brute(q, k, v, g, pos, bands, base, eps, visible=None, beta=None, rms=None):
    """O(N^2) form of one head: o_n = sum_m beta_m (q_n^r . k_m^r) v_m / (sum_m q_n^+ . k_m^+ + eps)
    * sigmoid(g_n) (the quotient RMS-normalised first when ``rms = (gamma, norm_eps)``).

    ``visible[n, m]`` (bool) restricts which keys token n reads; None means all.
    This is the pair-wise form the linear one is the associative rewrite of.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    qp, kp = relu(q), relu(k)
    qr, kr = rope3d(qp, pos, bands, base), rope3d(kp, pos, bands, base)
    N = q.shape[0]
    out = np.empty_like(q)
    for n in range(N):
        m = np.arange(N) if visible is None else np.nonzero(visible[n])[0]
        a = kr[m] @ qr[n]  # rotated similarities
        if beta is not None:
            a = a * np.asarray(beta, dtype=np.float64)[m]
        b = kp[m] @ qp[n]  # un-rotated similarities
        y = (a @ v[m]) / (b.sum() + float(eps))
        if rms is not None:
            y = rms_norm(y, rms[0], rms[1])
        out[n] = y * sigmoid(g[n])
    return out


def tokencausal_rows(q, k, v, g, pos, bands, base, eps, rows=None):
    """Token-causal output of one head at the listed token indices (all when None):
    o_n = (RoPE(q_n^+) S_{<=n}) / (q_n^+ . z_{<=n} + eps) * sigmoid(g_n), with
    S_{<=n} = sum_{m<=n} RoPE(k_m^+)^T v_m and z_{<=n} = sum_{m<=n} k_m^+.

    A running prefix sum: the tokens are walked in order and, before row n is evaluated, the
    tokens since the previous requested row (up to n itself) are added to (S, z)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    N, d = q.shape
    order = np.arange(N) if rows is None else np.unique(np.asarray(rows))
    kp = relu(k)
    kr = rope3d(kp, pos, bands, base)
    S = np.zeros((d, d))
    z = np.zeros(d)
    done = 0  # tokens 0 .. done-1 are in (S, z)
    out = {}
    for n in order:
        n = int(n)
        S = S + kr[done:n + 1].T @ v[done:n + 1]
        z = z + kp[done:n + 1].sum(axis=0)
        done = n + 1
        out[n] = head_apply(q[n:n + 1], g[n:n + 1], S, z, pos[n:n + 1], bands, base, eps)[0]
    return np.array([out[int(n)] for n in (np.arange(N) if rows is None else np.asarray(rows))])


def forward_tokencausal(Q, K, V, G, grid, bands, base=10000.0, eps=1e-6):
    """Token-causal mixer over [B, H, N, d] inputs on a (T, Hh, W) latent grid."""
    T, Hh, W = grid
    pos = grid_positions(T, Hh, W)
    B, H, N, d = np.shape(Q)
    q, k, v, g = _heads(Q), _heads(K), _heads(V), _heads(G)
    O = np.empty((B * H, N, d))
    for u in range(B * H):
        O[u] = tokencausal_rows(q[u], k[u], v[u], g[u], pos, bands, base, eps)
    return O.reshape(B, H, N, d)


# ----------------------------------------------------------------- gradients (bidirectional form)

def rope3d_transpose(x: np.ndarray, pos: np.ndarray, bands, base: float) -> np.ndarray:
    """The transpose of the RoPE map at each position (rotation by the opposite angle):
    (x0, x1) -> (x0 cos a + x1 sin a, -x0 sin a + x1 cos a)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    o = 0
    for axis, D in enumerate(bands):
        if D == 0:
            continue
        theta = band_frequencies(D, base)
        ang = pos[:, axis:axis + 1].astype(np.float64) * theta[None, :]
        c, s_ = np.cos(ang), np.sin(ang)
        x0, x1 = x[:, o:o + D:2], x[:, o + 1:o + D:2]
        out[:, o:o + D:2] = x0 * c + x1 * s_
        out[:, o + 1:o + D:2] = -x0 * s_ + x1 * c
        o += D
    return out


def head_backward(q, k, v, g, do, pos, bands, base, eps):
    """Gradients of the bidirectional mixer of one head with respect to q, k, v, g, given the
    output gradient ``do``.  With phi = RoPE(ReLU), S = sum phi(k)^T v, z = sum ReLU(k),
    num = phi(q) S, den = ReLU(q).z + eps, y = num / den, o = y * sigmoid(g), the chain rule
    gives, per token n (ReLU'(x) taken as [x > 0]):
      dg = do * y * s (1 - s),  dy = do * s,  dnum = dy / den,  dden = -(dy . y) / den
      dS = sum_n phi(q_n)^T dnum_n,  dz = sum_n dden_n ReLU(q_n)
      dq = [q > 0] * (RoPE^T(dnum S^T) + dden z)
      dv = phi(k) dS,  dk = [k > 0] * (RoPE^T(v dS^T) + dz)."""
    q, k, v, g, do = (np.asarray(a, dtype=np.float64) for a in (q, k, v, g, do))
    qp, kp = relu(q), relu(k)
    qr, kr = rope3d(qp, pos, bands, base), rope3d(kp, pos, bands, base)
    S = kr.T @ v
    z = kp.sum(axis=0)
    num = qr @ S
    den = qp @ z + float(eps)
    y = num / den[:, None]
    sg = sigmoid(g)
    dg = do * y * sg * (1.0 - sg)
    dy = do * sg
    dnum = dy / den[:, None]
    dden = -np.sum(dy * y, axis=1) / den
    dS = qr.T @ dnum
    dz = qp.T @ dden
    dq = (q > 0) * (rope3d_transpose(dnum @ S.T, pos, bands, base) + dden[:, None] * z[None, :])
    dv = kr @ dS
    dk = (k > 0) * (rope3d_transpose(v @ dS.T, pos, bands, base) + dz[None, :])
    return dq, dk, dv, dg


def head_backward_gated(q, k, v, g, do, pos, bands, base, eps, block_frames=0, beta=None, rms=None):
    """Gradients of one head of the operator in its full form: block-causal when block_frames > 0
    (token n reads the summed states of the blocks up to its own), write gate beta per token on the
    state, RMSNorm (rms = (gamma, norm_eps)) before the output gate.  Returns dq, dk, dv, dg, dbeta
    (None without beta) and dgamma (None without RMSNorm or with gamma None).

    Forward, per token n in block b(n) (one block in the bidirectional form):
      S_b = sum_{m: b(m) <= b} beta_m phi(k_m)^T v_m,  z_b = sum_{m: b(m) <= b} ReLU(k_m),
      y_n = (phi(q_n) S_{b(n)}) / (ReLU(q_n) . z_{b(n)} + eps),
      u_n = y_n / r_n * gamma with r_n = sqrt(mean(y_n^2) + norm_eps)   (u = y without RMSNorm),
      o_n = u_n * sigmoid(g_n).
    Chain rule:
      dg = do u s (1 - s),  du = do s,  dgamma = sum_n du_n y_n / r_n,
      dy = (dyh - yh (yh . dyh) / d) / r with yh = y / r and dyh = du gamma   (dy = du without),
      dnum = dy / den,  dden = -(dy . y) / den,
      dS_b = sum_{n in block b} phi(q_n)^T dnum_n,  dz_b = sum_{n in block b} dden_n ReLU(q_n),
      and a key of block c feeds every S_b with b >= c, so it sees the suffix sums
      dS^c = sum_{b >= c} dS_b,  dz^c = sum_{b >= c} dz_b:
      dq = [q > 0] (RoPE^T(dnum S_{b(n)}^T) + dden z_{b(n)}),
      dv_m = beta_m phi(k_m) dS^{b(m)},  dk_m = [k > 0] (RoPE^T(beta_m v_m dS^{b(m)T}) + dz^{b(m)}),
      dbeta_m = phi(k_m) . (dS^{b(m)} v_m)."""
    q, k, v, g, do = (np.asarray(a, dtype=np.float64) for a in (q, k, v, g, do))
    N, d = q.shape
    bt = np.ones(N) if beta is None else np.asarray(beta, dtype=np.float64)
    blk = block_of_tokens(pos, block_frames) if block_frames > 0 else np.zeros(N, dtype=np.int64)
    nblk = int(blk.max()) + 1 if N else 0
    qp, kp = relu(q), relu(k)
    qr, kr = rope3d(qp, pos, bands, base), rope3d(kp, pos, bands, base)
    # inclusive states per block: each block's own sums, then the running sum over blocks
    Sb = np.zeros((nblk, d, d))
    zb = np.zeros((nblk, d))
    for b in range(nblk):
        sel = blk == b
        Sb[b] = (kr[sel] * bt[sel][:, None]).T @ v[sel]
        zb[b] = kp[sel].sum(axis=0)
    S = np.cumsum(Sb, axis=0)
    z = np.cumsum(zb, axis=0)
    num = np.empty((N, d))
    den = np.empty(N)
    for b in range(nblk):                        # each token reads its own block's state
        sel = blk == b
        num[sel] = qr[sel] @ S[b]
        den[sel] = qp[sel] @ z[b] + float(eps)
    y = num / den[:, None]
    sg = sigmoid(g)
    if rms is not None:
        gamma = np.ones(d) if rms[0] is None else np.asarray(rms[0], dtype=np.float64)
        r = np.sqrt(np.mean(y * y, axis=1) + float(rms[1]))
        yh = y / r[:, None]
        u = yh * gamma
    else:
        u = y
    dg = do * u * sg * (1.0 - sg)
    du = do * sg
    dgamma = None
    if rms is not None:
        if rms[0] is not None:
            dgamma = np.sum(du * yh, axis=0)
        dyh = du * gamma
        dy = (dyh - yh * np.sum(yh * dyh, axis=1, keepdims=True) / d) / r[:, None]
    else:
        dy = du
    dnum = dy / den[:, None]
    dden = -np.sum(dy * y, axis=1) / den
    dSb = np.zeros((nblk, d, d))
    dzb = np.zeros((nblk, d))
    for b in range(nblk):
        sel = blk == b
        dSb[b] = qr[sel].T @ dnum[sel]
        dzb[b] = qp[sel].T @ dden[sel]
    dSs = np.cumsum(dSb[::-1], axis=0)[::-1]     # suffix sums over blocks
    dzs = np.cumsum(dzb[::-1], axis=0)[::-1]
    dphq = np.empty((N, d))                      # dnum S_b^T
    P = np.empty((N, d))                         # v dS^{b T}
    kS = np.empty((N, d))                        # phi(k) dS^b
    for b in range(nblk):
        sel = blk == b
        dphq[sel] = dnum[sel] @ S[b].T
        P[sel] = v[sel] @ dSs[b].T
        kS[sel] = kr[sel] @ dSs[b]
    dq = (q > 0) * (rope3d_transpose(dphq, pos, bands, base) + dden[:, None] * z[blk])
    dv = bt[:, None] * kS
    dk = (k > 0) * (rope3d_transpose(bt[:, None] * P, pos, bands, base) + dzs[blk])
    dbeta = np.sum(kr * P, axis=1) if beta is not None else None
    return dq, dk, dv, dg, dbeta, dgamma


def backward_gated(Q, K, V, G, dO, grid, bands, base=10000.0, eps=1e-6, block_frames=0, beta=None, rms=None):
    """head_backward_gated over [B, H, N, d] inputs (beta: [B, H, N]).  Returns dQ, dK, dV, dG,
    dbeta ([B, H, N] or None) and dgamma ([d], summed over the heads, or None)."""
    T, Hh, W = grid
    pos = grid_positions(T, Hh, W)
    B, H, N, d = np.shape(Q)
    q, k, v, g, do = _heads(Q), _heads(K), _heads(V), _heads(G), _heads(dO)
    bt = None if beta is None else np.asarray(beta, dtype=np.float64).reshape(B * H, N)
    outs = [np.empty((B * H, N, d)) for _ in range(4)]
    dbeta = None if beta is None else np.empty((B * H, N))
    dgamma = None
    for u in range(B * H):
        r = head_backward_gated(q[u], k[u], v[u], g[u], do[u], pos, bands, base, eps, block_frames,
                                None if bt is None else bt[u], rms)
        for o, x in zip(outs, r[:4]):
            o[u] = x
        if dbeta is not None:
            dbeta[u] = r[4]
        if r[5] is not None:
            dgamma = r[5] if dgamma is None else dgamma + r[5]
    res = [o.reshape(B, H, N, d) for o in outs]
    return (*res, None if dbeta is None else dbeta.reshape(B, H, N), dgamma)


def backward_bidir(Q, K, V, G, dO, grid, bands, base=10000.0, eps=1e-6):
    """Gradients (dQ, dK, dV, dG) of the bidirectional mixer over [B, H, N, d] inputs."""
    T, Hh, W = grid
    pos = grid_positions(T, Hh, W)
    B, H, N, d = np.shape(Q)
    q, k, v, g, do = _heads(Q), _heads(K), _heads(V), _heads(G), _heads(dO)
    outs = [np.empty((B * H, N, d)) for _ in range(4)]
    for u in range(B * H):
        for o, r in zip(outs, head_backward(q[u], k[u], v[u], g[u], do[u], pos, bands, base, eps)):
            o[u] = r
    return tuple(o.reshape(B, H, N, d) for o in outs)
